"""FP8 (e4m3, power-of-two block scales) expert FFN and layer against the fp64 oracle.

The oracle dequantises the e4m3 codes with their 1x128 / 128x128 scales, stores h in
e4m3 with one power-of-two scale per row and 128 columns, and is compared with the
block-scaled tcgen05 path under the FP8 bound (max |err| <= 6e-2 RMS, mean rel <= 5e-3)."""
import numpy as np
import pytest
import torch

from mixture_experts_ffn_08_b200 import binding as B
from mixture_experts_ffn_08_b200 import inputs, workloads as W
from oracle import moe_oracle as o
from tests import parity as P

pytestmark = pytest.mark.gpu
BM = B.BLOCK_M


def _permute_fp8(wl, ids_np, d):
    p = B.params(wl)
    ws = P.alloc_ws(p)
    rows = B.moe_max_padded_rows(p)
    ids = torch.as_tensor(ids_np, dtype=torch.int32, device="cuda")
    r = dict(counts=torch.empty(wl.E, dtype=torch.int32, device="cuda"),
             offs=torch.empty(wl.E + 1, dtype=torch.int32, device="cuda"),
             rop=torch.empty(wl.T * wl.K, dtype=torch.int32, device="cuda"),
             por=torch.empty(rows, dtype=torch.int32, device="cuda"),
             xp=torch.empty((rows, wl.H), dtype=torch.uint8, device="cuda"),
             xps=torch.empty((rows, wl.H // 128), dtype=torch.float32, device="cuda"), ws=ws)
    B.check(B.moe_permute(p, ids, d["x_q"], d["x_scale"], r["counts"], r["offs"], r["rop"], r["por"],
                          r["xp"], r["xps"], ws, ws.numel()))
    return r


def _expert_ffn_fp8(wl, d, ids_np):
    r = _permute_fp8(wl, ids_np, d)
    p = B.params(wl)
    rows = B.moe_max_padded_rows(p)
    y = torch.full((rows, wl.H), float("nan"), dtype=torch.bfloat16, device="cuda")
    B.check(B.moe_expert_ffn(p, r["xp"], r["xps"], r["offs"], r["counts"], d["w_gate_q"], d["w_up_q"],
                             d["w_down_q"], d["w_gate_s"], d["w_up_s"], d["w_down_s"], y, r["ws"],
                             r["ws"].numel()))
    torch.cuda.synchronize()
    assert B.moe_get_device_status(r["ws"]) == 0
    return r, y


def _check_vs_oracle(wl, d, ids_np, r, y):
    x = P.x_f64(d, wl)
    ref, _ = o.expert_outputs(x, ids_np, P.expert_weights_fn(d, wl), wl.E,
                              B.moe_effective_block_m(B.params(wl)), h_format="e4m3")
    offs = r["offs"].cpu().numpy()
    total = offs[wl.E]
    real = r["por"].cpu().numpy()[:total] >= 0
    got = P.f64(y[:total])
    return P.check_close(got[real], ref[real], P.FP8_MAX_TOL, "fp8 y_perm")


def _unit_scale_inputs(wl, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)

    def codes(shape, std):
        v = torch.randn(shape, generator=g, device="cuda") * std
        return v.to(torch.float8_e4m3fn).view(torch.uint8)

    E, H, I, T = wl.E, wl.H, wl.I, wl.T
    return dict(x_q=codes((T, H), 1.0), x_scale=torch.ones((T, H // 128), device="cuda"),
                w_gate_q=codes((E, I, H), 0.05), w_up_q=codes((E, I, H), 0.05), w_down_q=codes((E, H, I), 0.05),
                w_gate_s=torch.ones((E, I // 128, H // 128), device="cuda"),
                w_up_s=torch.ones((E, I // 128, H // 128), device="cuda"),
                w_down_s=torch.ones((E, H // 128, I // 128), device="cuda"))


@pytest.mark.parametrize("E,K,T,H,I", [(1, 1, 200, 256, 256), (4, 2, 300, 512, 384)])
def test_fp8_expert_ffn_unit_scales(E, K, T, H, I):
    wl = W.Workload("f8u", T=T, H=H, I=I, E=E, K=K, dtype=W.DTYPE_FP8)
    d = _unit_scale_inputs(wl, 3)
    rng = np.random.default_rng(3)
    ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    r, y = _expert_ffn_fp8(wl, d, ids)
    _check_vs_oracle(wl, d, ids, r, y)


@pytest.mark.parametrize("E,K,T,H,I,bm", [(1, 1, 200, 256, 256, 0), (6, 2, 500, 512, 384, 0),
                                          (16, 4, 300, 1024, 768, 0), (1, 1, 300, 256, 256, 256),
                                          (6, 2, 700, 512, 384, 256), (3, 3, 600, 1024, 768, 256)])
def test_fp8_expert_ffn_block_scales(E, K, T, H, I, bm):
    wl = W.Workload("f8", T=T, H=H, I=I, E=E, K=K, dtype=W.DTYPE_FP8, block_m=bm)
    d = inputs.make_inputs(wl, seed=4, device="cuda")
    rng = np.random.default_rng(4)
    ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    r, y = _expert_ffn_fp8(wl, d, ids)
    _check_vs_oracle(wl, d, ids, r, y)


SMALL_FP8 = W.SKEWED_FP8.with_(name="skewed_fp8_small", T=600, H=512, I=384, E=16, K=4)


@pytest.mark.parametrize("bm", [0, 256])
def test_fp8_layer_small_all_elements(bm):
    wl = SMALL_FP8.with_(block_m=bm)
    d = inputs.make_inputs(wl, seed=0, device="cuda")
    res = P.run_layer(wl, d)
    assert B.moe_get_device_status(res["ws"]) == 0
    gpu_ids = res["ids"].cpu().numpy()
    x = P.x_f64(d, wl)
    s = o.scores(o.router_logits(x, P.f64(d["w_r"])), wl.score_fn)
    _, w_or = P.check_routing(gpu_ids, res["w"].cpu().numpy(), s, None, wl)
    ref = o.forward_given_routing(x, gpu_ids, w_or, P.expert_weights_fn(d, wl), wl.E, None, h_format="e4m3")
    P.check_close(P.f64(res["out"]), ref, P.FP8_MAX_TOL, wl.name)


def test_fp8_layer_full_size_sampled():
    wl = W.SKEWED_FP8
    d = inputs.make_inputs(wl, seed=0, device="cuda")
    res = P.run_layer(wl, d)
    assert B.moe_get_device_status(res["ws"]) == 0
    gpu_ids = res["ids"].cpu().numpy()
    x = P.x_f64(d, wl)
    s = o.scores(o.router_logits(x, P.f64(d["w_r"])), wl.score_fn)
    n_mism, w_or = P.check_routing(gpu_ids, res["w"].cpu().numpy(), s, None, wl)
    assert n_mism <= max(2, wl.T // 1000)
    counts = res["counts"].cpu().numpy()
    assert counts.sum() == wl.T * wl.K and counts.max() >= 0.85 * wl.T
    # rows spread over the hot expert's bucket (~15k rows, ~120 M-tiles), the last
    # partial M-tile of several other experts, and a few uniform draws
    toks = P.stratified_tokens(gpu_ids, wl.E, np.random.default_rng(0), n_random=4, n_tail_experts=6,
                               hot_rows=16)
    hot = int(np.argmax(counts))
    assert (gpu_ids[toks] == hot).any(axis=1).sum() >= 16
    ref = o.forward_given_routing(x[toks], gpu_ids[toks], w_or[toks], P.expert_weights_fn(d, wl), wl.E, None,
                                  h_format="e4m3")
    got = P.f64(res["out"][torch.as_tensor(toks, device="cuda")])
    P.check_close(got, ref, P.FP8_MAX_TOL, f"{wl.name} ({len(toks)} tokens)")


def test_fp8_host_entry_point_matches_device_entry_point():
    wl = SMALL_FP8
    d = inputs.make_inputs(wl, seed=2, device="cuda")
    res = P.run_layer(wl, d)
    p = B.params(wl)
    a = P.device_inputs_ptrs(d, wl)
    out_host = torch.empty((wl.T, wl.H), dtype=torch.bfloat16).pin_memory()
    B.check(B.moe_layer_forward_host(p, d["x_q"].cpu().pin_memory(), d["x_scale"].cpu().pin_memory(),
                                     a["w_r"], None, a["w_gate"], a["w_up"], a["w_down"], a["w_gate_scale"],
                                     a["w_up_scale"], a["w_down_scale"], None, None, None, out_host,
                                     res["ws"], res["ws"].numel()))
    torch.cuda.synchronize()
    assert torch.equal(out_host, res["out"].cpu())
