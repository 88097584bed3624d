"""FP8 x FP4 expert GEMMs (e4m3 activations, e2m1 weights with a UE8M0 scale per 32 K
elements) against the fp64 oracle: the scale-atom preparation bit-exact, the expert FFN
and the layer within the FP8 bound (max |err| <= 6e-2 RMS, mean rel <= 5e-3)."""
import numpy as np
import pytest
import torch

from mixture_experts_ffn_08_b200 import binding as B
from mixture_experts_ffn_08_b200 import inputs, workloads as W
from oracle import moe_oracle as o
from tests import parity as P

pytestmark = pytest.mark.gpu


def _atom_offset(m):
    return 16 * (m % 32) + 4 * (m // 32)


def test_fp4_scale_atoms_layout():
    rows, K = 256, 512
    g = torch.Generator(device="cuda").manual_seed(0)
    sb = torch.randint(0, 256, (rows, K // 32), generator=g, device="cuda", dtype=torch.int32).to(torch.uint8)
    atoms = torch.full((rows * K // 32,), 0xEE, dtype=torch.uint8, device="cuda")
    B.check(B.moe_prepare_fp4_scales(sb, rows, K, atoms))
    torch.cuda.synchronize()
    a = atoms.cpu().numpy().reshape(rows // 128, K // 128, 512)
    s = sb.cpu().numpy()
    for r in range(rows):
        for kb in range(K // 128):
            off = _atom_offset(r % 128)
            assert a[r // 128, kb, off:off + 4].tolist() == s[r, 4 * kb:4 * kb + 4].tolist()


def test_fp4_prepare_rejects_bad_sizes():
    t = torch.empty(4096, dtype=torch.uint8, device="cuda")
    assert B.moe_prepare_fp4_scales(t, 100, 128, t) == 1      # rows not a multiple of 128
    assert B.moe_prepare_fp4_scales(t, 128, 96, t) == 1       # K not a multiple of 128


def _permute(wl, ids_np, d):
    p = B.params(wl)
    ws = P.alloc_ws(p)
    rows = B.moe_max_padded_rows(p)
    r = dict(counts=torch.empty(wl.E, dtype=torch.int32, device="cuda"),
             offs=torch.empty(wl.E + 1, dtype=torch.int32, device="cuda"),
             rop=torch.empty(wl.T * wl.K, dtype=torch.int32, device="cuda"),
             por=torch.empty(rows, dtype=torch.int32, device="cuda"),
             xp=torch.empty((rows, wl.H), dtype=torch.uint8, device="cuda"),
             xps=torch.empty((rows, wl.H // 128), dtype=torch.float32, device="cuda"), ws=ws)
    B.check(B.moe_permute(p, torch.as_tensor(ids_np, dtype=torch.int32, device="cuda"), d["x_q"], d["x_scale"],
                          r["counts"], r["offs"], r["rop"], r["por"], r["xp"], r["xps"], ws, ws.numel()))
    return r


def _expert_ffn(wl, d, ids_np):
    r = _permute(wl, ids_np, d)
    p = B.params(wl)
    rows = B.moe_max_padded_rows(p)
    a = P.device_inputs_ptrs(d, wl)
    y = torch.full((rows, wl.H), float("nan"), dtype=torch.bfloat16, device="cuda")
    B.check(B.moe_expert_ffn(p, r["xp"], r["xps"], r["offs"], r["counts"], a["w_gate"], a["w_up"], a["w_down"],
                             a["w_gate_scale"], a["w_up_scale"], a["w_down_scale"], y, r["ws"], r["ws"].numel()))
    torch.cuda.synchronize()
    assert B.moe_get_device_status(r["ws"]) == 0
    return r, y


def _check_ffn(wl, d, ids, r, y):
    ref, rop_ref = o.expert_outputs(P.x_f64(d, wl), ids, P.expert_weights_fn(d, wl), wl.E, 1, h_format="e4m3")
    rop = r["rop"].cpu().numpy()
    got = P.f64(y[torch.as_tensor(rop, device="cuda", dtype=torch.long)])
    P.check_close(got, ref[rop_ref], P.FP8_MAX_TOL, "fp4 y_perm")


def _ids(wl, seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.choice(wl.E, wl.K, replace=False) for _ in range(wl.T)]).astype(np.int32)


def test_fp4_expert_ffn_unit_scales_all_codes():
    """Unit scales (byte 127) and weight codes drawn from all 16 e2m1 values."""
    wl = W.Workload("f4u", T=200, H=256, I=256, E=2, K=1, dtype=W.DTYPE_FP8_FP4)
    d = inputs.make_inputs(wl, seed=5, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(5)
    for n in ("w_gate", "w_up", "w_down"):
        d[n + "_q"] = torch.randint(0, 256, d[n + "_q"].shape, generator=g, device="cuda",
                                    dtype=torch.int32).to(torch.uint8)
        d[n + "_s"] = torch.full_like(d[n + "_s"], 127 - 5)   # 2^-5: keeps the activations moderate
    ids = _ids(wl, 5)
    r, y = _expert_ffn(wl, d, ids)
    _check_ffn(wl, d, ids, r, y)


@pytest.mark.parametrize("E,K,T,H,I", [(1, 1, 200, 256, 256), (6, 2, 500, 512, 384), (8, 4, 300, 384, 512),
                                       (16, 4, 300, 1024, 768)])
def test_fp4_expert_ffn_block_scales(E, K, T, H, I):
    wl = W.Workload("f4", T=T, H=H, I=I, E=E, K=K, dtype=W.DTYPE_FP8_FP4)
    d = inputs.make_inputs(wl, seed=6, device="cuda")
    ids = _ids(wl, 6)
    r, y = _expert_ffn(wl, d, ids)
    _check_ffn(wl, d, ids, r, y)


SMALL_FP4 = W.DSV3_DECODE_FP4.with_(name="dsv3_fp4_small", T=300, H=512, I=256, E=32, n_group=4, topk_group=2)


@pytest.mark.parametrize("masked", [False, True])
def test_fp4_layer_small_all_elements(masked):
    wl = SMALL_FP4.with_(masked_cap=384 if masked else 0)
    d = inputs.make_inputs(wl, seed=7, device="cuda")
    res = P.run_layer(wl, d)
    assert B.moe_get_device_status(res["ws"]) == 0
    gpu_ids = res["ids"].cpu().numpy()
    x = P.x_f64(d, wl)
    s = o.scores(o.router_logits(x, P.f64(d["w_r"])), wl.score_fn)
    _, w_or = P.check_routing(gpu_ids, res["w"].cpu().numpy(), s, P.f64(d["bias"]), wl)
    ref = o.forward_given_routing(x, gpu_ids, w_or, P.expert_weights_fn(d, wl), wl.E, None, h_format="e4m3")
    P.check_close(P.f64(res["out"]), ref, P.FP8_MAX_TOL, wl.name)


def test_fp4_layer_full_size_decode_sampled():
    wl = W.DSV3_DECODE_FP4
    d = inputs.make_inputs(wl, seed=0, device="cuda")
    res = P.run_layer(wl, d)
    assert B.moe_get_device_status(res["ws"]) == 0
    gpu_ids = res["ids"].cpu().numpy()
    x = P.x_f64(d, wl)
    s = o.scores(o.router_logits(x, P.f64(d["w_r"])), wl.score_fn)
    n_mism, w_or = P.check_routing(gpu_ids, res["w"].cpu().numpy(), s, P.f64(d["bias"]), wl)
    assert n_mism <= 2
    toks = P.stratified_tokens(gpu_ids, wl.E, np.random.default_rng(0), n_random=8, n_tail_experts=8, hot_rows=4)
    ref = o.forward_given_routing(x[toks], gpu_ids[toks], w_or[toks], P.expert_weights_fn(d, wl), wl.E, None,
                                  h_format="e4m3")
    got = P.f64(res["out"][torch.as_tensor(toks, device="cuda")])
    P.check_close(got, ref, P.FP8_MAX_TOL, f"{wl.name} ({len(toks)} tokens)")


# ---------------------------------------------------------------- few tokens per expert
# Decode-like shapes (at most 32 pairs per expert on average): M-tiles that are mostly pad
# rows, experts with no token, and buckets of one or two partial 32-row groups.

def _ids_from_counts(counts, seed):
    ids = np.concatenate([np.full(n, e) for e, n in enumerate(counts)]).astype(np.int32)
    np.random.default_rng(seed).shuffle(ids)
    return ids[:, None]


@pytest.mark.parametrize("E,K,T,H,I", [(32, 4, 64, 512, 384), (16, 2, 200, 256, 256), (64, 6, 100, 1024, 768)])
def test_fp4_few_tokens_expert_ffn(E, K, T, H, I):
    wl = W.Workload("f4s", T=T, H=H, I=I, E=E, K=K, dtype=W.DTYPE_FP8_FP4)
    d = inputs.make_inputs(wl, seed=8, device="cuda")
    ids = _ids(wl, 8)
    r, y = _expert_ffn(wl, d, ids)
    _check_ffn(wl, d, ids, r, y)


def test_fp4_bucket_edges():
    """Experts with 0, 1, 31, 32, 33, 64 and 65 tokens: empty buckets and buckets just
    under, at and over multiples of 32 rows inside one 128-row M-tile."""
    counts = [0, 1, 31, 32, 33, 64, 65, 0]
    wl = W.Workload("f4e", T=sum(counts), H=256, I=256, E=len(counts), K=1, dtype=W.DTYPE_FP8_FP4)
    d = inputs.make_inputs(wl, seed=9, device="cuda")
    ids = _ids_from_counts(counts, 9)
    r, y = _expert_ffn(wl, d, ids)
    assert r["counts"].cpu().numpy().tolist() == counts
    _check_ffn(wl, d, ids, r, y)


@pytest.mark.parametrize("masked", [False, True])
def test_fp4_decode_like_layer_small_all_elements(masked):
    wl = SMALL_FP4.with_(name="dsv3_fp4_decode_small", T=100, masked_cap=128 if masked else 0)
    d = inputs.make_inputs(wl, seed=10, device="cuda")
    res = P.run_layer(wl, d)
    assert B.moe_get_device_status(res["ws"]) == 0
    gpu_ids = res["ids"].cpu().numpy()
    x = P.x_f64(d, wl)
    s = o.scores(o.router_logits(x, P.f64(d["w_r"])), wl.score_fn)
    _, w_or = P.check_routing(gpu_ids, res["w"].cpu().numpy(), s, P.f64(d["bias"]), wl)
    ref = o.forward_given_routing(x, gpu_ids, w_or, P.expert_weights_fn(d, wl), wl.E, None, h_format="e4m3")
    P.check_close(P.f64(res["out"]), ref, P.FP8_MAX_TOL, wl.name)
