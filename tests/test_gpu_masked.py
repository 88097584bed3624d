"""The masked grouped layout (expert e owns rows [e*cap, (e+1)*cap)) on the CUDA path
against the oracle's `permute_masked`: the bucketing bit-exact, the expert FFN and the
layer within the output bounds, overflow past cap reported and left out, and tiles
wholly past an expert's count skipped (their rows never written)."""
import numpy as np
import pytest
import torch

from mixture_experts_ffn_08_b200 import binding as B
from mixture_experts_ffn_08_b200 import inputs, workloads as W
from oracle import moe_oracle as o
from tests import parity as P

pytestmark = pytest.mark.gpu


def _ids(wl, seed, hot=None):
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.choice(wl.E, wl.K, replace=False) for _ in range(wl.T)]).astype(np.int32)
    if hot is not None:  # make expert `hot` the first choice of every token
        for t in range(wl.T):
            if hot not in ids[t]:
                ids[t, 0] = hot
    return ids


def _permute(wl, ids_np, d=None):
    p = B.params(wl)
    ws = P.alloc_ws(p)
    rows = B.moe_max_padded_rows(p)
    fp8 = wl.dtype == W.DTYPE_FP8
    if d is None:
        d = dict(x=torch.randn((wl.T, wl.H), device="cuda").to(torch.bfloat16))
    x = d["x_q"] if fp8 else d["x"]
    r = dict(counts=torch.empty(wl.E, dtype=torch.int32, device="cuda"),
             offs=torch.empty(wl.E + 1, dtype=torch.int32, device="cuda"),
             rop=torch.empty(wl.T * wl.K, dtype=torch.int32, device="cuda"),
             por=torch.full((rows,), 12345, dtype=torch.int32, device="cuda"),
             xp=torch.full((rows, wl.H), 7 if fp8 else 7.0, dtype=torch.uint8 if fp8 else torch.bfloat16,
                           device="cuda"),
             xps=torch.full((rows, wl.H // 128), 3.0, device="cuda") if fp8 else None, ws=ws, x=x)
    B.check(B.moe_permute(p, torch.as_tensor(ids_np, dtype=torch.int32, device="cuda"), x, d.get("x_scale"),
                          r["counts"], r["offs"], r["rop"], r["por"], r["xp"], r["xps"], ws, ws.numel()))
    torch.cuda.synchronize()
    return r


def _check_masked_perm(wl, ids_np, r):
    cap = wl.masked_cap
    counts, offs, rop, por, dropped = o.permute_masked(ids_np, wl.E, cap)
    assert r["counts"].cpu().numpy().tolist() == counts.tolist()
    assert r["offs"].cpu().numpy().tolist() == offs.tolist()
    assert r["rop"].cpu().numpy().tolist() == rop.tolist()
    assert r["por"].cpu().numpy().tolist() == por.tolist()
    status = B.moe_get_device_status(r["ws"])
    assert bool(status & B.MOE_DEV_CAPACITY) == (dropped > 0)
    # used rows hold their token's x; unused rows are left as they were
    used = np.where(por >= 0)[0]
    unused = np.where(por < 0)[0]
    xp = r["xp"]
    src = r["x"][torch.as_tensor(por[used] // wl.K, device="cuda", dtype=torch.long)]
    assert torch.equal(xp[torch.as_tensor(used, device="cuda")], src)
    fill = 7 if wl.dtype == W.DTYPE_FP8 else 7.0
    assert (xp[torch.as_tensor(unused, device="cuda")] == fill).all()
    return dropped


@pytest.mark.parametrize("T,E,K,cap", [(300, 16, 4, 128), (1000, 8, 2, 384), (200, 64, 6, 256)])
def test_masked_permute_matches_oracle(T, E, K, cap):
    wl = W.Workload("mp", T=T, H=256, I=128, E=E, K=K, masked_cap=cap)
    ids = _ids(wl, T)
    assert _check_masked_perm(wl, ids, _permute(wl, ids)) == 0


def test_masked_permute_overflow_is_reported_and_left_out():
    wl = W.Workload("mpo", T=700, H=128, I=128, E=8, K=2, masked_cap=256)
    ids = _ids(wl, 5, hot=3)  # expert 3 gets all 700 tokens, 444 past cap
    assert _check_masked_perm(wl, ids, _permute(wl, ids)) == 700 - 256


def test_masked_permute_fp8_scales():
    wl = W.Workload("mp8", T=300, H=512, I=128, E=16, K=4, dtype=W.DTYPE_FP8, masked_cap=128)
    d = inputs.make_inputs(wl, seed=1, device="cuda", weights=False)
    ids = _ids(wl, 1)
    r = _permute(wl, ids, d)
    _check_masked_perm(wl, ids, r)
    por = r["por"].cpu().numpy()
    used = np.where(por >= 0)[0]
    got = r["xps"][torch.as_tensor(used, device="cuda")]
    ref = d["x_scale"][torch.as_tensor(por[used] // wl.K, device="cuda", dtype=torch.long)]
    assert torch.equal(got, ref)


def _expert_ffn_masked(wl, d, ids_np, pass_offsets):
    r = _permute(wl, ids_np, d)
    p = B.params(wl)
    rows = B.moe_max_padded_rows(p)
    fp8 = wl.dtype == W.DTYPE_FP8
    y = torch.full((rows, wl.H), float("nan"), dtype=torch.bfloat16 if fp8 else torch.float32, device="cuda")
    a = P.device_inputs_ptrs(d, wl)
    B.check(B.moe_expert_ffn(p, r["xp"], r["xps"], r["offs"] if pass_offsets else None, r["counts"],
                             a["w_gate"], a["w_up"], a["w_down"], a["w_gate_scale"], a["w_up_scale"],
                             a["w_down_scale"], y, r["ws"], r["ws"].numel()))
    torch.cuda.synchronize()
    return r, y


@pytest.mark.parametrize("dtype,cap,pass_offsets", [(W.DTYPE_BF16, 128, True), (W.DTYPE_BF16, 512, False),
                                                    (W.DTYPE_FP8, 256, True), (W.DTYPE_FP8, 384, False)])
def test_masked_expert_ffn_matches_oracle_and_skips_empty_tiles(dtype, cap, pass_offsets):
    wl = W.Workload("mf", T=250, H=512, I=384, E=12, K=3, dtype=dtype, masked_cap=cap)
    d = inputs.make_inputs(wl, seed=2, device="cuda")
    ids = _ids(wl, 2)
    r, y = _expert_ffn_masked(wl, d, ids, pass_offsets)
    assert B.moe_get_device_status(r["ws"]) == 0
    fmt = o.activation_format(dtype)
    y_ref, rop_ref = o.expert_outputs(P.x_f64(d, wl), ids, P.expert_weights_fn(d, wl), wl.E, 1, h_format=fmt)
    rop = r["rop"].cpu().numpy()
    got = P.f64(y[torch.as_tensor(rop, device="cuda", dtype=torch.long)])
    P.check_close(got, y_ref[rop_ref], P.FP8_MAX_TOL if dtype == W.DTYPE_FP8 else P.BF16_MAX_TOL, "masked ffn")
    # rows of 128-row tiles that lie wholly past an expert's count are never written
    counts = r["counts"].cpu().numpy()
    yn = torch.isnan(y.float()).all(dim=1).cpu().numpy()
    for e in range(wl.E):
        first_empty = e * cap + (counts[e] + 127) // 128 * 128
        assert yn[first_empty:(e + 1) * cap].all()


@pytest.mark.parametrize("base", ["small_dsv3", "small_fp8"])
def test_masked_layer_matches_contiguous_layer(base):
    if base == "small_dsv3":
        wl = W.DSV3_PREFILL.with_(name="small_dsv3", T=200, H=512, I=256, E=32, n_group=4, topk_group=2,
                                  I_shared=256)
    else:
        wl = W.SKEWED_FP8.with_(name="small_fp8", T=300, H=512, I=384, E=16, K=4)
    d = inputs.make_inputs(wl, seed=3, device="cuda")
    contig = P.run_layer(wl, d)
    masked = P.run_layer(wl.with_(masked_cap=(wl.T + 127) // 128 * 128), d)
    assert B.moe_get_device_status(masked["ws"]) == 0
    assert torch.equal(contig["ids"], masked["ids"])
    # same per-pair arithmetic, same combine order: identical bits
    assert torch.equal(contig["out"], masked["out"])


def test_masked_layer_with_fused_combine():
    """Masked layout and the fused down + combine together: the same outputs as the
    contiguous deterministic layer within the bf16 bounds (atomics reorder the sums)."""
    wl = W.DSV3_PREFILL.with_(name="small_dsv3_fused", T=200, H=512, I=256, E=32, n_group=4, topk_group=2,
                              I_shared=256)
    d = inputs.make_inputs(wl, seed=5, device="cuda")
    ref = P.run_layer(wl, d)
    got = P.run_layer(wl.with_(masked_cap=256, fused_combine=True), d)
    assert B.moe_get_device_status(got["ws"]) == 0
    assert torch.equal(ref["ids"], got["ids"])
    P.check_close(P.f64(got["out"]), P.f64(ref["out"]), P.BF16_MAX_TOL, "masked fused")


def test_masked_layer_overflow_leaves_pairs_out():
    # a selection-only bias of +10 on expert 3 makes every token choose it: 400 pairs
    # for 128 rows (the weights still come from the unbiased scores)
    wl = W.Workload("mlo", T=400, H=256, I=256, E=8, K=2, masked_cap=128, has_bias=True)
    d = inputs.make_inputs(wl, seed=4, device="cuda")
    d["bias"] = torch.zeros(wl.E, device="cuda")
    d["bias"][3] = 10.0
    res = P.run_layer(wl, d)
    gpu_ids = res["ids"].cpu().numpy()
    counts, _, rop_m, _, dropped = o.permute_masked(gpu_ids, wl.E, wl.masked_cap)
    assert dropped > 0 and B.moe_get_device_status(res["ws"]) & B.MOE_DEV_CAPACITY
    assert res["counts"].cpu().numpy().tolist() == counts.tolist()
    x = P.x_f64(d, wl)
    s = o.scores(o.router_logits(x, P.f64(d["w_r"])), wl.score_fn)
    _, w_or = P.check_routing(gpu_ids, res["w"].cpu().numpy(), s, P.f64(d["bias"]), wl)
    assert (gpu_ids == 3).any(axis=1).all() and dropped == wl.T - wl.masked_cap
    y, rop_c = o.expert_outputs(x, gpu_ids, P.expert_weights_fn(d, wl), wl.E, 1, h_format="bf16")
    kept_rows = np.where(rop_m >= 0, rop_c, -1)
    ref = o.combine(y, kept_rows, w_or)
    P.check_close(P.f64(res["out"]), ref, P.BF16_MAX_TOL, "masked overflow layer")
