"""Stage-by-stage parity of the CUDA path (moe_route, moe_permute, moe_expert_ffn,
moe_shared_expert_ffn, moe_combine) against the fp64 oracle, with edge cases."""
import numpy as np
import pytest
import torch

from mixture_experts_ffn_08_b200 import binding as B
from mixture_experts_ffn_08_b200 import inputs, workloads as W
from oracle import moe_oracle as o
from tests import parity as P

pytestmark = pytest.mark.gpu

BM = B.BLOCK_M


def _ws(wl):
    return P.alloc_ws(B.params(wl))


# ------------------------------------------------------------------ routing
ROUTE_CASES = {
    "tiny": W.TINY,
    "mixtral_full": W.MIXTRAL_PREFILL,
    "dsv3_full": W.DSV3_PREFILL,
    "skewed_fp8_full": W.SKEWED_FP8,
    "grouped_softmax_kernelswift": W.Workload("kernelswift", T=83, H=7168, I=128, E=256, K=8,
                                              n_group=8, topk_group=4, group_topn=1),
    "sigmoid_no_renorm": W.Workload("sig", T=333, H=384, I=128, E=64, K=6, score_fn=W.SCORE_SIGMOID,
                                    renormalize=False, routed_scale=1.5),
    "e_1000": W.Workload("e1000", T=50, H=256, I=128, E=1000, K=32, n_group=8, topk_group=5,
                         group_topn=3, has_bias=True),
    # few output tiles: the router GEMM splits the H reduction into K-slices (28 here)
    "dsv3_decode_full": W.DSV3_DECODE,
    # 5 K-slices over 22 K-blocks of 64: slices of 4 and 5 blocks
    "split_uneven": W.Workload("split5", T=300, H=1408, I=128, E=96, K=4, score_fn=W.SCORE_SIGMOID,
                               has_bias=True),
}


@pytest.mark.parametrize("name", list(ROUTE_CASES))
def test_route(name):
    wl = ROUTE_CASES[name]
    d = inputs.make_inputs(wl, seed=0, device="cuda", weights=False)
    p = B.params(wl)
    ws = _ws(wl)
    ids = torch.empty((wl.T, wl.K), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.K), dtype=torch.float32, device="cuda")
    x = d["x_q"] if wl.dtype == W.DTYPE_FP8 else d["x"]
    B.check(B.moe_route(p, x, d.get("x_scale"), d["w_r"], d["bias"], ids, w, ws, ws.numel()))
    torch.cuda.synchronize()
    xs = P.x_f64(d, wl)
    s = o.scores(o.router_logits(xs, P.f64(d["w_r"])), wl.score_fn)
    bias = P.f64(d["bias"]) if d["bias"] is not None else None
    n_mism, _ = P.check_routing(ids.cpu().numpy(), w.cpu().numpy(), s, bias, wl)
    assert n_mism <= max(2, wl.T // 1000)
    if wl.skewed:
        counts = np.bincount(ids.cpu().numpy().ravel(), minlength=wl.E)
        assert counts.max() >= 0.85 * wl.T


def test_route_exact_ties_pick_lower_index():
    # All logits equal: every expert ties; ids must be 0..K-1 in order with equal weights.
    wl = W.Workload("ties", T=40, H=128, I=128, E=16, K=4)
    p = B.params(wl)
    ws = _ws(wl)
    x = torch.zeros((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    w_r = torch.ones((wl.E, wl.H), dtype=torch.bfloat16, device="cuda")
    ids = torch.empty((wl.T, wl.K), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.K), dtype=torch.float32, device="cuda")
    B.check(B.moe_route(p, x, None, w_r, None, ids, w, ws, ws.numel()))
    torch.cuda.synchronize()
    assert (ids.cpu().numpy() == np.arange(4)[None, :]).all()
    np.testing.assert_allclose(w.cpu().numpy(), 0.25, rtol=1e-6)


# ------------------------------------------------------------------ permutation
def _permute(wl, ids_np, x=None):
    p = B.params(wl)
    ws = _ws(wl)
    rows = B.moe_max_padded_rows(p)
    ids = torch.as_tensor(ids_np, dtype=torch.int32, device="cuda")
    if x is None:
        x = torch.randn((wl.T, wl.H), device="cuda").to(torch.bfloat16)
    counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    offs = torch.empty(wl.E + 1, dtype=torch.int32, device="cuda")
    rop = torch.empty(wl.T * wl.K, dtype=torch.int32, device="cuda")
    por = torch.full((rows,), 12345, dtype=torch.int32, device="cuda")
    xp = torch.full((rows, wl.H), 7.0, dtype=torch.bfloat16, device="cuda")
    B.check(B.moe_permute(p, ids, x, None, counts, offs, rop, por, xp, None, ws, ws.numel()))
    torch.cuda.synchronize()
    return dict(x=x, counts=counts.cpu().numpy(), offs=offs.cpu().numpy(), rop=rop.cpu().numpy(),
                por=por.cpu().numpy(), xp=xp, ws=ws)


def _check_perm(wl, ids_np, r):
    P.check_permutation(ids_np, wl.E, r["counts"], r["offs"], r["rop"], r["por"],
                        B.moe_effective_block_m(B.params(wl)))
    total = r["offs"][wl.E]
    por = r["por"][:total]
    real = por >= 0
    xp = r["xp"][:total]
    src = r["x"][torch.as_tensor(por[real] // wl.K, device="cuda", dtype=torch.long)]
    assert torch.equal(xp[torch.as_tensor(np.where(real)[0], device="cuda")], src)
    assert (xp[torch.as_tensor(np.where(~real)[0], device="cuda")] == 0).all()


@pytest.mark.parametrize("seed,block_m", [(0, 0), (1, 0), (2, 256)])
def test_permute_random(seed, block_m):
    wl = W.Workload("perm", T=3000, H=256, I=128, E=64, K=6, block_m=block_m)
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.choice(wl.E, wl.K, replace=False) for _ in range(wl.T)]).astype(np.int32)
    r = _permute(wl, ids)
    _check_perm(wl, ids, r)
    assert B.moe_get_device_status(r["ws"]) == 0


@pytest.mark.parametrize("E,K,T,cap", [(1000, 2, 1000, 0), (1024, 4, 512, 0), (16, 8, 256, 128)])
def test_permute_one_block_path_many_experts(E, K, T, cap):
    """At most 2048 pairs: one block counts, scans and ranks; up to 1024 experts, and the
    masked layout's capacity."""
    wl = W.Workload("perm1", T=T, H=128, I=128, E=E, K=K, masked_cap=cap)
    rng = np.random.default_rng(E + K)
    ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    if cap:
        p = B.params(wl)
        ws = _ws(wl)
        rows = B.moe_max_padded_rows(p)
        d_ids = torch.as_tensor(ids, device="cuda")
        x = torch.randn((T, wl.H), device="cuda").to(torch.bfloat16)
        counts = torch.empty(E, dtype=torch.int32, device="cuda")
        offs = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        rop = torch.empty(T * K, dtype=torch.int32, device="cuda")
        por = torch.empty(rows, dtype=torch.int32, device="cuda")
        xp = torch.empty((rows, wl.H), dtype=torch.bfloat16, device="cuda")
        B.check(B.moe_permute(p, d_ids, x, None, counts, offs, rop, por, xp, None, ws, ws.numel()))
        torch.cuda.synchronize()
        o_counts, o_offs, o_rop, o_por, _ = o.permute_masked(ids, E, cap)   # some experts overflow cap
        np.testing.assert_array_equal(offs.cpu().numpy(), o_offs)
        np.testing.assert_array_equal(counts.cpu().numpy(), o_counts)
        np.testing.assert_array_equal(rop.cpu().numpy(), o_rop)
        np.testing.assert_array_equal(por.cpu().numpy(), o_por)
        return
    r = _permute(wl, ids)
    _check_perm(wl, ids, r)


@pytest.mark.parametrize("E,K,T", [(1, 1, 5000), (3, 2, 4000), (96, 8, 9000), (1000, 4, 3000), (1024, 8, 4096)])
def test_permute_chunked_scan(E, K, T):
    """More than 2048 pairs: count per 256-pair chunk, scan, rank.  The scan spreads each
    expert's chunks over 1024 // E threads: 1024 of them for one expert, 341 for three (more
    threads than chunks), 10 for 96 (ranges of 29 chunks), one for 1000 and 1024 experts."""
    wl = W.Workload("perm_chunked", T=T, H=128, I=128, E=E, K=K)
    rng = np.random.default_rng(E * 7 + K)
    ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    r = _permute(wl, ids)
    _check_perm(wl, ids, r)
    assert B.moe_get_device_status(r["ws"]) == 0


def test_permute_bucket_edge_sizes():
    # experts with 0, 1, BM-1, BM, BM+1, 2*BM+5 rows (K = 1 so counts are set directly)
    sizes = [0, 1, BM - 1, BM, BM + 1, 2 * BM + 5, 0, 3]
    ids = np.concatenate([np.full(n, e) for e, n in enumerate(sizes)]).astype(np.int32)
    rng = np.random.default_rng(3)
    rng.shuffle(ids)
    wl = W.Workload("edges", T=len(ids), H=128, I=128, E=len(sizes), K=1)
    r = _permute(wl, ids[:, None])
    _check_perm(wl, ids[:, None], r)
    assert r["counts"].tolist() == sizes


@pytest.mark.parametrize("cap", [0, 256])
def test_permute_empty_batch(cap):
    """T = 0: no pairs.  counts are all 0, offsets 0 (contiguous) or e*cap (masked),
    every masked row is marked unused, and x_perm is left as it was."""
    wl = W.Workload("empty", T=0, H=256, I=128, E=8, K=2, masked_cap=cap)
    r = _permute(wl, np.zeros((0, wl.K), dtype=np.int32))
    assert B.moe_get_device_status(r["ws"]) == 0
    assert r["counts"].tolist() == [0] * wl.E
    assert r["offs"].tolist() == [e * cap for e in range(wl.E + 1)]
    assert (r["por"] == (-1 if cap else 12345)).all()
    assert (r["xp"] == 7.0).all()


def test_layer_empty_batch_zeroes_counts():
    wl = W.DSV3_PREFILL.with_(name="empty_layer", T=0, H=512, I=256, E=32, I_shared=256)
    d = inputs.make_inputs(wl, seed=0, device="cuda")
    p = B.params(wl)
    ws = _ws(wl)
    a = P.device_inputs_ptrs(d, wl)
    counts = torch.full((wl.E,), 77, dtype=torch.int32, device="cuda")
    out = torch.empty((0, wl.H), dtype=torch.bfloat16, device="cuda")
    B.check(B.moe_layer_forward(p, a["x"], a["x_scale"], a["w_r"], a["bias"], a["w_gate"], a["w_up"],
                                a["w_down"], a["w_gate_scale"], a["w_up_scale"], a["w_down_scale"],
                                a["ws_gate"], a["ws_up"], a["ws_down"], out, None, None, counts, ws,
                                ws.numel()))
    torch.cuda.synchronize()
    assert counts.tolist() == [0] * wl.E
    assert B.moe_get_device_status(ws) == 0


def test_permute_page_bucket_example():
    from tests.conftest import load_golden
    g = load_golden("bucket_example.txt")
    ids = np.array([e for (_, e) in g["pairs"]], dtype=np.int32).reshape(g["T"], g["K"])
    wl = W.Workload("page", T=g["T"], H=128, I=128, E=g["E"], K=g["K"])
    r = _permute(wl, ids)
    assert r["counts"].tolist() == g["counts"]
    for e in range(g["E"]):
        rows = range(r["offs"][e], r["offs"][e] + r["counts"][e])
        assert [int(r["por"][q]) // g["K"] for q in rows] == g["buckets"][e]


def test_permute_bad_ids_are_reported_and_skipped():
    wl = W.Workload("bad", T=100, H=128, I=128, E=8, K=2)
    rng = np.random.default_rng(4)
    ids = np.stack([rng.choice(wl.E, wl.K, replace=False) for _ in range(wl.T)]).astype(np.int32)
    ids[5, 1] = 8
    ids[70, 0] = -3
    r = _permute(wl, ids)
    assert B.moe_get_device_status(r["ws"]) & B.MOE_DEV_BAD_EXPERT_ID
    assert r["counts"].sum() == wl.T * wl.K - 2
    assert r["rop"][5 * 2 + 1] == -1 and r["rop"][70 * 2] == -1
    good = ids.copy()
    good[5, 1] = -1
    good[70, 0] = -1
    flat = good.ravel()
    for e in range(wl.E):
        rows = range(r["offs"][e], r["offs"][e] + r["counts"][e])
        assert [int(r["por"][q]) for q in rows] == [p for p in range(flat.size) if flat[p] == e]


# ------------------------------------------------------------------ expert FFN
@pytest.mark.parametrize("E,K,T,H,I,bm", [(1, 1, 300, 256, 128, 0), (6, 2, 700, 384, 256, 0),
                                          (16, 4, 64, 512, 384, 0), (3, 3, 129, 1024, 640, 0),
                                          (4, 2, 1200, 512, 256, 0),  # two-M-tile gate/up and down kernels
                                          (1, 1, 300, 256, 128, 256), (6, 2, 700, 512, 256, 256),
                                          (3, 3, 700, 384, 640, 256)])
def test_expert_ffn_grouped_gemm(E, K, T, H, I, bm):
    wl = W.Workload("ffn", T=T, H=H, I=I, E=E, K=K, block_m=bm)
    d = inputs.make_inputs(wl, seed=5, device="cuda")
    rng = np.random.default_rng(5)
    ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    r = _permute(wl, ids, x=d["x"])
    p = B.params(wl)
    rows = B.moe_max_padded_rows(p)
    offs = torch.as_tensor(r["offs"], device="cuda")
    counts = torch.as_tensor(r["counts"], device="cuda")
    ew = P.expert_weights_fn(d, wl)
    ref, _ = o.expert_outputs(P.f64(d["x"]), ids, ew, E, B.moe_effective_block_m(p), h_format="bf16")
    ref_exact, _ = o.expert_outputs(P.f64(d["x"]), ids, ew, E, B.moe_effective_block_m(p), h_format=None)
    total = r["offs"][E]
    real = r["por"][:total] >= 0
    # with counts: pad rows are left untouched; without: they are computed (zero input -> 0)
    for cnt in (counts, None):
        y = torch.full((rows, H), float("nan"), dtype=torch.float32, device="cuda")
        B.check(B.moe_expert_ffn(p, r["xp"], None, offs, cnt, d["w_gate"], d["w_up"], d["w_down"], None,
                                 None, None, y, r["ws"], r["ws"].numel()))
        torch.cuda.synchronize()
        assert B.moe_get_device_status(r["ws"]) == 0
        got = P.f64(y[:total])
        # y_perm is fp32: against the exact-h oracle only h's bf16 storage separates them
        P.check_both_oracles(got[real], ref[real], ref_exact[real], P.BF16_MAX_TOL,
                             f"y_perm E{E} K{K} T{T} H{H} I{I} bm{bm}", exact_max=True)
        if cnt is None:
            assert np.all(got[~real] == 0)
        else:
            assert np.all(np.isnan(got[~real]))


def test_shared_expert_dense_ffn_ragged_T():
    wl = W.Workload("sh", T=200, H=512, I=128, E=4, K=1, I_shared=384)
    d = inputs.make_inputs(wl, seed=6, device="cuda")
    p = B.params(wl)
    ws = _ws(wl)
    y = torch.empty((wl.T, wl.H), dtype=torch.float32, device="cuda")
    B.check(B.moe_shared_expert_ffn(p, d["x"], d["ws_gate"], d["ws_up"], d["ws_down"], y, ws, ws.numel()))
    torch.cuda.synchronize()
    ref = o.swiglu_ffn(P.f64(d["x"]), *P.shared_weights(d, wl), h_format="bf16")
    ref_exact = o.swiglu_ffn(P.f64(d["x"]), *P.shared_weights(d, wl), h_format=None)
    P.check_both_oracles(P.f64(y), ref, ref_exact, P.BF16_MAX_TOL, "shared expert y (fp32)", exact_max=True)


# ------------------------------------------------------------------ combine
def test_combine_identity_experts_return_x_and_is_bitwise_reproducible():
    wl = W.Workload("comb", T=500, H=1024, I=128, E=16, K=4)
    rng = np.random.default_rng(7)
    ids = np.stack([rng.choice(wl.E, wl.K, replace=False) for _ in range(wl.T)]).astype(np.int32)
    x = torch.randn((wl.T, wl.H), device="cuda").to(torch.bfloat16)
    r = _permute(wl, ids, x=x)
    w = torch.as_tensor(rng.dirichlet(np.ones(wl.K), size=wl.T), dtype=torch.float32, device="cuda")
    p = B.params(wl)
    out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    rop = torch.as_tensor(r["rop"], device="cuda")
    yp = r["xp"].float()                                         # identity experts: y = x
    B.check(B.moe_combine(p, yp, rop, w, None, out))
    torch.cuda.synchronize()
    ref = P.f64(x) * P.f64(w).sum(axis=1, keepdims=True)
    np.testing.assert_allclose(P.f64(out), ref, rtol=2 ** -7, atol=1e-6)
    first = out.clone()
    for _ in range(10):
        B.check(B.moe_combine(p, yp, rop, w, None, out))
        torch.cuda.synchronize()
        assert torch.equal(out, first)
    # with a shared output added
    ysh = torch.randn((wl.T, wl.H), device="cuda")
    B.check(B.moe_combine(p, yp, rop, w, ysh, out))
    torch.cuda.synchronize()
    np.testing.assert_allclose(P.f64(out), ref + P.f64(ysh), rtol=2 ** -7, atol=2e-2)


# ------------------------------------------------------------------ argument errors
def test_invalid_arguments_return_status_without_launch():
    wl = W.TINY
    p = B.params(wl)
    ws = _ws(wl)
    x = torch.zeros((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros((wl.T, wl.K), dtype=torch.int32, device="cuda")
    w = torch.zeros((wl.T, wl.K), dtype=torch.float32, device="cuda")
    w_r = torch.zeros((wl.E, wl.H), dtype=torch.bfloat16, device="cuda")
    assert B.moe_route(p, None, None, w_r, None, ids, w, ws, ws.numel()) == 1
    assert B.moe_route(p, x, None, w_r, None, ids, w, ws, 16) == 1                  # small ws
    assert B.moe_route(p, x.view(torch.uint8)[:, 2:], None, w_r, None, ids, w, ws, ws.numel()) == 1
    bad = B.params(wl.with_(H=200))
    assert B.moe_route(bad, x, None, w_r, None, ids, w, ws, ws.numel()) == 2
    bad = B.params(wl.with_(K=9))
    assert B.moe_route(bad, x, None, w_r, None, ids, w, ws, ws.numel()) == 1
    torch.cuda.synchronize()


# ------------------------------------------------------------------ GroupedTopK, bias
def _grouped_topk(wl, logits, bias=None):
    ids = torch.empty((wl.T, wl.K), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.K), dtype=torch.float32, device="cuda")
    B.check(B.moe_grouped_topk(B.params(wl), logits, bias, ids, w))
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy()


def test_grouped_topk_page_example():
    # routing primer §七: scores of 8 experts in 4 groups of 2, group score = max, keep 2;
    # fed as logits log(score) through the softmax router (softmax keeps their order)
    from tests.conftest import load_golden
    g = load_golden("grouped_topk_example.txt")
    z = torch.log(torch.tensor([g["scores"]], dtype=torch.float32, device="cuda"))
    for K, want in ((3, g["grouped_top3"]), (4, g["grouped_top4"])):
        wl = W.Workload("ex", T=1, H=128, I=128, E=8, K=K, n_group=g["n_group"],
                        topk_group=g["topk_group"], group_topn=1)
        ids, w = _grouped_topk(wl, z)
        assert ids[0].tolist() == want
        s = np.array(g["scores"])[want]
        np.testing.assert_allclose(w[0], s / s.sum(), rtol=1e-6)


def test_grouped_topk_kernelswift_shape():
    # routing primer §十: 83 tokens, 256 experts in 8 groups of 32, keep 4 groups, top-8,
    # softmax, renormalised
    wl = W.Workload("ks", T=83, H=128, I=128, E=256, K=8, n_group=8, topk_group=4, group_topn=1)
    z = torch.randn((wl.T, wl.E), generator=torch.Generator(device="cuda").manual_seed(7), device="cuda") * 2
    ids, w = _grouped_topk(wl, z)
    s = o.scores(P.f64(z), 0)
    n_mism, _ = P.check_routing(ids, w, s, None, wl)
    assert n_mism == 0


def test_aux_free_bias_update_matches_oracle():
    from tests.conftest import load_golden
    g = load_golden("aux_free_bias_example.txt")
    counts = torch.tensor(g["counts"], dtype=torch.int32, device="cuda")
    bias = torch.tensor(g["bias"], dtype=torch.float32, device="cuda")
    B.check(B.moe_aux_free_bias_update(counts, 4, g["gamma"], bias))
    torch.cuda.synchronize()
    np.testing.assert_allclose(bias.cpu().numpy(), g["updated"], rtol=1e-6)
    rng = np.random.default_rng(8)
    c = rng.integers(0, 50, size=256).astype(np.int32)
    b0 = rng.normal(size=256).astype(np.float32)
    counts = torch.as_tensor(c, device="cuda")
    bias = torch.as_tensor(b0, device="cuda")
    B.check(B.moe_aux_free_bias_update(counts, 256, 0.01, bias))
    torch.cuda.synchronize()
    np.testing.assert_allclose(bias.cpu().numpy(), o.aux_free_bias_update(b0, c, 0.01), rtol=1e-6, atol=1e-7)
