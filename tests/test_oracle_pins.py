"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these tests needs a GPU.  Each pin checks the oracle against something other
than itself: the worked examples printed in "MoE 路由入门：从 Dense FFN 到 GroupedTopK"
(fixtures under tests/golden/), library routines that compute the same textbook
quantity (scipy softmax/expit, torch.topk, torch's SwiGLU pieces, torch's e4m3 cast),
closed-form invariants, and brute force over tiny inputs.
"""
import itertools

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

from oracle import moe_oracle as o
from tests.conftest import load_golden


# ------------------------------------------------------------------ worked examples
def test_top2_worked_example_raw_and_renormalised():
    g = load_golden("top2_worked_example.txt")
    s = np.array(g["scores"])
    ids, w = o.route_from_scores(s, g["K"], renormalize=False)
    assert ids.tolist() == g["topk_ids"]
    np.testing.assert_allclose(w, g["topk_weights"], rtol=0, atol=1e-15)
    ids2, w2 = o.route_from_scores(s, g["K"], renormalize=True)
    assert ids2.tolist() == g["topk_ids"]
    np.testing.assert_allclose(w2[0], g["renormalized_token0"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(w2.sum(axis=1), 1.0, rtol=0, atol=1e-15)


def test_top2_worked_example_through_softmax():
    # Each row of the printed scores sums to 1, so logits z = log(s) reproduce them
    # exactly through the softmax router.
    g = load_golden("top2_worked_example.txt")
    s = np.array(g["scores"])
    z = np.log(s)
    s2 = o.scores(z, 0)
    np.testing.assert_allclose(s2, s, rtol=1e-14, atol=0)
    ids, w = o.route_from_scores(s2, g["K"], renormalize=False)
    assert ids.tolist() == g["topk_ids"]
    np.testing.assert_allclose(w, g["topk_weights"], rtol=1e-14)


def test_bucket_example():
    g = load_golden("bucket_example.txt")
    ids = np.array([[e for (t, e) in g["pairs"][i * g["K"]:(i + 1) * g["K"]]] for i in range(g["T"])])
    counts, offs, row_of_pair, pair_of_row = o.permute(ids, g["E"], 1)
    assert counts.tolist() == g["counts"]
    assert ids.size == g["P"] == g["T"] * g["K"]
    for e in range(g["E"]):
        rows = range(offs[e], offs[e] + counts[e])
        assert [int(pair_of_row[r]) // g["K"] for r in rows] == g["buckets"][e]


@pytest.mark.parametrize("cap", [3, 4, 8])
def test_bucket_example_masked_layout(cap):
    """The page's dispatch example in the masked layout: expert e's tokens fill rows
    e*cap onwards in the printed order."""
    g = load_golden("bucket_example.txt")
    ids = np.array([[e for (t, e) in g["pairs"][i * g["K"]:(i + 1) * g["K"]]] for i in range(g["T"])])
    counts, offs, rop, por, dropped = o.permute_masked(ids, g["E"], cap)
    assert counts.tolist() == g["counts"] and dropped == 0
    assert offs.tolist() == [e * cap for e in range(g["E"] + 1)]
    for e in range(g["E"]):
        rows = range(e * cap, e * cap + counts[e])
        assert [int(por[r]) // g["K"] for r in rows] == g["buckets"][e]
        assert (por[e * cap + counts[e]:(e + 1) * cap] == -1).all()
    for p in range(ids.size):
        assert por[rop[p]] == p


def test_masked_layout_overflow_keeps_the_first_pairs():
    """Expert 2 of the page's dispatch example has 3 tokens; with cap 2 the third
    (token 2, the last pair of expert 2 in pair order) has no row."""
    g = load_golden("bucket_example.txt")
    ids = np.array([[e for (t, e) in g["pairs"][i * g["K"]:(i + 1) * g["K"]]] for i in range(g["T"])])
    counts, offs, rop, por, dropped = o.permute_masked(ids, g["E"], 2)
    assert counts.tolist() == [1, 1, 2, 1] and dropped == 1
    assert rop.tolist() == [2, 4, 0, 5, 6, -1]
    # the dropped pair adds nothing to its token: out[2] = w * y of expert 3 alone
    y = np.arange(8, dtype=np.float64)[:, None] * np.ones((1, 2))
    w = np.ones((3, 2))
    out = o.combine(y, rop, w)
    assert out[2].tolist() == [6.0, 6.0] and out[0].tolist() == [6.0, 6.0]


@pytest.mark.parametrize("cap", [37, 64])
def test_masked_ranks_match_contiguous_ranks(cap):
    """With room for every pair, the masked row of a pair is e*cap plus its rank, the
    same rank the contiguous layout gives (brute-force count of earlier pairs)."""
    rng = np.random.default_rng(cap)
    T, K, E = 37, 3, 9
    ids = np.stack([rng.choice(E, size=K, replace=False) for _ in range(T)])
    counts, offs, rop, por, dropped = o.permute_masked(ids, E, cap)
    assert dropped == 0 and counts.sum() == T * K
    flat = ids.ravel()
    for p in range(T * K):
        e = flat[p]
        assert rop[p] == e * cap + sum(1 for q in range(p) if flat[q] == e)


@pytest.mark.parametrize("group_topn", [1, 2])
def test_grouped_topk_example(group_topn):
    g = load_golden("grouped_topk_example.txt")
    c = np.array(g["scores"])
    kw = dict(n_group=g["n_group"], topk_group=g["topk_group"], group_topn=group_topn)
    assert o.select_experts(c, 3).tolist() == g["plain_top3"]
    assert o.select_experts(c, 3, **kw).tolist() == g["grouped_top3"]
    assert o.select_experts(c, 4).tolist() == g["plain_top4"]
    assert o.select_experts(c, 4, **kw).tolist() == g["grouped_top4"]


def test_grouped_topk_example_group_scores():
    # With group_topn = 1 the group score is the group maximum the page prints, and the
    # kept groups are the two best of those.
    g = load_golden("grouped_topk_example.txt")
    c = np.array(g["scores"]).reshape(g["n_group"], -1)
    np.testing.assert_allclose(c.max(axis=1), g["group_scores"])
    # the oracle masks exactly the groups outside kept_groups: ask for all survivors
    n_keep = g["topk_group"] * c.shape[1]
    sel = o.select_experts(c.ravel(), n_keep, n_group=g["n_group"], topk_group=g["topk_group"])
    assert sorted({int(e) // c.shape[1] for e in sel}) == sorted(g["kept_groups"])


# ------------------------------------------------------------------ library routines
def test_scores_match_scipy():
    rng = np.random.default_rng(1)
    z = rng.normal(size=(17, 33)) * 3
    np.testing.assert_allclose(o.scores(z, 0), scipy.special.softmax(z, axis=1), rtol=1e-13)
    np.testing.assert_allclose(o.scores(z, 1), scipy.special.expit(z), rtol=1e-13)


def test_router_logits_orientation():
    # z = x @ W_r^T with W_r stored [E, H]: logit (t, e) is the dot product of token t
    # with row e, checked element by element.
    rng = np.random.default_rng(2)
    x, w_r = rng.normal(size=(3, 5)), rng.normal(size=(4, 5))
    z = o.router_logits(x, w_r)
    assert z.shape == (3, 4)
    for t in range(3):
        for e in range(4):
            assert z[t, e] == pytest.approx(sum(x[t, h] * w_r[e, h] for h in range(5)), rel=1e-13)


@pytest.mark.parametrize("K", [1, 2, 8])
def test_plain_topk_matches_torch_topk(K):
    rng = np.random.default_rng(K)
    s = rng.random((50, 64))
    ids, w = o.route_from_scores(s, K, renormalize=False)
    tv, ti = torch.topk(torch.from_numpy(s), K, dim=1, sorted=True)
    assert (ids == ti.numpy()).all()
    np.testing.assert_array_equal(w, tv.numpy())


def test_sigmoid_plain_topk_is_topk_of_logits():
    # no bias, one group: top-k of sigmoid scores = top-k of the logits (monotone)
    rng = np.random.default_rng(3)
    z = rng.normal(size=(40, 32))
    ids, _ = o.route_from_scores(o.scores(z, 1), 4, renormalize=True)
    assert (ids == torch.topk(torch.from_numpy(z), 4, dim=1).indices.numpy()).all()


def test_ties_go_to_lower_index():
    s = np.array([[0.25, 0.25, 0.25, 0.25], [0.1, 0.3, 0.3, 0.3]])
    ids, _ = o.route_from_scores(s, 2)
    assert ids.tolist() == [[0, 1], [1, 2]]
    c = np.array([0.5, 0.5, 0.5, 0.5, 0.9, 0.1, 0.1, 0.1])
    # groups of 2: scores [0.5, 0.5, 0.9, 0.1] -> groups 2 then 0 (tie 0/1 -> 0)
    assert o.select_experts(c, 3, n_group=4, topk_group=2).tolist() == [4, 0, 1]


# ------------------------------------------------------------------ brute force
def _bruteforce_grouped(c, K, n_group, topk_group, group_topn):
    E = len(c)
    gs = E // n_group
    gscore = [max(sum(comb) for comb in itertools.combinations(c[j * gs:(j + 1) * gs], group_topn))
              for j in range(n_group)]
    best_groups = max(itertools.combinations(range(n_group), topk_group),
                      key=lambda gsub: sum(gscore[j] for j in gsub))
    allowed = [e for e in range(E) if e // gs in best_groups]
    best = max(itertools.combinations(allowed, K), key=lambda sub: sum(c[e] for e in sub))
    return set(best)


@pytest.mark.parametrize("seed", range(6))
def test_grouped_topk_bruteforce(seed):
    rng = np.random.default_rng(100 + seed)
    E, n_group, topk_group, K, topn = 16, 4, 2, 3, 2
    c = rng.random(E)
    sel = o.select_experts(c, K, n_group, topk_group, topn)
    assert set(sel.tolist()) == _bruteforce_grouped(c, K, n_group, topk_group, topn)
    assert all(c[sel[i]] >= c[sel[i + 1]] for i in range(K - 1))


def test_bias_only_chooses_and_scale_applies_after_renorm():
    s = np.array([[0.5, 0.3, 0.2]])
    bias = np.array([0.0, 0.0, 0.5])
    ids, w = o.route_from_scores(s, 1, bias=bias, renormalize=False)
    assert ids.tolist() == [[2]] and w[0, 0] == pytest.approx(0.2)
    ids, w = o.route_from_scores(s, 2, bias=bias, renormalize=True, routed_scale=2.5)
    assert ids.tolist() == [[2, 0]]
    np.testing.assert_allclose(w[0], [2.5 * 0.2 / 0.7, 2.5 * 0.5 / 0.7], rtol=1e-14)


def test_group_stage_ranks_groups_by_the_biased_scores():
    """The selection-only bias steers every selection step, the group stage included:
    groups are ranked on c = s + b.  Worked by hand on 4 experts in 2 groups, one group
    kept, group score = group maximum, K = 1.  s = [.5, .1, .45, .2], b = [0, 0, .1, 0]:
    biased group maxima are .5 and .55, so group {2, 3} stays and expert 2 (c = .55) wins.
    Ranking the groups on s instead (.5 and .45) would keep group {0, 1} and pick expert 0.
    The weight comes from the unbiased score and renormalises to the routed scale."""
    s = np.array([[0.5, 0.1, 0.45, 0.2]])
    b = np.array([0.0, 0.0, 0.1, 0.0])
    ids, w = o.route_from_scores(s, 1, b, n_group=2, topk_group=1, group_topn=1, routed_scale=2.5)
    assert ids.tolist() == [[2]] and w[0, 0] == pytest.approx(2.5)
    ids, _ = o.route_from_scores(s, 1, None, n_group=2, topk_group=1, group_topn=1)
    assert ids.tolist() == [[0]]  # without the bias the other group wins


def test_route_applies_the_selection_bias_end_to_end():
    """Logits through sigmoid, the bias steering the choice, the weight from the unbiased
    score.  x = [1, 0] and W_r rows [1, 0], [.9, 0], [0, 1] give logits [1, .9, 0] and
    scores expit(.) = [.731, .711, .5]; a bias of +.1 on expert 1 makes it the top-1
    (.811 > .731); without the bias expert 0 wins."""
    from types import SimpleNamespace
    wl = SimpleNamespace(K=1, score_fn=1, n_group=1, topk_group=1, group_topn=1, renormalize=False,
                         routed_scale=1.0)
    x = np.array([[1.0, 0.0]])
    w_r = np.array([[1.0, 0.0], [0.9, 0.0], [0.0, 1.0]])
    ids, w, s = o.route(x, w_r, np.array([0.0, 0.1, 0.0]), wl)
    assert ids.tolist() == [[1]] and w[0, 0] == pytest.approx(scipy.special.expit(0.9), rel=1e-15)
    ids, _, _ = o.route(x, w_r, None, wl)
    assert ids.tolist() == [[0]]


def test_weights_sum_to_routed_scale():
    rng = np.random.default_rng(4)
    s = scipy.special.expit(rng.normal(size=(30, 64)))
    bias = rng.normal(size=64) * 0.1
    _, w = o.route_from_scores(s, 8, bias, 8, 4, 2, True, 2.5)
    np.testing.assert_allclose(w.sum(axis=1), 2.5, rtol=1e-14)


def test_grouped_reduces_to_plain_when_one_group():
    rng = np.random.default_rng(5)
    s = rng.random((20, 32))
    a, _ = o.route_from_scores(s, 4, n_group=1)
    b, _ = o.route_from_scores(s, 4, n_group=4, topk_group=4, group_topn=2)
    assert (a == b).all()


# ------------------------------------------------------------------ permutation
@pytest.mark.parametrize("block_m", [1, 4, 128])
def test_permute_invariants_and_bruteforce(block_m):
    rng = np.random.default_rng(block_m)
    T, K, E = 37, 3, 9
    ids = np.stack([rng.choice(E, size=K, replace=False) for _ in range(T)])
    counts, offs, rop, por = o.permute(ids, E, block_m)
    assert counts.sum() == T * K
    assert (counts == np.bincount(ids.ravel(), minlength=E)).all()
    assert (offs % block_m == 0).all() and offs[0] == 0
    assert (np.diff(offs) >= counts).all() and (np.diff(offs) < counts + block_m).all()
    flat = ids.ravel()
    for p in range(T * K):
        e = flat[p]
        assert rop[p] == offs[e] + sum(1 for q in range(p) if flat[q] == e)
        assert por[rop[p]] == p
    assert (por == -1).sum() == offs[E] - T * K


# ------------------------------------------------------------------ FFN and combine
def _torch_swiglu(x, wg, wu, wd):
    x, wg, wu, wd = (torch.from_numpy(np.asarray(a, np.float64)) for a in (x, wg, wu, wd))
    return F.linear(F.silu(F.linear(x, wg)) * F.linear(x, wu), wd).numpy()


def test_single_expert_layer_is_dense_swiglu():
    # E = 1, K = 1, renormalised: every token goes to the one expert with weight 1, so
    # the layer is the dense SwiGLU FFN (computed here with torch's linear and silu).
    rng = np.random.default_rng(6)
    T, H, I = 11, 16, 24
    x = rng.normal(size=(T, H))
    wg, wu, wd = rng.normal(size=(I, H)) * .2, rng.normal(size=(I, H)) * .2, rng.normal(size=(H, I)) * .2
    ids = np.zeros((T, 1), dtype=np.int32)
    w = np.ones((T, 1))
    out = o.forward_given_routing(x, ids, w, lambda e: (wg, wu, wd), 1, block_m=4)
    np.testing.assert_allclose(out, _torch_swiglu(x, wg, wu, wd), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(o.swiglu_ffn(x, wg, wu, wd), _torch_swiglu(x, wg, wu, wd), rtol=1e-12)


def test_combine_of_identity_experts_returns_x():
    rng = np.random.default_rng(7)
    T, H, E, K = 13, 8, 5, 3
    x = rng.normal(size=(T, H))
    s = scipy.special.softmax(rng.normal(size=(T, E)), axis=1)
    ids, w = o.route_from_scores(s, K, renormalize=True)
    counts, offs, rop, por = o.permute(ids, E, 4)
    y_perm = np.zeros((offs[E], H))
    real = por >= 0
    y_perm[real] = x[por[real] // K]          # identity expert: y = x
    np.testing.assert_allclose(o.combine(y_perm, rop, w), x, rtol=1e-13, atol=1e-14)


def _loop_swiglu(xt, wg, wu, wd):
    I, H = wg.shape
    h = []
    for i in range(I):
        g = sum(wg[i, j] * xt[j] for j in range(H))
        u = sum(wu[i, j] * xt[j] for j in range(H))
        h.append(g / (1 + np.exp(-g)) * u)
    return np.array([sum(wd[j, i] * h[i] for i in range(I)) for j in range(H)])


@pytest.mark.parametrize("case", ["softmax_plain", "sigmoid_grouped_bias_shared"])
def test_layer_equals_dense_mixture_masked_to_topk(case):
    # Dense all-experts mixture (every expert run on every token, routing page §二),
    # masked to the chosen top-K with their renormalised weights, in plain Python
    # loops; must equal the oracle's sparse dispatch -> grouped FFN -> combine path.
    rng = np.random.default_rng(8)
    T, H, I, E, K = 6, 8, 6, 8, 2
    x = rng.normal(size=(T, H))
    w_r = rng.normal(size=(E, H)) * 0.5
    Wg, Wu = rng.normal(size=(E, I, H)) * .3, rng.normal(size=(E, I, H)) * .3
    Wd = rng.normal(size=(E, H, I)) * .3
    from types import SimpleNamespace as NS
    if case == "softmax_plain":
        wl = NS(E=E, K=K, score_fn=0, n_group=1, topk_group=1, group_topn=1, renormalize=True,
                routed_scale=1.0, dtype=0)
        bias, shared = None, None
    else:
        wl = NS(E=E, K=K, score_fn=1, n_group=4, topk_group=2, group_topn=2, renormalize=True,
                routed_scale=2.5, dtype=0)
        bias = rng.normal(size=E) * 0.1
        shared = (rng.normal(size=(4, H)) * .3, rng.normal(size=(4, H)) * .3, rng.normal(size=(H, 4)) * .3)
    out, ids, w, s = o.layer_forward(x, w_r, bias, lambda e: (Wg[e], Wu[e], Wd[e]), wl, shared,
                                     h_format=None)
    for t in range(T):
        dense = np.zeros(H)
        for e in range(E):
            p = 0.0
            if e in ids[t]:
                k = list(ids[t]).index(e)
                p = w[t, k]
            dense += p * _loop_swiglu(x[t], Wg[e], Wu[e], Wd[e])
        if shared is not None:
            dense += _loop_swiglu(x[t], *shared)
        np.testing.assert_allclose(out[t], dense, rtol=1e-10, atol=1e-12)


# ------------------------------------------------------------------ e4m3
def test_e4m3_decode_table_matches_torch_and_spot_values():
    codes = np.arange(256, dtype=np.uint8)
    mine = o.decode_e4m3(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert (np.isnan(mine) == nan).all() and nan.sum() == 2
    np.testing.assert_array_equal(mine[~nan], ref[~nan])
    assert mine[0x7E] == 448.0 and mine[0x01] == 2.0 ** -9 and mine[0x08] == 2.0 ** -6
    assert mine[0x38] == 1.0 and mine[0xB8] == -1.0 and mine[0x07] == 7 * 2.0 ** -9


def test_e4m3_quantize_is_nearest_even_by_search():
    grid_codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    grid = o.decode_e4m3(grid_codes)
    rng = np.random.default_rng(9)
    pos = np.sort(np.unique(np.abs(grid)))
    mids = (pos[1:] + pos[:-1]) / 2
    v = np.concatenate([rng.normal(size=2000) * 50, mids, -mids, [0.0, 448.0, 470, 1e6, -1e6, 2.0 ** -11]])
    q = o.quantize_e4m3(v)
    for vi, qi in zip(v, q):
        if abs(vi) >= 448:
            assert qi == np.copysign(448.0, vi)
            continue
        d = np.abs(grid - vi)
        cand = grid_codes[d == d.min()]
        cand_vals = o.decode_e4m3(cand)
        if len(set(cand_vals.tolist())) > 1:   # a true midpoint: pick the even code
            cand = cand[(cand & 1) == 0]
        assert qi == o.decode_e4m3(cand[:1])[0] or (qi == 0 and vi == 0)
    inr = np.abs(v) < 448
    tq = torch.from_numpy(v[inr]).to(torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(np.abs(q[inr]), np.abs(tq))


def test_block_dequant_of_constant_codes_is_the_scale_grid():
    """Codes that all decode to 1.0 dequantise to the block-scale grid itself: element
    (r, c) takes scales[r // 128, c // 128].  A non-symmetric 2 x 2 grid tells rows from
    columns."""
    codes = np.full((256, 256), 0x38, dtype=np.uint8)  # e4m3 1.0
    assert o.decode_e4m3(np.array([0x38]))[0] == 1.0
    scales = np.array([[1.0, 2.0], [4.0, 8.0]])
    got = o.dequant_blocks(codes, scales, 128)
    assert got[0, 0] == 1.0 and got[0, 255] == 2.0 and got[255, 0] == 4.0 and got[255, 255] == 8.0
    assert got[127, 127] == 1.0 and got[128, 127] == 4.0 and got[127, 128] == 2.0
    # one scale per row and 128 columns (rows_per_block = 1) for activations
    x_scales = np.array([[1.0, 0.5]] * 3 + [[2.0, 4.0]])
    got = o.dequant_blocks(np.full((4, 256), 0x38, dtype=np.uint8), x_scales, 1)
    assert got[0, 0] == 1.0 and got[0, 128] == 0.5 and got[3, 0] == 2.0 and got[3, 255] == 4.0


def test_activation_format_of_each_dtype():
    """h is stored in the activation format of the layer: bf16 for the bf16 layer, and
    e4m3 with 1 x 128 scales whenever the activations are e4m3 (the FP8 layer and the
    FP8 x FP4 layer, whose FP4 operand is the weights only)."""
    assert o.activation_format(0) == "bf16"
    assert o.activation_format(1) == "e4m3"
    assert o.activation_format(2) == "e4m3"


def test_pow2_scale_definition():
    rng = np.random.default_rng(10)
    amax = np.concatenate([rng.random(500) * 10.0 ** rng.integers(-6, 6, 500), [448.0, 896.0, 224.0, 0.0]])
    s = o.pow2_scale(amax)
    for a, si in zip(amax, s):
        if a == 0:
            assert si == 1.0
            continue
        assert np.log2(si) == np.round(np.log2(si))
        assert a / si <= 448.0 < a / (si / 2)


def test_rowwise_requant_error_bound():
    rng = np.random.default_rng(11)
    h = rng.normal(size=(5, 256)) * np.exp(rng.normal(size=(5, 1)))
    q = o.quantize_rows_1x128(h)
    b = h.reshape(5, 2, 128)
    s = o.pow2_scale(np.abs(b).max(axis=2))[:, :, None]
    err = np.abs(q.reshape(5, 2, 128) - b)
    # half a unit in the last place of e4m3 (3 mantissa bits), or of the subnormal step
    bound = np.maximum(np.abs(b) * 2.0 ** -4, s * 2.0 ** -10)
    assert (err <= bound + 1e-300).all()


def test_requant_scales_each_128_column_block_on_its_own():
    """Values that are e4m3 codes times a power of two come back exactly when each 1 x 128
    block gets its own scale: block 0 holds codes x 2^-20 (its maximum 448 x 2^-20 makes
    the scale 2^-20), block 1 codes x 1.  One scale for the whole row (1) would flush
    block 0 below e4m3's smallest subnormal, 2^-9."""
    codes = o.decode_e4m3(np.arange(0, 0x7F, dtype=np.uint8))      # every finite positive code and 0
    row0 = np.resize(codes, 128) * np.where(np.arange(128) % 2, -1.0, 1.0)
    row0[5] = 448.0
    h = np.concatenate([row0 * 2.0 ** -20, row0])[None, :]
    np.testing.assert_array_equal(o.quantize_rows_1x128(h), h)


# ------------------------------------------------------------------ bf16 activations
def test_round_bf16_matches_torch_on_fp32_values():
    rng = np.random.default_rng(12)
    v = (rng.normal(size=200000) * np.exp(rng.normal(size=200000) * 3)).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(o.round_bf16(v.astype(np.float64)), ref)


def test_round_bf16_nearest_even_by_grid():
    rng = np.random.default_rng(13)
    v = np.abs(rng.normal(size=3000)) * 10.0 ** rng.integers(-3, 4, 3000)
    for vi, qi in zip(v, o.round_bf16(v)):
        k = np.floor(np.log2(vi))
        ulp = 2.0 ** (k - 7)                      # 8 significant bits
        lo = np.floor(vi / ulp) * ulp
        hi = lo + ulp
        if vi - lo < hi - vi:
            want = lo
        elif vi - lo > hi - vi:
            want = hi
        else:
            want = lo if int(round(lo / ulp)) % 2 == 0 else hi
        assert qi == want, (vi, qi, want)
    # exact midpoints between neighbours go to the even neighbour
    assert o.round_bf16(1.0 + 2.0 ** -8) == 1.0
    assert o.round_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    assert o.round_bf16(-(1.0 + 2.0 ** -8)) == -1.0


def test_store_activation_formats():
    h = np.random.default_rng(14).normal(size=(3, 256))
    np.testing.assert_array_equal(o.store_activation(h, None), h)
    np.testing.assert_array_equal(o.store_activation(h, "bf16"), o.round_bf16(h))
    np.testing.assert_array_equal(o.store_activation(h, "e4m3"), o.quantize_rows_1x128(h))
    # SwiGLU with h stored in bf16 equals torch's pieces with an explicit bf16 round trip
    rng = np.random.default_rng(15)
    x, wg, wu, wd = rng.normal(size=(4, 16)), rng.normal(size=(8, 16)) * .3, rng.normal(size=(8, 16)) * .3, rng.normal(size=(16, 8)) * .3
    g = torch.from_numpy(x) @ torch.from_numpy(wg).T
    u = torch.from_numpy(x) @ torch.from_numpy(wu).T
    h = (F.silu(g) * u).float().to(torch.bfloat16).double()
    want = (h @ torch.from_numpy(wd).T).numpy()
    got = o.swiglu_ffn(x, wg, wu, wd, h_format="bf16")
    # torch rounds through fp32 first; both are within one bf16 rounding of each other
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ aux-free bias
def test_aux_free_bias_update_example():
    g = load_golden("aux_free_bias_example.txt")
    got = o.aux_free_bias_update(g["bias"], g["counts"], g["gamma"])
    np.testing.assert_allclose(got, g["updated"], rtol=0, atol=1e-15)


def test_aux_free_bias_update_balanced_is_fixed_point():
    b = np.array([0.3, -0.2, 0.1])
    np.testing.assert_array_equal(o.aux_free_bias_update(b, [5, 5, 5], 0.01), b)
    # only the sign of the imbalance matters, not its size
    a = o.aux_free_bias_update(np.zeros(3), [1, 2, 100], 0.5)
    np.testing.assert_array_equal(a, [0.5, 0.5, -0.5])


# ------------------------------------------------------------------ e2m1 (FP4) weights
def test_e2m1_decode_matches_ml_dtypes():
    """All 16 codes against an independent implementation of OCP FP4 (ml_dtypes)."""
    ml = pytest.importorskip("ml_dtypes")
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(ml.float4_e2m1fn).astype(np.float64)
    got = o.decode_e2m1(codes)
    assert np.array_equal(got, ref) and np.array_equal(np.signbit(got), np.signbit(ref))


def test_e2m1_spec_constants():
    """OCP MX v1.0 FP4 E2M1: largest normal 6.0, smallest normal 1.0, only subnormal
    0.5; positive codes increase with the code; the sign bit negates."""
    v = o.decode_e2m1(np.arange(16))
    assert v[7] == 6.0 and v[2] == 1.0 and v[1] == 0.5 and v[0] == 0.0
    assert (np.diff(v[:8]) > 0).all()
    assert np.array_equal(v[8:], -v[:8])


def test_dequant_fp4_nibble_order_and_block_scales():
    """Element 2j sits in the low nibble; each 32-element block has its own 2^(s-127)."""
    packed = np.zeros((1, 32), dtype=np.uint8)      # 64 elements, two scale blocks
    packed[0, 0] = 0x71                             # element 0 = code 1 (0.5), element 1 = code 7 (6)
    packed[0, 16] = 0x2A                            # element 32 = code 0xA (-1), element 33 = code 2 (1)
    scales = np.array([[127 + 3, 127 - 1]], dtype=np.uint8)
    w = o.dequant_fp4(packed, scales)
    assert w.shape == (1, 64)
    assert w[0, 0] == 0.5 * 8 and w[0, 1] == 6.0 * 8
    assert w[0, 32] == -0.5 and w[0, 33] == 0.5
    assert (w[0, 2:32] == 0).all() and (w[0, 34:] == 0).all()
