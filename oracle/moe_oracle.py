"""CPU oracle of the single-GPU MoE FFN layer forward, in float64.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or runs this
module: only the tests, the smoke check of the package entry file and the CPU
baseline leg of the benchmark do.  It shares no code with the CUDA library.

It is the plain definition of the layer, written so that each step can be checked
against the pages by eye:

  * router logits z = x @ W_r^T                    ("MoE" chapter index, §0 data-path
                                                    diagram; routing primer §三)
  * scores s = softmax(z_t) or sigmoid(z)          (routing primer §三)
  * selection score c = s + bias, bias used only   ("MoE" §0: "+bias, only for
    for choosing                                    selection"; §2.2 aux-free bias)
  * grouped top-k: group score, keep the best      (routing primer §六, §七, §九, §十)
    groups, mask the rest, then top-K
  * weights from the unbiased s, renormalised      (routing primer §四)
    over the K chosen, then times routed_scale
  * token-expert pairs bucketed by expert          (routing primer §5.1)
  * per-expert SwiGLU FFN                          (routing primer §一, §5.2)
      W_down (SiLU(W_gate x) * W_up x)
  * weighted combine y_t = sum_k w_tk y_tk         (routing primer §5.3)
    plus the always-active shared expert           ("MoE" §0 diagram, §2.1)

Readings where the pages are silent (each also listed in the design notes):
  - W_r is stored [E, H] (logits x @ W_r^T).
  - The group stage ranks groups by the biased selection score c; the group score is
    the sum of the `group_topn` largest c in the group (1 = the group maximum used in
    the routing primer's §七 example).
  - Order and ties: experts (and groups) are taken in descending score; an exact tie
    goes to the lower index.
  - Pairs p = t*K + k are bucketed stably: inside an expert, rows follow p.
  - Each expert's rows start at a multiple of `block_m`; pad rows carry no pair.
  - Masked layout: expert e owns rows [e*cap, (e+1)*cap); a pair ranked cap or later
    inside its expert gets no row and contributes nothing.
  - Renormalise first, then multiply by routed_scale; the shared expert is added with
    weight 1.
  - The SwiGLU output h is an activation and is stored in the workload's activation
    format before the down projection: bf16 (round to nearest even) for the bf16
    workloads, since the expert FFN computes in FP16/BF16 and only the router
    statistics are kept in FP32 (routing primer §8.4); e4m3 with one power-of-two
    scale per row and 128 columns for the FP8 workload, as the Mega MoE pipeline
    casts h in its "SwiGLU / FP8 Cast" stage (MoE optimisation blog, §5.1).  The
    pages fix no rounding of h for the bf16 case beyond that, so h_format=None (h
    kept exact) is offered beside it and the tests report the error against both.
  - FP8 workload: e4m3 (max 448, round to nearest even, saturating); one
    power-of-two scale per 1x128 activation block and per 128x128 weight block.
  - FP8 x FP4 workload: activations as in the FP8 workload; weights e2m1 (OCP MX
    FP4) with one UE8M0 (power-of-two) scale per row and 32 consecutive K elements.
  - No residual is added; the layer returns routed + shared only.

Parity status: routed_scale and group_topn = 2 are not fixed by any worked example on
the pages; they are pinned only by self-consistency (weights sum to routed_scale;
group_topn and routed_scale reduce to the printed examples when set to 1).
"""
from __future__ import annotations


import numpy as np

FP8_MAX = 448.0
QBLOCK = 128


# ----------------------------------------------------------------------------------
# e4m3 (OCP FP8, "fn" variant: no infinities, 0x7F/0xFF are NaN, max 448)
# ----------------------------------------------------------------------------------
def decode_e4m3(codes) -> np.ndarray:
    """Value of each e4m3 byte: sign bit 7, 4 exponent bits (bias 7), 3 mantissa
    bits; exponent field 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = (1.0 + m / 8.0) * np.power(2.0, e - 7.0)
    sub = (m / 8.0) * 2.0 ** -6
    v = sign * np.where(e == 0, sub, normal)
    return np.where((c & 0x7F) == 0x7F, np.nan, v)


def _e4m3_positive_grid():
    codes = np.arange(0x7F, dtype=np.uint8)        # 0x00 .. 0x7E: all finite, >= 0
    return codes, decode_e4m3(codes)


def quantize_e4m3(v) -> np.ndarray:
    """Nearest e4m3 value to each element (ties to the even code, i.e. the one whose
    mantissa LSB is 0), saturating at +-448.  Returned as float64 values."""
    v = np.asarray(v, dtype=np.float64)
    codes, grid = _e4m3_positive_grid()
    a = np.minimum(np.abs(v), FP8_MAX)
    hi = np.clip(np.searchsorted(grid, a, side="left"), 0, len(grid) - 1)
    lo = np.clip(hi - 1, 0, len(grid) - 1)
    d_lo = a - grid[lo]
    d_hi = grid[hi] - a
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ((codes[hi] & 1) == 0))
    q = np.where(take_hi, grid[hi], grid[lo])
    return np.copysign(q, v)


def pow2_scale(amax) -> np.ndarray:
    """2^ceil(log2(amax / 448)) taken exactly from the binary exponent; 1 where
    amax == 0."""
    amax = np.asarray(amax, dtype=np.float64)
    mant, expo = np.frexp(np.where(amax > 0, amax, FP8_MAX) / FP8_MAX)   # mant in [0.5, 1)
    e = np.where(mant == 0.5, expo - 1, expo)
    return np.where(amax > 0, np.ldexp(1.0, e), 1.0)


def dequant_blocks(codes, scales, rows_per_block: int) -> np.ndarray:
    """codes [R, C] e4m3 with scales [R/rows_per_block, C/128] -> float64 [R, C]."""
    v = decode_e4m3(codes)
    s = np.repeat(np.repeat(np.asarray(scales, np.float64), rows_per_block, axis=0), QBLOCK, axis=1)
    return v * s


def quantize_rows_1x128(h) -> np.ndarray:
    """Re-quantise an activation matrix [R, C] to e4m3 with one power-of-two scale per
    row and 128 columns; returns the dequantised float64 values."""
    h = np.asarray(h, np.float64)
    R, C = h.shape
    b = h.reshape(R, C // QBLOCK, QBLOCK)
    s = pow2_scale(np.abs(b).max(axis=2))
    return (quantize_e4m3(b / s[:, :, None]) * s[:, :, None]).reshape(R, C)


# ----------------------------------------------------------------------------------
# e2m1 (OCP MX FP4) weights with one UE8M0 scale per 32 consecutive K elements: the
# FP4 operand of the FP8 x FP4 GEMM ("DeepGEMM质变", §5.3; §一 1.3 for the UE8M0
# scale buffers of the FP4 path)
# ----------------------------------------------------------------------------------
FP4_BLOCK = 32


def decode_e2m1(codes) -> np.ndarray:
    """Value of each 4-bit code: sign bit 3, 2 exponent bits (bias 1), 1 mantissa bit;
    exponent field 0 is subnormal (m/2).  No infinities or NaN."""
    c = np.asarray(codes, dtype=np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = c & 0x1
    return sign * np.where(e == 0, m / 2.0, (1.0 + m / 2.0) * np.power(2.0, e - 1.0))


def dequant_fp4(packed, scale_bytes) -> np.ndarray:
    """packed [R, C/2] uint8 (element 2j in the low nibble, 2j+1 in the high one) with
    UE8M0 scale bytes [R, C/32] (value 2^(byte-127)) -> float64 [R, C]."""
    p = np.asarray(packed, dtype=np.uint8)
    R = p.shape[0]
    codes = np.empty((R, p.shape[1] * 2), dtype=np.uint8)
    codes[:, 0::2] = p & 0xF
    codes[:, 1::2] = p >> 4
    s = np.ldexp(1.0, np.asarray(scale_bytes, np.int64) - 127)
    return decode_e2m1(codes) * np.repeat(s, FP4_BLOCK, axis=1)


def round_bf16(v) -> np.ndarray:
    """Nearest bfloat16 value (8 significant bits, ties to even) of each element, as
    float64.  Values here stay far inside bf16's normal range."""
    v = np.asarray(v, np.float64)
    m, e = np.frexp(v)                         # v = m * 2^e, |m| in [0.5, 1)
    return np.ldexp(np.round(np.ldexp(m, 8)), e - 8)   # np.round: half to even


def store_activation(h, h_format):
    """h in the activation format of the layer: None (exact), "bf16" or "e4m3"."""
    if h_format is None:
        return np.asarray(h, np.float64)
    if h_format == "bf16":
        return round_bf16(h)
    if h_format == "e4m3":
        return quantize_rows_1x128(h)
    raise ValueError(h_format)


# ----------------------------------------------------------------------------------
# Router, scores, selection
# ----------------------------------------------------------------------------------
def router_logits(x, w_r) -> np.ndarray:
    """z[t, e] = sum_h x[t, h] * W_r[e, h]  (x @ W_r^T)."""
    return np.asarray(x, np.float64) @ np.asarray(w_r, np.float64).T


def scores(z, score_fn: int) -> np.ndarray:
    """score_fn 0: softmax over the experts of each token; 1: sigmoid per expert."""
    z = np.asarray(z, np.float64)
    if score_fn == 0:
        ez = np.exp(z - z.max(axis=1, keepdims=True))
        return ez / ez.sum(axis=1, keepdims=True)
    return 1.0 / (1.0 + np.exp(-z))


def _desc_order(v) -> np.ndarray:
    """Indices by descending value; equal values keep ascending index order."""
    return np.argsort(-np.asarray(v, np.float64), kind="stable")


def select_experts(c_row, K: int, n_group: int = 1, topk_group: int = 1, group_topn: int = 1):
    """Top-K experts of one token by selection score c_row [E], descending.

    With n_group > 1 the E experts form n_group consecutive groups; a group's score is
    the sum of its `group_topn` largest c; only the `topk_group` best groups stay
    candidates and the others are masked before the final top-K."""
    c = np.asarray(c_row, np.float64).copy()
    E = c.shape[0]
    if n_group > 1:
        gs = E // n_group
        groups = c.reshape(n_group, gs)
        gscore = np.array([np.sort(groups[j])[::-1][:group_topn].sum() for j in range(n_group)])
        keep = _desc_order(gscore)[:topk_group]
        allowed = np.zeros(E, dtype=bool)
        for j in keep:
            allowed[j * gs:(j + 1) * gs] = True
        c = np.where(allowed, c, -np.inf)
    return _desc_order(c)[:K]


def route_from_scores(s, K: int, bias=None, n_group: int = 1, topk_group: int = 1,
                      group_topn: int = 1, renormalize: bool = True, routed_scale: float = 1.0):
    """Routing decision from scores s [T, E]: ids [T, K] int32, weights [T, K] float64."""
    s = np.asarray(s, np.float64)
    T, E = s.shape
    c = s + (np.asarray(bias, np.float64)[None, :] if bias is not None else 0.0)
    ids = np.empty((T, K), dtype=np.int32)
    w = np.empty((T, K), dtype=np.float64)
    for t in range(T):
        sel = select_experts(c[t], K, n_group, topk_group, group_topn)
        ids[t] = sel
        wt = s[t, sel]
        if renormalize:
            wt = wt / wt.sum()
        w[t] = wt * routed_scale
    return ids, w


def route(x, w_r, bias, wl):
    """Full routing of workload `wl` (any object with K, score_fn, n_group, topk_group,
    group_topn, renormalize, routed_scale).  Returns ids, weights, scores."""
    s = scores(router_logits(x, w_r), wl.score_fn)
    ids, w = route_from_scores(s, wl.K, bias, wl.n_group, wl.topk_group, wl.group_topn,
                               bool(wl.renormalize), wl.routed_scale)
    return ids, w, s


def aux_free_bias_update(bias, counts, gamma: float) -> np.ndarray:
    """One step of the auxiliary-loss-free balancing bias ("MoE" chapter index §2.2):
    b_e <- b_e + gamma * sign(mean_load - load_e), with mean_load the average of the
    per-expert loads (pair counts); an expert exactly at the mean is left unchanged."""
    load = np.asarray(counts, np.float64)
    return np.asarray(bias, np.float64) + gamma * np.sign(load.mean() - load)


# ----------------------------------------------------------------------------------
# Dispatch: pairs bucketed by expert
# ----------------------------------------------------------------------------------
def permute(ids, E: int, block_m: int):
    """Bucket the P = T*K pairs p = t*K + k by expert, stably in p.

    Returns counts [E], offsets_padded [E+1] (expert e's rows start at
    offsets_padded[e], a multiple of block_m), row_of_pair [P] and pair_of_row
    [offsets_padded[E]] (-1 on pad rows)."""
    flat = np.asarray(ids, np.int64).reshape(-1)
    P = flat.shape[0]
    counts = np.zeros(E, dtype=np.int64)
    for e in flat:
        counts[e] += 1
    padded = ((counts + block_m - 1) // block_m) * block_m
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(padded)
    row_of_pair = np.empty(P, dtype=np.int64)
    pair_of_row = np.full(int(offsets[E]), -1, dtype=np.int64)
    fill = offsets[:E].copy()
    for p in range(P):
        e = flat[p]
        row_of_pair[p] = fill[e]
        pair_of_row[fill[e]] = p
        fill[e] += 1
    return (counts.astype(np.int32), offsets.astype(np.int32),
            row_of_pair.astype(np.int32), pair_of_row.astype(np.int32))


def permute_masked(ids, E: int, cap: int):
    """The masked grouped layout ("MoE" chapter index §1, the grouped-GEMM entry: the
    second of its two layouts): expert e owns the fixed row range [e*cap, (e+1)*cap)
    and its pairs fill the first rows of that range, stably in p.

    The page names the layout only.  Reading used here: a pair whose rank inside its
    expert is cap or more has no row (row_of_pair = -1) and is left out of the layer
    output; counts [E] is the number of rows in use, min(n_e, cap).  With cap >= T no
    pair is ever left out, since a token chooses K distinct experts.

    Returns counts [E], offsets [E+1] = e*cap, row_of_pair [P], pair_of_row [E*cap]
    (-1 on unused rows) and the number of pairs left out."""
    flat = np.asarray(ids, np.int64).reshape(-1)
    P = flat.shape[0]
    rank = np.zeros(E, dtype=np.int64)
    row_of_pair = np.full(P, -1, dtype=np.int64)
    pair_of_row = np.full(E * cap, -1, dtype=np.int64)
    dropped = 0
    for p in range(P):
        e = flat[p]
        if rank[e] < cap:
            row = e * cap + rank[e]
            row_of_pair[p] = row
            pair_of_row[row] = p
        else:
            dropped += 1
        rank[e] += 1
    counts = np.minimum(rank, cap)
    offsets = np.arange(E + 1, dtype=np.int64) * cap
    return (counts.astype(np.int32), offsets.astype(np.int32), row_of_pair.astype(np.int32),
            pair_of_row.astype(np.int32), dropped)


# ----------------------------------------------------------------------------------
# Expert FFN and combine
# ----------------------------------------------------------------------------------
def silu(g):
    return g / (1.0 + np.exp(-g))


def swiglu_ffn(xr, wg, wu, wd, h_format=None):
    """W_down (SiLU(W_gate x) * W_up x) for each row of xr [n, H]; weights [out, in].
    h_format: format h is stored in between the two projections (see store_activation)."""
    xr = np.asarray(xr, np.float64)
    g = xr @ np.asarray(wg, np.float64).T
    u = xr @ np.asarray(wu, np.float64).T
    h = store_activation(silu(g) * u, h_format)
    return h @ np.asarray(wd, np.float64).T


def expert_outputs(x, ids, expert_weights, E: int, block_m: int, h_format=None):
    """y_perm [P_pad, H]: the output of every pair's expert on its token, laid out in
    the bucketed row order of `permute` (pad rows are zero).  `expert_weights(e)`
    returns (W_gate[e], W_up[e], W_down[e]) as arrays [I,H], [I,H], [H,I]."""
    x = np.asarray(x, np.float64)
    K = ids.shape[1]
    counts, offsets, row_of_pair, pair_of_row = permute(ids, E, block_m)
    y = np.zeros((int(offsets[E]), x.shape[1]), dtype=np.float64)
    for e in range(E):
        n = int(counts[e])
        if n == 0:
            continue
        rows = np.arange(offsets[e], offsets[e] + n)
        toks = pair_of_row[rows] // K
        wg, wu, wd = expert_weights(e)
        y[rows] = swiglu_ffn(x[toks], wg, wu, wd, h_format)
    return y, row_of_pair


def combine(y_perm, row_of_pair, w, y_shared=None) -> np.ndarray:
    """out[t] = sum_k w[t, k] * y_perm[row_of_pair[t*K + k]]  (+ y_shared[t]).
    A pair without a row (row_of_pair = -1, left out by the masked layout) adds 0."""
    w = np.asarray(w, np.float64)
    T, K = w.shape
    y_perm = np.asarray(y_perm, np.float64)
    out = np.zeros((T, y_perm.shape[1]), dtype=np.float64)
    for t in range(T):
        for k in range(K):
            r = row_of_pair[t * K + k]
            if r >= 0:
                out[t] += w[t, k] * y_perm[r]
    if y_shared is not None:
        out += np.asarray(y_shared, np.float64)
    return out


def forward_given_routing(x, ids, w, expert_weights, E: int, shared=None,
                          h_format=None, block_m: int = 1):
    """Layer output [T, H] for a given routing decision (ids, w).  `shared` is
    (W_gate, W_up, W_down) of the shared expert or None."""
    y_perm, row_of_pair = expert_outputs(x, ids, expert_weights, E, block_m, h_format)
    y_sh = swiglu_ffn(x, *shared, h_format=h_format) if shared is not None else None
    return combine(y_perm, row_of_pair, w, y_sh)


def activation_format(dtype: int):
    """Storage format of h for a workload dtype: 0 = bf16; 1 (FP8) and 2 (FP8 x FP4, whose
    FP4 operand is the weights) have e4m3 activations, so h is e4m3 with 1x128 scales."""
    return "e4m3" if dtype in (1, 2) else "bf16"


def layer_forward(x, w_r, bias, expert_weights, wl, shared=None, h_format="auto"):
    """Route, then run the chosen experts and combine.  Returns (out, ids, w, s).
    h_format "auto" stores h in the workload's activation format."""
    ids, w, s = route(x, w_r, bias, wl)
    if h_format == "auto":
        h_format = activation_format(wl.dtype)
    out = forward_given_routing(x, ids, w, expert_weights, wl.E, shared, h_format=h_format)
    return out, ids, w, s
