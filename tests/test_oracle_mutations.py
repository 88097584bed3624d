"""The oracle's pins catch plausible mistakes: each test here plants one mistake in a copy
of an oracle function (on the CPU, through monkeypatch), runs every pin of
test_oracle_pins.py, and requires at least one of them to fail."""
import inspect
import itertools

import numpy as np
import pytest

from oracle import moe_oracle as o
from tests import test_oracle_pins as pins


def _pin_cases():
    """(name, function, kwargs) for every pin, parametrized ones expanded."""
    out = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_") or fn.__module__ != pins.__name__:
            continue
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if not marks:
            out.append((name, fn, {}))
            continue
        grids = []
        for m in marks:
            argnames, argvalues = m.args[0], m.args[1]
            names = [a.strip() for a in argnames.split(",")] if isinstance(argnames, str) else list(argnames)
            grids.append([dict(zip(names, v if len(names) > 1 else (v,))) for v in argvalues])
        for combo in itertools.product(*grids):
            kw = {}
            for d in combo:
                kw.update(d)
            out.append((name, fn, kw))
    return out


PIN_CASES = _pin_cases()


def _failures():
    failed = []
    for name, fn, kw in PIN_CASES:
        params = inspect.signature(fn).parameters
        if any(p not in kw for p in params):
            continue  # needs a pytest fixture; not run here
        try:
            fn(**kw)
        except pytest.skip.Exception:
            continue
        except Exception:  # noqa: BLE001 - any failure of a pin counts
            failed.append(name)
    return failed


def test_pins_pass_on_the_unmodified_oracle():
    assert PIN_CASES, "no pins collected"
    assert _failures() == []


# ------------------------------------------------------------------ planted mistakes
def _route_no_renorm(s, K, bias=None, n_group=1, topk_group=1, group_topn=1, renormalize=True,
                     routed_scale=1.0):
    s = np.asarray(s, np.float64)
    c = s + (np.asarray(bias, np.float64)[None, :] if bias is not None else 0.0)
    ids = np.stack([o.select_experts(c[t], K, n_group, topk_group, group_topn) for t in range(s.shape[0])])
    w = np.stack([s[t, ids[t]] * routed_scale for t in range(s.shape[0])])   # renormalisation dropped
    return ids.astype(np.int32), w


def _route_scale_before_renorm(s, K, bias=None, n_group=1, topk_group=1, group_topn=1, renormalize=True,
                               routed_scale=1.0):
    s = np.asarray(s, np.float64)
    c = s + (np.asarray(bias, np.float64)[None, :] if bias is not None else 0.0)
    ids = np.stack([o.select_experts(c[t], K, n_group, topk_group, group_topn) for t in range(s.shape[0])])
    w = []
    for t in range(s.shape[0]):
        wt = s[t, ids[t]] * routed_scale
        w.append(wt / wt.sum() if renormalize else wt)                        # scale undone
    return ids.astype(np.int32), np.stack(w)


def _route_weights_from_biased(s, K, bias=None, n_group=1, topk_group=1, group_topn=1, renormalize=True,
                               routed_scale=1.0):
    s = np.asarray(s, np.float64)
    c = s + (np.asarray(bias, np.float64)[None, :] if bias is not None else 0.0)
    ids = np.stack([o.select_experts(c[t], K, n_group, topk_group, group_topn) for t in range(s.shape[0])])
    w = []
    for t in range(s.shape[0]):
        wt = c[t, ids[t]]                                                      # bias leaks into the weights
        w.append((wt / wt.sum() if renormalize else wt) * routed_scale)
    return ids.astype(np.int32), np.stack(w)


def _select_group_max(c_row, K, n_group=1, topk_group=1, group_topn=1):
    return _select_orig(c_row, K, n_group, topk_group, 1)                      # group_topn ignored


def _select_ties_high(c_row, K, n_group=1, topk_group=1, group_topn=1):
    c = np.asarray(c_row, np.float64)
    E = c.shape[0]
    order = np.argsort(-c[::-1], kind="stable")                               # ties to the higher index
    rev = (E - 1 - order)
    if n_group > 1:
        return _select_orig(c_row, K, n_group, topk_group, group_topn)[::-1].copy()
    return rev[:K]


def _scores_wrong_axis(z, score_fn):
    z = np.asarray(z, np.float64)
    if score_fn == 0:
        ez = np.exp(z - z.max(axis=0, keepdims=True))
        return ez / ez.sum(axis=0, keepdims=True)                             # softmax over tokens
    return 1.0 / (1.0 + np.exp(-z))


def _silu_sign(g):
    return g / (1.0 + np.exp(g))                                               # sigmoid of -g


def _router_no_transpose(x, w_r):
    w = np.asarray(w_r, np.float64)
    return np.asarray(x, np.float64) @ w.reshape(w.shape[1], w.shape[0])       # W_r read as [H, E]


def _permute_reversed(ids, E, block_m):
    counts, offsets, rop, por = _permute_orig(ids, E, block_m)
    flat = np.asarray(ids).reshape(-1)
    rop = rop.copy()
    por = por.copy()
    for e in range(E):
        rows = np.arange(offsets[e], offsets[e] + counts[e])
        ps = por[rows][::-1]                                                    # bucket order reversed
        por[rows] = ps
        rop[ps] = rows
    return counts, offsets, rop, por


def _combine_unweighted(y_perm, row_of_pair, w, y_shared=None):
    return _combine_orig(y_perm, row_of_pair, np.ones_like(np.asarray(w, np.float64)), y_shared)


def _pow2_floor(amax):
    amax = np.asarray(amax, np.float64)
    mant, expo = np.frexp(np.where(amax > 0, amax, o.FP8_MAX) / o.FP8_MAX)
    return np.where(amax > 0, np.ldexp(1.0, expo - 1), 1.0)                    # rounds the exponent down


def _e2m1_bias2(codes):
    return _e2m1_orig(codes) / 2.0                                             # exponent bias 2


def _fp4_nibbles_swapped(packed, scale_bytes):
    p = np.asarray(packed, dtype=np.uint8)
    return _dequant_fp4_orig(((p & 0xF) << 4) | (p >> 4), scale_bytes)


def _bf16_truncate(v):
    v = np.asarray(v, np.float64)
    m, e = np.frexp(v)
    return np.ldexp(np.trunc(np.ldexp(m, 8)), e - 8)                          # truncation, not RNE


def _masked_keeps_last(ids, E, cap):
    flat = np.asarray(ids, np.int64).reshape(-1)
    P = flat.shape[0]
    n = np.bincount(flat, minlength=E)
    rank = np.zeros(E, dtype=np.int64)
    rop = np.full(P, -1, dtype=np.int64)
    por = np.full(E * cap, -1, dtype=np.int64)
    for p in range(P):
        e = flat[p]
        r = rank[e] - max(n[e] - cap, 0)                                       # keeps the last cap pairs
        if r >= 0:
            rop[p] = e * cap + r
            por[e * cap + r] = p
        rank[e] += 1
    counts = np.minimum(n, cap)
    return (counts.astype(np.int32), (np.arange(E + 1) * cap).astype(np.int32), rop.astype(np.int32),
            por.astype(np.int32), int(np.maximum(n - cap, 0).sum()))


def _route_groups_on_unbiased(s, K, bias=None, n_group=1, topk_group=1, group_topn=1, renormalize=True,
                              routed_scale=1.0):
    s = np.asarray(s, np.float64)
    T, E = s.shape
    c = s + (np.asarray(bias, np.float64)[None, :] if bias is not None else 0.0)
    ids = np.empty((T, K), dtype=np.int32)
    w = np.empty((T, K))
    for t in range(T):
        cc = c[t].copy()
        if n_group > 1:
            gs = E // n_group
            g = np.sort(s[t].reshape(n_group, gs), axis=1)[:, ::-1][:, :group_topn].sum(axis=1)  # unbiased s
            allowed = np.zeros(E, dtype=bool)
            for j in np.argsort(-g, kind="stable")[:topk_group]:
                allowed[j * gs:(j + 1) * gs] = True
            cc = np.where(allowed, cc, -np.inf)
        ids[t] = np.argsort(-cc, kind="stable")[:K]
        wt = s[t, ids[t]]
        w[t] = (wt / wt.sum() if renormalize else wt) * routed_scale
    return ids, w


def _dequant_scales_transposed(codes, scales, rows_per_block):
    sc = np.asarray(scales, np.float64)
    return _dequant_blocks_orig(codes, sc.T if sc.shape[0] == sc.shape[1] else sc, rows_per_block)


def _requant_one_scale_per_row(h):
    h = np.asarray(h, np.float64)
    s = o.pow2_scale(np.abs(h).max(axis=1))[:, None]                          # whole row, not 1 x 128
    return o.quantize_e4m3(h / s) * s


def _route_ignores_bias(x, w_r, bias, wl):
    return _route_orig(x, w_r, None, wl)                                       # bias never reaches selection


_select_orig = o.select_experts
_route_orig = o.route
_dequant_blocks_orig = o.dequant_blocks
_permute_orig = o.permute
_combine_orig = o.combine
_e2m1_orig = o.decode_e2m1
_dequant_fp4_orig = o.dequant_fp4

MUTATIONS = {
    "renormalisation dropped": ("route_from_scores", _route_no_renorm),
    "routed scale applied before renormalising": ("route_from_scores", _route_scale_before_renorm),
    "weights taken from the biased scores": ("route_from_scores", _route_weights_from_biased),
    "group score = group max whatever group_topn": ("select_experts", _select_group_max),
    "ties go to the higher index": ("select_experts", _select_ties_high),
    "softmax over the wrong axis": ("scores", _scores_wrong_axis),
    "SiLU with the sign flipped": ("silu", _silu_sign),
    "W_r read as [H, E]": ("router_logits", _router_no_transpose),
    "buckets in reverse pair order": ("permute", _permute_reversed),
    "combine ignores the weights": ("combine", _combine_unweighted),
    "FP8 scale exponent rounded down": ("pow2_scale", _pow2_floor),
    "e2m1 exponent bias 2": ("decode_e2m1", _e2m1_bias2),
    "e2m1 nibbles swapped": ("dequant_fp4", _fp4_nibbles_swapped),
    "bf16 rounding truncates": ("round_bf16", _bf16_truncate),
    "masked layout keeps the last pairs": ("permute_masked", _masked_keeps_last),
    "groups ranked on the unbiased scores": ("route_from_scores", _route_groups_on_unbiased),
    "128x128 block scales transposed": ("dequant_blocks", _dequant_scales_transposed),
    "h re-quantised with one scale per row": ("quantize_rows_1x128", _requant_one_scale_per_row),
    "route drops the selection bias": ("route", _route_ignores_bias),
}


@pytest.mark.parametrize("what", list(MUTATIONS))
def test_planted_mistake_fails_a_pin(what, monkeypatch):
    name, mutant = MUTATIONS[what]
    monkeypatch.setattr(o, name, mutant)
    failed = _failures()
    assert failed, f"no pin catches: {what}"
