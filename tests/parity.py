"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI, bring
its results to the host, and judge them against the fp64 oracle.

Acceptance rules:
  * topk weights: within 1e-4 relative of the oracle's weights for the same ids (the
    router logits are accumulated in fp32 over H terms on the tensor cores; observed
    logit errors reach a few 1e-5 at H = 7168, and a renormalised weight's relative
    error is at most twice the logit error).
  * topk ids: equal to the oracle's, except where candidate selection scores (or, for
    group-limited routing, group scores) lie within 1e-5 of each other; then the CUDA
    choice must be a valid top-K of the oracle's fp64 scores within that 1e-5.
  * counts / offsets / permutation: bit-exact against the oracle's bucketing of the ids
    the CUDA path chose.
  * outputs: against the oracle run on the CUDA path's routing, max |err| <= tol * RMS(ref)
    (tol = 2e-2 bf16, 6e-2 FP8) and mean|err| / mean|ref| <= 5e-3 (mean relative error).
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

from mixture_experts_ffn_08_b200 import binding as B
from mixture_experts_ffn_08_b200 import workloads as W
from oracle import moe_oracle as o

TIE_EPS = 1e-5
BF16_MAX_TOL = 2e-2
FP8_MAX_TOL = 6e-2
MEAN_REL_TOL = 5e-3


def f64(t) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def x_f64(d, wl, rows=None):
    """Exact values of x (dequantised for FP8) as float64, optionally a row subset."""
    if wl.dtype in (W.DTYPE_FP8, W.DTYPE_FP8_FP4):
        q, s = d["x_q"], d["x_scale"]
        if rows is not None:
            q, s = q[rows], s[rows]
        return o.dequant_blocks(q.cpu().numpy(), s.cpu().numpy(), 1)
    x = d["x"] if rows is None else d["x"][rows]
    return f64(x)


def expert_weights_fn(d, wl):
    """Callable e -> (W_gate[e], W_up[e], W_down[e]) in float64, copied on demand."""
    cache = {}

    def get(e):
        if e not in cache:
            if len(cache) > 8:
                cache.clear()
            if wl.dtype == W.DTYPE_FP8:
                cache[e] = tuple(
                    o.dequant_blocks(d[n + "_q"][e].cpu().numpy(), d[n + "_s"][e].cpu().numpy(), 128)
                    for n in ("w_gate", "w_up", "w_down"))
            elif wl.dtype == W.DTYPE_FP8_FP4:
                cache[e] = tuple(o.dequant_fp4(d[n + "_q"][e].cpu().numpy(), d[n + "_s"][e].cpu().numpy())
                                 for n in ("w_gate", "w_up", "w_down"))
            else:
                cache[e] = tuple(f64(d[n][e]) for n in ("w_gate", "w_up", "w_down"))
        return cache[e]
    return get


def shared_weights(d, wl):
    if not wl.I_shared:
        return None
    return tuple(f64(d[n]) for n in ("ws_gate", "ws_up", "ws_down"))


def prepare_fp4_atoms(d, wl):
    """Scale atoms of the three e2m1 weight tensors (moe_prepare_fp4_scales), stored in
    d as <name>_atoms."""
    for n, rows, K in (("w_gate", wl.E * wl.I, wl.H), ("w_up", wl.E * wl.I, wl.H), ("w_down", wl.E * wl.H, wl.I)):
        if n + "_atoms" not in d:
            atoms = torch.empty(rows * K // 32, dtype=torch.uint8, device="cuda")
            B.check(B.moe_prepare_fp4_scales(d[n + "_s"], rows, K, atoms), "moe_prepare_fp4_scales")
            d[n + "_atoms"] = atoms
    return d


def device_inputs_ptrs(d, wl):
    if wl.dtype == W.DTYPE_FP8_FP4:
        prepare_fp4_atoms(d, wl)
        return dict(
            x=d["x_q"], x_scale=d["x_scale"], w_r=d["w_r"], bias=d["bias"], w_gate=d["w_gate_q"],
            w_up=d["w_up_q"], w_down=d["w_down_q"], w_gate_scale=d["w_gate_atoms"], w_up_scale=d["w_up_atoms"],
            w_down_scale=d["w_down_atoms"], ws_gate=None, ws_up=None, ws_down=None)
    fp8 = wl.dtype == W.DTYPE_FP8
    return dict(
        x=d["x_q"] if fp8 else d["x"], x_scale=d.get("x_scale"), w_r=d["w_r"], bias=d["bias"],
        w_gate=d["w_gate_q"] if fp8 else d["w_gate"], w_up=d["w_up_q"] if fp8 else d["w_up"],
        w_down=d["w_down_q"] if fp8 else d["w_down"], w_gate_scale=d.get("w_gate_s"),
        w_up_scale=d.get("w_up_s"), w_down_scale=d.get("w_down_s"), ws_gate=d.get("ws_gate"),
        ws_up=d.get("ws_up"), ws_down=d.get("ws_down"))


def alloc_ws(p) -> torch.Tensor:
    n = B.moe_workspace_size_host(p)
    assert n > 0
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    B.check(B.moe_clear_device_status(ws))
    return ws


def run_layer(wl, d, ws=None):
    """One moe_layer_forward; returns out, ids, w, counts (device tensors) and ws."""
    p = B.params(wl)
    if ws is None:
        ws = alloc_ws(p)
    a = device_inputs_ptrs(d, wl)
    out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    ids = torch.empty((wl.T, wl.K), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.K), dtype=torch.float32, device="cuda")
    counts = torch.empty((wl.E,), dtype=torch.int32, device="cuda")
    B.check(B.moe_layer_forward(p, a["x"], a["x_scale"], a["w_r"], a["bias"], a["w_gate"], a["w_up"],
                                a["w_down"], a["w_gate_scale"], a["w_up_scale"], a["w_down_scale"],
                                a["ws_gate"], a["ws_up"], a["ws_down"], out, ids, w, counts, ws,
                                ws.numel()), "moe_layer_forward")
    torch.cuda.synchronize()
    return dict(out=out, ids=ids, w=w, counts=counts, ws=ws)


# ------------------------------------------------------------------ routing judgement
def _group_scores(c, wl):
    gs = wl.E // wl.n_group
    g = np.sort(c.reshape(wl.n_group, gs), axis=1)[:, ::-1]
    return g[:, :wl.group_topn].sum(axis=1)


def token_choice_ok(gpu_ids, c, wl, eps=TIE_EPS) -> bool:
    """Is gpu_ids a top-K (descending) of the fp64 selection scores c within eps?"""
    E, K = wl.E, wl.K
    if len(set(gpu_ids.tolist())) != K or gpu_ids.min() < 0 or gpu_ids.max() >= E:
        return False
    allowed = np.ones(E, dtype=bool)
    if wl.n_group > 1:
        gs = E // wl.n_group
        G = _group_scores(c, wl)
        thr = np.sort(G)[::-1][wl.topk_group - 1]
        chosen_groups = set((gpu_ids // gs).tolist())
        if any(G[j] < thr - eps for j in chosen_groups) or len(chosen_groups) > wl.topk_group:
            return False
        sure = {j for j in range(wl.n_group) if G[j] > thr + eps}
        keep = sure | chosen_groups
        allowed = np.array([(e // gs) in keep for e in range(E)])
    chosen = np.zeros(E, dtype=bool)
    chosen[gpu_ids] = True
    cv = c[gpu_ids]
    if np.any(np.diff(cv) > eps):          # must be descending within eps
        return False
    rest = c[allowed & ~chosen]
    return rest.size == 0 or cv.min() >= rest.max() - eps


def check_routing(gpu_ids, gpu_w, s, bias, wl, w_rtol=1e-4):
    """Judge CUDA ids/weights for all tokens; returns (n_exact_mismatch_tokens, oracle_w
    on the CUDA ids)."""
    s = np.asarray(s, np.float64)
    c = s + (np.asarray(bias, np.float64)[None, :] if bias is not None else 0.0)
    o_ids, _ = o.route_from_scores(s, wl.K, bias, wl.n_group, wl.topk_group, wl.group_topn,
                                   bool(wl.renormalize), wl.routed_scale)
    mism = np.where((o_ids != gpu_ids).any(axis=1))[0]
    for t in mism:
        assert token_choice_ok(gpu_ids[t], c[t], wl), (
            f"token {t}: cuda ids {gpu_ids[t].tolist()} vs oracle {o_ids[t].tolist()}; "
            f"c={c[t][gpu_ids[t]].tolist()} vs {c[t][o_ids[t]].tolist()}")
    # weights the oracle gives to the CUDA path's choice
    wt = np.take_along_axis(s, gpu_ids.astype(np.int64), axis=1)
    if wl.renormalize:
        wt = wt / wt.sum(axis=1, keepdims=True)
    wt = wt * wl.routed_scale
    np.testing.assert_allclose(gpu_w, wt, rtol=w_rtol, atol=1e-7)
    return len(mism), wt


def check_permutation(gpu_ids, E, counts, offsets, rop, por, block_m=B.BLOCK_M):
    o_counts, o_off, o_rop, o_por = o.permute(gpu_ids, E, block_m)
    np.testing.assert_array_equal(counts, o_counts)
    np.testing.assert_array_equal(offsets, o_off)
    np.testing.assert_array_equal(rop, o_rop)
    np.testing.assert_array_equal(por[:o_off[E]], o_por)


def error_stats(got, ref):
    """(max|err| / RMS(ref), mean|err| / mean|ref|)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    rms = np.sqrt(np.mean(ref * ref))
    return float(err.max() / rms), float(err.mean() / max(np.abs(ref).mean(), 1e-300))


def check_close(got, ref, max_tol, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    rms = np.sqrt(np.mean(ref * ref))
    mean_rel = err.mean() / max(np.abs(ref).mean(), 1e-300)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert err.max() <= max_tol * rms, f"{what}: max|err| {err.max():.4g} > {max_tol} * RMS {rms:.4g}"
    assert mean_rel <= MEAN_REL_TOL, f"{what}: mean rel err {mean_rel:.4g} > {MEAN_REL_TOL}"
    return err.max() / rms, mean_rel


def _report(record):
    """Append one JSON line to the file named by MOE_PARITY_REPORT (if set) and print it."""
    line = json.dumps(record)
    print("PARITY " + line)
    path = os.environ.get("MOE_PARITY_REPORT")
    if path:
        with open(path, "a", encoding="utf-8") as f:
            f.write(line + "\n")


def check_both_oracles(got, ref_reading, ref_exact, max_tol, what, exact_max=False):
    """Judge a bf16 layer output against two oracles.

    ref_reading stores h in bf16 between the two projections (the expert FFN computes in
    BF16, routing primer §8.4); ref_exact keeps h exact (fp64).  The bound is asserted
    against ref_reading.  Against ref_exact the mean relative error bound is always
    asserted and the max bound only where `exact_max` says it holds.  Both errors are
    reported, with the floor that rounding the exact output once to bf16 already costs
    (no bf16 output can be closer to ref_exact than that)."""
    got = np.asarray(got, np.float64)
    m_read, r_read = check_close(got, ref_reading, max_tol, what + " (h bf16)")
    m_ex, r_ex = error_stats(got, ref_exact)
    floor_max, floor_rel = error_stats(o.round_bf16(ref_exact), ref_exact)
    _report({"case": what, "n_outputs": int(got.size),
             "h_bf16": {"max_over_rms": m_read, "mean_rel": r_read},
             "h_exact": {"max_over_rms": m_ex, "mean_rel": r_ex},
             "bf16_output_rounding_floor": {"max_over_rms": floor_max, "mean_rel": floor_rel}})
    assert r_ex <= MEAN_REL_TOL, f"{what}: mean rel err vs exact-h oracle {r_ex:.4g} > {MEAN_REL_TOL}"
    if exact_max:
        assert m_ex <= max_tol, f"{what}: max|err|/RMS vs exact-h oracle {m_ex:.4g} > {max_tol}"
    return (m_read, r_read), (m_ex, r_ex)


def stratified_tokens(gpu_ids, E, rng, n_random=4, n_tail_experts=6, hot_rows=0):
    """Token sample for full-size parity that reaches the places uniform sampling misses.

    * n_random tokens drawn uniformly;
    * for n_tail_experts experts whose bucket ends in a partially filled 128-row M-tile,
      the token of the bucket's last pair (its row is in that partial tile);
    * hot_rows tokens of the most loaded expert, at ranks spread evenly over its bucket
      from the first row to the last, so they fall in many of its M-tiles.
    Buckets are stable in pair id p = t*K + k, so the rank of a pair inside its expert's
    bucket is its position among that expert's pairs in ascending p."""
    ids = np.asarray(gpu_ids)
    T, K = ids.shape
    flat = ids.ravel()
    counts = np.bincount(flat, minlength=E)
    toks = set(rng.choice(T, size=min(n_random, T), replace=False).tolist())
    partial = [e for e in range(E) if counts[e] % 128 != 0]
    for e in rng.permutation(partial)[:n_tail_experts]:
        pairs = np.flatnonzero(flat == e)
        toks.add(int(pairs[-1] // K))
    if hot_rows > 0:
        e = int(np.argmax(counts))
        pairs = np.flatnonzero(flat == e)
        ranks = np.unique(np.linspace(0, len(pairs) - 1, hot_rows).round().astype(np.int64))
        toks.update((pairs[ranks] // K).tolist())
    return np.array(sorted(toks), dtype=np.int64)
