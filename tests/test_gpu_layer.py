"""Whole-layer parity: moe_layer_forward through the C ABI against the fp64 oracle.

Small workloads keep the shapes' features (routing rules, several M/N/K tiles, ragged
buckets) at sizes the oracle finishes in seconds and are compared on every element.
The full workloads run in the configuration the benchmark times and are compared on the
whole routing decision and permutation, plus output rows: every token of the decode
workload, and for the prefill workloads a stratified sample that includes tokens in
several experts' last, partially filled M-tiles and rows spread over the most loaded
expert's bucket.

Every output is judged against two oracles: h stored in bf16 between the projections
(the bf16 expert FFN, routing primer §8.4), where both bounds are asserted, and h kept
exact, where the mean relative bound is asserted and the max bound wherever it holds
(every case but those in EXACT_MAX_EXCEEDS); both errors are printed and, with
MOE_PARITY_REPORT set, appended to that file.
"""
import numpy as np
import pytest
import torch

from mixture_experts_ffn_08_b200 import binding as B
from mixture_experts_ffn_08_b200 import inputs, workloads as W
from oracle import moe_oracle as o
from tests import parity as P

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": W.TINY,
    "mixtral_small": W.MIXTRAL_PREFILL.with_(name="mixtral_small", T=1000, H=512, I=384),
    "dsv3_small": W.DSV3_PREFILL.with_(name="dsv3_small", T=200, H=512, I=256, E=32, I_shared=256),
    "dsv3_decode_small": W.DSV3_DECODE.with_(name="dsv3_decode_small", T=16, H=512, I=256, E=32,
                                             I_shared=256),
    # H not a multiple of 256: the shared expert's down projection does not take in the
    # combine, which then runs as its own kernel
    "dsv3_small_h384": W.DSV3_PREFILL.with_(name="dsv3_small_h384", T=200, H=384, I=256, E=32, I_shared=256),
    "one_token": W.MIXTRAL_PREFILL.with_(name="one_token", T=1, H=256, I=128, E=4, K=2),
    "dense_like": W.TINY.with_(name="dense_like", T=300, E=1, K=1),
    # T*K >= 256*E: the two-M-tile gate/up kernel (pairs of M-tiles plus one-tile tails)
    "mixtral_small_dual": W.MIXTRAL_PREFILL.with_(name="mixtral_small_dual", T=1200, H=512, I=384),
    "dsv3_small_dual": W.DSV3_PREFILL.with_(name="dsv3_small_dual", T=1100, H=512, I=256, E=32, I_shared=256),
    "mixtral_small_dual_masked": W.MIXTRAL_PREFILL.with_(name="mixtral_small_dual_masked", T=1200, H=512, I=384,
                                                         masked_cap=640),
    # more than 16384 pairs: the shared expert runs on the caller's stream through the
    # two-tile kernels as one dense group with an fp16 output, beside fp32 routed outputs
    # (T*K < 256*E) or fp16 ones (T*K >= 256*E)
    "dsv3_small_shared_dense": W.DSV3_PREFILL.with_(name="dsv3_small_shared_dense", T=2100, H=512, I=256,
                                                    E=128, I_shared=256),
    "dsv3_small_shared_dense_y16": W.DSV3_PREFILL.with_(name="dsv3_small_shared_dense_y16", T=2100, H=512,
                                                        I=256, E=64, I_shared=256),
    # buckets aligned to 256 rows: the two-SM (cta_group::2) GEMMs
    "mixtral_small_pair": W.MIXTRAL_PREFILL.with_(name="mixtral_small_pair", T=1000, H=512, I=384, block_m=256),
    "dsv3_small_pair": W.DSV3_PREFILL.with_(name="dsv3_small_pair", T=300, H=512, I=256, E=32, I_shared=256,
                                            block_m=256),
    # down projection fused with the combine (fp32 atomic accumulation)
    "mixtral_small_fused": W.MIXTRAL_PREFILL.with_(name="mixtral_small_fused", T=1000, H=512, I=384,
                                                   fused_combine=True),
    "dsv3_small_fused": W.DSV3_PREFILL.with_(name="dsv3_small_fused", T=200, H=384, I=256, E=32, I_shared=256,
                                             fused_combine=True),
}


# Cases whose max|err| against the exact-h oracle is above 2e-2 * RMS: the Mixtral-shaped
# small layer (T=1000, H=512, I=384) in its three forms, measured at 0.0208 (0.0159 against
# the bf16-h oracle), of which 0.0159 is the floor that rounding the exact output once to
# bf16 already costs on these 512,000 outputs.  Every other case
# asserts the max bound against the exact-h oracle as well.
EXACT_MAX_EXCEEDS = {"mixtral_small", "mixtral_small_pair", "mixtral_small_fused"}


def _both(x, ids, w, d, wl):
    """Oracle outputs with h in bf16 and with h exact, on the given routing."""
    sh = P.shared_weights(d, wl)
    ew = P.expert_weights_fn(d, wl)
    return tuple(o.forward_given_routing(x, ids, w, ew, wl.E, sh, h_format=f) for f in ("bf16", None))


def _oracle_full(d, wl, gpu_ids):
    x = P.x_f64(d, wl)
    s = o.scores(o.router_logits(x, P.f64(d["w_r"])), wl.score_fn)
    bias = P.f64(d["bias"]) if d["bias"] is not None else None
    return x, s, bias


@pytest.mark.parametrize("name", list(SMALL))
def test_layer_small_all_elements(name):
    wl = SMALL[name]
    d = inputs.make_inputs(wl, seed=0, device="cuda")
    r = P.run_layer(wl, d)
    assert B.moe_get_device_status(r["ws"]) == 0
    gpu_ids = r["ids"].cpu().numpy()
    x, s, bias = _oracle_full(d, wl, gpu_ids)
    _, w_or = P.check_routing(gpu_ids, r["w"].cpu().numpy(), s, bias, wl)
    np.testing.assert_array_equal(r["counts"].cpu().numpy(), np.bincount(gpu_ids.ravel(), minlength=wl.E))
    ref, ref_exact = _both(x, gpu_ids, w_or, d, wl)
    P.check_both_oracles(P.f64(r["out"]), ref, ref_exact, P.BF16_MAX_TOL, name,
                         exact_max=name not in EXACT_MAX_EXCEEDS)


def test_layer_is_deterministic():
    wl = SMALL["dsv3_small"]
    d = inputs.make_inputs(wl, seed=1, device="cuda")
    first = P.run_layer(wl, d)
    for _ in range(5):
        again = P.run_layer(wl, d, ws=first["ws"])
        assert torch.equal(again["out"], first["out"])
        assert torch.equal(again["ids"], first["ids"])


FULL = ["mixtral_prefill", "dsv3_prefill", "dsv3_decode", "dsv3_prefill_fused"]


@pytest.mark.parametrize("name", FULL)
def test_layer_full_size_sampled(name):
    wl = W.ALL[name] if name in W.ALL else W.ALL[name[:-len("_fused")]].with_(fused_combine=True)
    d = inputs.make_inputs(wl, seed=0, device="cuda")
    r = P.run_layer(wl, d)
    assert B.moe_get_device_status(r["ws"]) == 0
    gpu_ids = r["ids"].cpu().numpy()
    x, s, bias = _oracle_full(d, wl, gpu_ids)
    n_mism, w_or = P.check_routing(gpu_ids, r["w"].cpu().numpy(), s, bias, wl)
    assert n_mism <= max(2, wl.T // 1000), f"{n_mism} near-tie tokens"
    counts = r["counts"].cpu().numpy()
    assert counts.sum() == wl.T * wl.K
    np.testing.assert_array_equal(counts, np.bincount(gpu_ids.ravel(), minlength=wl.E))
    rng = np.random.default_rng(0)
    if wl.T <= 128:
        toks = np.arange(wl.T)                     # decode: every token
    elif wl.E <= 8:
        toks = P.stratified_tokens(gpu_ids, wl.E, rng, n_random=8, n_tail_experts=wl.E, hot_rows=8)
    else:
        toks = P.stratified_tokens(gpu_ids, wl.E, rng, n_random=4, n_tail_experts=8, hot_rows=4)
    ref, ref_exact = _both(x[toks], gpu_ids[toks], w_or[toks], d, wl)
    got = P.f64(r["out"][torch.as_tensor(toks, device="cuda")])
    P.check_both_oracles(got, ref, ref_exact, P.BF16_MAX_TOL, f"{name} ({len(toks)} tokens)",
                         exact_max=name not in EXACT_MAX_EXCEEDS)
    del d, r
    torch.cuda.empty_cache()


def test_host_entry_point_matches_device_entry_point():
    wl = SMALL["dsv3_small"]
    d = inputs.make_inputs(wl, seed=2, device="cuda")
    r = P.run_layer(wl, d)
    p = B.params(wl)
    a = P.device_inputs_ptrs(d, wl)
    x_host = d["x"].cpu().pin_memory()
    out_host = torch.empty((wl.T, wl.H), dtype=torch.bfloat16).pin_memory()
    ws = r["ws"]
    B.check(B.moe_layer_forward_host(p, x_host, None, a["w_r"], a["bias"], a["w_gate"], a["w_up"],
                                     a["w_down"], None, None, None, a["ws_gate"], a["ws_up"],
                                     a["ws_down"], out_host, ws, ws.numel()))
    torch.cuda.synchronize()
    assert torch.equal(out_host, r["out"].cpu())


def test_expert_output_beyond_fp16_range_is_reported():
    """At prefill sizes the layer keeps routed expert outputs in fp16: one beyond 65504
    must set MOE_DEV_RANGE (and nothing else) in the status word."""
    wl = SMALL["mixtral_small_dual"]
    d = inputs.make_inputs(wl, seed=0, device="cuda")
    orig = d["w_down"]
    # y has an RMS of ~0.04 here; scaled by 1e6 its largest values pass 65504
    d["w_down"] = (orig.float() * 1.0e6).to(torch.bfloat16)
    r = P.run_layer(wl, d)
    assert B.moe_get_device_status(r["ws"]) == B.MOE_DEV_RANGE
    d["w_down"] = orig
    r = P.run_layer(wl, d)
    assert B.moe_get_device_status(r["ws"]) == 0
