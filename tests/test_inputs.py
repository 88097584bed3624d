"""The seeded input generator: shapes, reproducibility, FP8 encoding and skew shape."""
import numpy as np
import torch

from mixture_experts_ffn_08_b200 import inputs, workloads as W
from oracle import moe_oracle as o


def test_shapes_and_reproducible():
    wl = W.DSV3_PREFILL.with_(T=10, H=256, I=128, E=16, n_group=4, topk_group=2, I_shared=128)
    a = inputs.make_inputs(wl, seed=3)
    b = inputs.make_inputs(wl, seed=3)
    c = inputs.make_inputs(wl, seed=4)
    assert a["x"].shape == (10, 256) and a["x"].dtype == torch.bfloat16
    assert a["w_gate"].shape == (16, 128, 256) and a["w_down"].shape == (16, 256, 128)
    assert a["ws_down"].shape == (256, 128) and a["bias"].shape == (16,)
    for k in a:
        assert torch.equal(a[k], b[k])
    assert not torch.equal(a["x"], c["x"])
    assert abs(a["w_gate"].float().std().item() - 0.02) < 0.002


def test_fp8_inputs_decode_close_to_gaussian_source():
    wl = W.SKEWED_FP8.with_(T=4, H=256, I=128, E=4, skewed=False)
    d = inputs.make_inputs(wl, seed=0)
    assert d["x_q"].dtype == torch.uint8 and d["x_scale"].shape == (4, 2)
    assert d["w_gate_s"].shape == (4, 1, 2) and d["w_down_s"].shape == (4, 2, 1)
    x = o.dequant_blocks(d["x_q"].numpy(), d["x_scale"].numpy(), 1)
    g = torch.Generator().manual_seed(1)        # same tag as the generator's "x"
    src = torch.randn((4, 256), generator=g).numpy()
    assert np.abs(x - src).max() <= np.abs(src).max() * 2.0 ** -4 + 1e-6
    s = d["x_scale"].numpy()
    assert (np.log2(s) == np.round(np.log2(s))).all()
    amax = np.abs(o.decode_e4m3(d["x_q"].numpy())).reshape(4, 2, 128).max(axis=2)
    assert (amax <= 448).all() and (amax > 224).all()


def test_skew_router_makes_one_expert_hot():
    wl = W.SKEWED_FP8.with_(T=512)
    d = inputs.make_inputs(wl, seed=0, weights=False)
    x = o.dequant_blocks(d["x_q"].numpy(), d["x_scale"].numpy(), 1)
    ids, _ = o.route_from_scores(o.scores(o.router_logits(x, d["w_r"].double().numpy()), 0), wl.K)
    counts = np.bincount(ids.ravel(), minlength=wl.E)
    mean = wl.T * wl.K / wl.E
    assert counts.max() >= 0.85 * wl.T and counts.max() / mean >= 13
    assert (counts == 0).sum() >= 1


def test_e2m1_weight_quantiser_is_nearest_with_minimal_scale():
    """The FP8 x FP4 workload's weights: each value is the nearest e2m1 code times the
    block's power-of-two scale (ties to the even code), and the scale is the smallest
    power of two that keeps the block's largest magnitude within 6."""
    torch.manual_seed(1)
    w = torch.randn(6, 128) * 0.02
    w[0, :4] = torch.tensor([0.0, 0.25, 0.75, -1.25]) * 2.0 ** -3   # exact ties on the grid
    packed, sb = inputs.quantize_rows_e2m1(w)
    assert packed.shape == (6, 64) and sb.shape == (6, 4)
    deq = o.dequant_fp4(packed.numpy(), sb.numpy())
    grid = o.decode_e2m1(np.arange(16))
    wv = w.double().numpy().reshape(6, 4, 32)
    scale = np.ldexp(1.0, sb.numpy().astype(np.int64) - 127)
    amax = np.abs(wv).max(axis=2)
    assert (amax / scale <= 6.0).all() and ((amax / (scale / 2) > 6.0) | (amax == 0)).all()
    for r in range(6):
        for b in range(4):
            for j in range(32):
                a = wv[r, b, j] / scale[r, b]
                d = np.abs(grid - a)
                best = np.flatnonzero(d == d.min())
                vals = {float(grid[c]) for c in best}
                got = deq[r, 32 * b + j] / scale[r, b]
                assert got in vals
                if len(vals) > 1:  # a tie: the even code wins
                    even = [c for c in best if c % 2 == 0]
                    assert got == grid[even[0]]
