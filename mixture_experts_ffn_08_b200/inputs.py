"""Seeded synthetic inputs for the MoE layer workloads.

This module only draws numbers: Gaussian activations and weights of the sizes a
workload names, the selection bias, the Zipf-shaped router of the skew stress case
and, for the FP8 workloads, the e4m3 (and e2m1 weight) codes plus power-of-two block
scales that the layer then consumes as given inputs. It computes no part of the layer (no routing,
no permutation, no expert FFN, no combine), so both the CUDA path and the CPU
oracle can be fed from it without sharing any of the method's arithmetic.

Every tensor has its own torch.Generator seeded from (seed, tensor tag); large
tensors are drawn expert by expert so peak temporary memory stays at one slice.
Draws on a CUDA device and on the CPU give different (but each reproducible)
numbers; tests that compare the two sides copy the device tensors to the host.
"""
from __future__ import annotations

import math

import torch

from .workloads import Workload, DTYPE_FP8, DTYPE_FP8_FP4

_TAGS = {"x": 1, "w_r": 2, "bias": 3, "w_gate": 4, "w_up": 5, "w_down": 6,
         "ws_gate": 7, "ws_up": 8, "ws_down": 9, "skew_m": 10, "skew_rank": 11}

WEIGHT_STD = 0.02
BIAS_STD = 0.1
FP8_MAX = 448.0
QBLOCK = 128

# Skew stress router: row e of W_r is 0.02*n_e + beta_e * m / |m|^2 with
# beta_e = -ZIPF_S * SKEW_TAU * ln(rank_e), rank_e a seeded permutation of 1..E,
# and every token carries the common direction m (|m| = sqrt(H)/2).  The logit of
# expert e is then about beta_e plus N(0, 1.4^2) noise, so popularity falls off as
# a Zipf(1.2) power of the rank.  SKEW_TAU was chosen so that the hottest expert is
# picked by about 94% of the tokens (about 15x the mean load), close to the most one
# expert can receive when every token picks K distinct experts (T pairs = 16x the
# mean); about a tenth of the experts then receive no token at all.
ZIPF_S = 1.2
SKEW_TAU = 1.0


def _gen(device, seed: int, tag: str) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + _TAGS[tag])
    return g


def _normal(shape, std, g, device, out_dtype=torch.bfloat16):
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(out_dtype)


def _stacked_normal(n, shape, std, g, device):
    out = torch.empty((n, *shape), dtype=torch.bfloat16, device=device)
    for e in range(n):
        out[e] = _normal(shape, std, g, device)
    return out


def _pow2_scale(amax: torch.Tensor) -> torch.Tensor:
    """Smallest power of two s with amax / s <= 448 (1 where amax == 0), exactly."""
    v = amax / FP8_MAX
    mant, expo = torch.frexp(v)            # v = mant * 2**expo, mant in [0.5, 1)
    e = torch.where(mant == 0.5, expo - 1, expo)
    s = torch.ldexp(torch.ones_like(v), e)
    return torch.where(amax > 0, s, torch.ones_like(v))


def quantize_blocks_e4m3(v: torch.Tensor, rows_per_block: int):
    """Encode a [R, C] fp32 matrix as e4m3 codes with one power-of-two scale per
    (rows_per_block x 128) block.  Returns (codes uint8 [R, C], scales fp32
    [R/rows_per_block, C/128]).  The cast itself is torch's float8_e4m3fn
    conversion; this is how the FP8 workload's given inputs are produced."""
    R, C = v.shape
    assert R % rows_per_block == 0 and C % QBLOCK == 0
    blocks = v.reshape(R // rows_per_block, rows_per_block, C // QBLOCK, QBLOCK)
    amax = blocks.abs().amax(dim=(1, 3))
    s = _pow2_scale(amax)
    q = (blocks / s[:, None, :, None]).reshape(R, C).to(torch.float8_e4m3fn)
    return q.view(torch.uint8), s.contiguous()


FP4_MAX = 6.0
FP4_BLOCK = 32
# The eight non-negative e2m1 values (OCP MX FP4), in code order 0..7.
_E2M1_POS = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def quantize_rows_e2m1(v: torch.Tensor):
    """Encode a [R, C] fp32 matrix as e2m1 codes with one power-of-two scale per row and
    32 columns (the smallest with amax / scale <= 6), nearest value with ties to the
    even code.  Returns (packed uint8 [R, C/2] with element 2j in the low nibble, UE8M0
    scale bytes uint8 [R, C/32] = log2(scale) + 127).  This is how the FP8 x FP4
    workload's given weights are produced."""
    R, C = v.shape
    assert C % FP4_BLOCK == 0 and C % 2 == 0
    b = v.reshape(R, C // FP4_BLOCK, FP4_BLOCK)
    amax = b.abs().amax(dim=2)
    mant, expo = torch.frexp(amax / FP4_MAX)
    e = torch.where(mant == 0.5, expo - 1, expo)
    e = torch.where(amax > 0, e, torch.zeros_like(e)).clamp(-127, 127)
    a = (b.abs() / torch.ldexp(torch.ones_like(amax), e)[:, :, None]).clamp(max=FP4_MAX)
    grid = torch.tensor(_E2M1_POS, device=v.device, dtype=a.dtype)
    hi = torch.bucketize(a, grid).clamp(max=len(_E2M1_POS) - 1)      # first grid value >= a
    lo = (hi - 1).clamp(min=0)
    d_lo = a - grid[lo]
    d_hi = grid[hi] - a
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = torch.where(take_hi, hi, lo) | torch.where(b < 0, 8, 0)
    code = code.reshape(R, C).to(torch.uint8)
    packed = code[:, 0::2] | (code[:, 1::2] << 4)
    return packed.contiguous(), (e + 127).to(torch.uint8).contiguous()


def _stacked_fp4(n, rows, cols, g, device):
    packed = torch.empty((n, rows, cols // 2), dtype=torch.uint8, device=device)
    scales = torch.empty((n, rows, cols // FP4_BLOCK), dtype=torch.uint8, device=device)
    for e in range(n):
        w = torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32) * WEIGHT_STD
        packed[e], scales[e] = quantize_rows_e2m1(w)
    return packed, scales


def _stacked_fp8(n, rows, cols, g, device):
    codes = torch.empty((n, rows, cols), dtype=torch.uint8, device=device)
    scales = torch.empty((n, rows // QBLOCK, cols // QBLOCK), dtype=torch.float32, device=device)
    for e in range(n):
        w = torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32) * WEIGHT_STD
        codes[e], scales[e] = quantize_blocks_e4m3(w, QBLOCK)
    return codes, scales


def make_inputs(wl: Workload, seed: int = 0, device="cpu", weights: bool = True) -> dict:
    """All inputs of one layer forward for workload `wl`.

    Keys (bf16 workloads): x [T,H] bf16, w_r [E,H] bf16, bias [E] fp32 or None,
    w_gate/w_up [E,I,H] bf16, w_down [E,H,I] bf16, and for a shared expert
    ws_gate/ws_up [I_sh,H], ws_down [H,I_sh] bf16.
    FP8 workload: x is replaced by x_q [T,H] uint8 (e4m3 codes) + x_scale
    [T,H/128] fp32, and each expert weight W by W_q uint8 + W_s fp32
    [E, rows/128, cols/128].  FP8 x FP4 workload: x as for FP8; W_q is packed e2m1
    uint8 [E, rows, cols/2] and W_s UE8M0 bytes uint8 [E, rows, cols/32].  With
    weights=False only x (and the router) are drawn.
    """
    T, H, I, E = wl.T, wl.H, wl.I, wl.E
    out = {}
    g = _gen(device, seed, "x")
    if wl.skewed:
        gm = _gen(device, seed, "skew_m")
        m = torch.randn((H,), generator=gm, device=device, dtype=torch.float32)
        m = m * (math.sqrt(H) / 2) / m.norm()
        x = torch.randn((T, H), generator=g, device=device, dtype=torch.float32) + m
    else:
        x = torch.randn((T, H), generator=g, device=device, dtype=torch.float32)
    if wl.dtype in (DTYPE_FP8, DTYPE_FP8_FP4):
        out["x_q"], out["x_scale"] = quantize_blocks_e4m3(x, 1)
    else:
        out["x"] = x.to(torch.bfloat16)
    del x

    g = _gen(device, seed, "w_r")
    if wl.skewed:
        gr = _gen(device, seed, "skew_rank")
        rank = torch.randperm(E, generator=gr, device=device).to(torch.float32) + 1.0
        beta = -ZIPF_S * SKEW_TAU * torch.log(rank)
        w_r = torch.randn((E, H), generator=g, device=device, dtype=torch.float32) * WEIGHT_STD
        w_r = w_r + beta[:, None] * (m / (m * m).sum())[None, :]
        out["w_r"] = w_r.to(torch.bfloat16)
    else:
        out["w_r"] = _normal((E, H), WEIGHT_STD, g, device)
    if wl.has_bias:
        gb = _gen(device, seed, "bias")
        out["bias"] = torch.randn((E,), generator=gb, device=device, dtype=torch.float32) * BIAS_STD
    else:
        out["bias"] = None
    if not weights:
        return out

    if wl.dtype == DTYPE_FP8:
        for name, rows, cols in (("w_gate", I, H), ("w_up", I, H), ("w_down", H, I)):
            out[name + "_q"], out[name + "_s"] = _stacked_fp8(E, rows, cols, _gen(device, seed, name), device)
    elif wl.dtype == DTYPE_FP8_FP4:
        for name, rows, cols in (("w_gate", I, H), ("w_up", I, H), ("w_down", H, I)):
            out[name + "_q"], out[name + "_s"] = _stacked_fp4(E, rows, cols, _gen(device, seed, name), device)
    else:
        out["w_gate"] = _stacked_normal(E, (I, H), WEIGHT_STD, _gen(device, seed, "w_gate"), device)
        out["w_up"] = _stacked_normal(E, (I, H), WEIGHT_STD, _gen(device, seed, "w_up"), device)
        out["w_down"] = _stacked_normal(E, (H, I), WEIGHT_STD, _gen(device, seed, "w_down"), device)
    if wl.I_shared:
        Is = wl.I_shared
        out["ws_gate"] = _normal((Is, H), WEIGHT_STD, _gen(device, seed, "ws_gate"), device)
        out["ws_up"] = _normal((Is, H), WEIGHT_STD, _gen(device, seed, "ws_up"), device)
        out["ws_down"] = _normal((H, Is), WEIGHT_STD, _gen(device, seed, "ws_down"), device)
    return out
