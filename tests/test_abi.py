"""The C-ABI library without a GPU: it loads, exports every function include/moe.h
declares, sizes workspaces and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from mixture_experts_ffn_08_b200 import binding as B
from mixture_experts_ffn_08_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if not h.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", h), encoding="utf-8").read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(B._LIB_PATH):
        from mixture_experts_ffn_08_b200 import build
        build.build()
    return B.lib(require_gpu=False)


def test_exports_every_declared_symbol(lib):
    declared = _declared_functions()
    assert {"moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_layer_forward"} <= declared
    raw = ctypes.CDLL(B._LIB_PATH)
    for name in declared:
        assert hasattr(raw, name), name
    assert declared == set(B.EXPORTED), declared ^ set(B.EXPORTED)
    assert lib.moe_abi_version() == 6


def test_params_struct_matches_header():
    src = open(os.path.join(ROOT, "include", "moe.h"), encoding="utf-8").read()
    body = re.search(r"typedef struct moe_params \{(.*?)\} moe_params_t;", src, re.S).group(1)
    fields = re.findall(r"(?:int32_t|float)\s+(\w+);", re.sub(r"/\*.*?\*/", "", body, flags=re.S))
    assert fields == [f[0] for f in B.MoeParams._fields_]
    assert ctypes.sizeof(B.MoeParams) == 4 * len(fields)


def test_sizes(lib):
    for wl in W.ALL.values():
        p = B.params(wl)
        rows = B.moe_max_padded_rows(p)
        bm = B.moe_effective_block_m(p)
        assert bm == 128 and B.moe_effective_block_m(B.params(wl.with_(block_m=256))) == 256
        assert rows == wl.T * wl.K + wl.E * (bm - 1)
        ws = B.moe_workspace_size(p)
        assert ws >= rows * wl.H * (1 if wl.dtype else 2) * 2
        assert B.moe_workspace_size_host(p) > ws
        # router, top-k, 4 permutation kernels (2 for at most 2048 pairs), gate/up, down, combine;
        # FP8: x dequantised for the router and the three weights' scale atoms (the copy into
        # the buckets writes x's)
        perm = 2 if wl.T * wl.K <= 2048 else 4
        # the shared expert's two GEMMs: on a side stream for at most 16384 pairs, else (bf16,
        # routed experts in two-M-tile items) one more group of the routed launches
        merged = (wl.I_shared > 0 and wl.dtype == W.DTYPE_BF16 and wl.T * wl.K > 16384 and wl.T >= 256
                  and wl.T * wl.K >= 256 * wl.E and wl.H % 256 == 0 and wl.I_shared % 128 == 0)
        shared = 2 if wl.I_shared and not merged else 0
        assert B.moe_layer_launch_count(p) == 5 + perm + shared + (4 if wl.dtype else 0)


def test_masked_layout_sizes(lib):
    wl = W.DSV3_DECODE.with_(masked_cap=128)
    p = B.params(wl)
    assert B.moe_max_padded_rows(p) == wl.E * 128
    assert B.moe_effective_block_m(p) == 128
    assert B.moe_workspace_size(p) >= wl.E * 128 * wl.H * 4
    for bad in (dict(masked_cap=100), dict(masked_cap=128, block_m=256), dict(masked_cap=-128)):
        q = B.params(wl.with_(**bad))
        assert B.moe_workspace_size(q) == 0 and B.moe_max_padded_rows(q) == -1


@pytest.mark.parametrize("change", [dict(H=100), dict(I=200), dict(K=0), dict(E=2000), dict(block_m=64),
                                    dict(K=40), dict(n_group=3), dict(topk_group=9),
                                    dict(group_topn=40), dict(score_fn=5), dict(dtype=7),
                                    dict(I_shared=100), dict(T=-1)])
def test_invalid_params_give_no_workspace(lib, change):
    wl = W.DSV3_PREFILL.with_(**change)
    p = B.params(wl)
    assert B.moe_workspace_size(p) == 0
    assert B.moe_max_padded_rows(p) == -1


def test_invalid_args_rejected_on_host(lib):
    p = B.params(W.TINY)
    size = B.moe_workspace_size(p)
    # a null pointer, a misaligned workspace and a short workspace all fail before any launch
    assert lib.moe_route(ctypes.byref(p), None, None, None, None, None, None, 256, size, None) == 1
    assert lib.moe_route(ctypes.byref(p), 256, None, 256, None, 256, 256, 260, size, None) == 1
    assert lib.moe_route(ctypes.byref(p), 256, None, 256, None, 256, 256, 256, 100, None) == 1
    assert lib.moe_combine(ctypes.byref(p), None, None, None, None, None, None) == 1
    bad = B.params(W.TINY.with_(H=100))
    assert lib.moe_layer_forward(ctypes.byref(bad), *([256] * 18), size, None) == 2
    assert B.moe_status_string(2) == "unsupported configuration"


def test_product_path_refuses_to_run_without_cuda(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(B.MoEError):
        B.moe_route(B.params(W.TINY), None, None, None, None, None, None, None, 0, 0)


def test_binding_argument_counts_match_header(lib):
    src = open(os.path.join(ROOT, "include", "moe.h"), encoding="utf-8").read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    for name, params in re.findall(r"\b(moe_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", src):
        n = 0 if params.strip() in ("", "void") else params.count(",") + 1
        assert len(B._SIGS[name][1]) == n, (name, n, len(B._SIGS[name][1]))


def test_selftest_argument_errors_need_no_gpu(lib):
    import ctypes
    assert lib.moe_selftest_bounded_wait(None, 50, None) == 1
    assert lib.moe_selftest_bounded_wait(ctypes.c_void_p(4096), 0, None) == 1       # limit too small
    assert lib.moe_selftest_bounded_wait(ctypes.c_void_p(4096 + 8), 50, None) == 1  # misaligned ws


@pytest.mark.parametrize("dtype", [W.DTYPE_BF16, W.DTYPE_FP8])
def test_empty_batch_returns_ok_without_touching_the_device(lib, dtype):
    """T = 0: after the parameter and workspace checks every entry point returns MOE_OK,
    with NULL for every array that has a T or T*K dimension.  None of these calls issues
    a CUDA call (no counts_out given), so they run without a GPU."""
    wl = W.DSV3_PREFILL.with_(name="empty", T=0, dtype=dtype,
                              I_shared=W.DSV3_PREFILL.I_shared if dtype == W.DTYPE_BF16 else 0)
    p = B.params(wl)
    size, size_host = B.moe_workspace_size(p), lib.moe_workspace_size_host(ctypes.byref(p))
    assert size > 0 and size_host >= size
    ws = 4096  # never dereferenced
    pp = ctypes.byref(p)
    assert lib.moe_route(pp, None, None, None, None, None, None, ws, size, None) == 0
    assert lib.moe_grouped_topk(pp, None, None, None, None, None) == 0
    assert lib.moe_expert_ffn(pp, *([None] * 11), ws, size, None) == 0
    assert lib.moe_combine(pp, None, None, None, None, None, None) == 0
    assert lib.moe_layer_forward(pp, *([None] * 17), ws, size, None) == 0
    assert lib.moe_layer_forward_host(pp, *([None] * 14), ws, size_host, None) == 0
    if wl.I_shared > 0:
        assert lib.moe_shared_expert_ffn(pp, None, None, None, None, None, ws, size, None) == 0
    # the parameter and workspace checks still come first
    assert lib.moe_route(pp, None, None, None, None, None, None, ws, size - 1, None) == 1
    assert lib.moe_layer_forward(pp, *([None] * 17), ws + 8, size, None) == 1
    bad = B.params(wl.with_(H=100))
    assert lib.moe_combine(ctypes.byref(bad), None, None, None, None, None, None) == 2


def test_fp4_launch_counts(lib):
    """FP8 x FP4 layers add one launch to the bf16 layer's: x dequantised for the router
    (the weights bring their scale atoms, and the copy into the buckets writes x's).  The
    bf16 layer has nine, seven when one block does the counting, scan and ranking of at
    most 2048 pairs."""
    for wl in W.FP4.values():
        bf16 = 7 if wl.T * wl.K <= 2048 else 9
        assert B.moe_layer_launch_count(B.params(wl)) == bf16 + 1


def test_trace_kernel_ids_match_the_header():
    """The binding's kernel ids and names follow the header's MOE_K_* enum."""
    src = open(os.path.join(ROOT, "include", "moe.h"), encoding="utf-8").read()
    ids = {name: int(v) for name, v in re.findall(r"\bMOE_K_([A-Z0-9_]+)\s*=\s*(\d+)", src)}
    assert ids["COUNT"] == len(B.KERNEL_NAMES)
    assert (B.K_GATEUP, B.K_DOWN, B.K_SHARED_GATEUP, B.K_SHARED_DOWN, B.K_COMBINE, B.K_DEQUANT_X) == (
        ids["GATEUP"], ids["DOWN"], ids["SHARED_GATEUP"], ids["SHARED_DOWN"], ids["COMBINE"], ids["DEQUANT_X"])
    for name, i in ids.items():
        if name != "COUNT":
            # the names are the header's in lower case; the routed gate/up carries its SwiGLU
            assert B.KERNEL_NAMES[i] == ("gateup_swiglu" if name == "GATEUP" else name.lower()), (name, i)


def test_device_status_bits_match_the_header():
    src = open(os.path.join(ROOT, "include", "moe.h"), encoding="utf-8").read()
    bits = {name: int(v, 16) for name, v in re.findall(r"#define (MOE_DEV_[A-Z_]+) (0x[0-9a-fA-F]+)", src)}
    assert bits == {"MOE_DEV_BAD_EXPERT_ID": B.MOE_DEV_BAD_EXPERT_ID, "MOE_DEV_TIMEOUT": B.MOE_DEV_TIMEOUT,
                    "MOE_DEV_CAPACITY": B.MOE_DEV_CAPACITY, "MOE_DEV_RANGE": B.MOE_DEV_RANGE}
    assert len(set(bits.values())) == len(bits) and all(v & (v - 1) == 0 for v in bits.values())
