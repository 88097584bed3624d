"""Python binding of the C ABI in include/moe.h (ctypes; argument marshalling only).

Every function here has the name of the C entry point it calls and the same argument
order.  Tensor arguments may be torch tensors (their data_ptr() is passed), plain
integer addresses, or None for a NULL pointer; `stream` defaults to torch's current
CUDA stream.  Each call returns the moe_status_t code; `check()` turns a non-zero code
into an exception.  All computation happens in the CUDA library: if libmoe_b200.so is
missing or there is no CUDA device, `lib()` raises instead of falling back to anything.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import workloads as W

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")
_lib = None

MOE_OK = 0
MOE_DEV_BAD_EXPERT_ID = 0x1
MOE_DEV_TIMEOUT = 0x2
MOE_DEV_CAPACITY = 0x4
MOE_DEV_RANGE = 0x8
BLOCK_M = 128

# Kernel ids for tracing (include/moe.h).
K_ROUTER_GEMM, K_TOPK, K_PERM_COUNT, K_PERM_SCAN, K_PERM_RANK, K_PERM_GATHER = range(6)
K_GATEUP, K_DOWN, K_SHARED_GATEUP, K_SHARED_DOWN, K_COMBINE, K_DEQUANT_X = range(6, 12)
K_SCALE_ATOMS = 12
KERNEL_NAMES = ["router_gemm", "topk", "perm_count", "perm_scan", "perm_rank", "perm_gather",
                "gateup_swiglu", "down", "shared_gateup", "shared_down", "combine", "dequant_x",
                "scale_atoms"]


class MoEError(RuntimeError):
    pass


class MoeParams(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("E", ctypes.c_int32), ("K", ctypes.c_int32), ("n_group", ctypes.c_int32),
                ("topk_group", ctypes.c_int32), ("group_topn", ctypes.c_int32),
                ("score_fn", ctypes.c_int32), ("renormalize", ctypes.c_int32),
                ("routed_scale", ctypes.c_float), ("I_shared", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("block_m", ctypes.c_int32),
                ("fused_combine", ctypes.c_int32), ("masked_cap", ctypes.c_int32)]


def params(wl: W.Workload) -> MoeParams:
    return MoeParams(wl.T, wl.H, wl.I, wl.E, wl.K, wl.n_group, wl.topk_group, wl.group_topn,
                     wl.score_fn, int(wl.renormalize), float(wl.routed_scale), wl.I_shared,
                     wl.dtype, wl.block_m, int(wl.fused_combine), wl.masked_cap)


_P = ctypes.c_void_p
_PP = ctypes.POINTER(MoeParams)
_SIGS = {
    "moe_workspace_size": (ctypes.c_size_t, [_PP]),
    "moe_workspace_size_host": (ctypes.c_size_t, [_PP]),
    "moe_max_padded_rows": (ctypes.c_int64, [_PP]),
    "moe_effective_block_m": (ctypes.c_int32, [_PP]),
    "moe_route": (ctypes.c_int, [_PP, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_permute": (ctypes.c_int, [_PP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_grouped_topk": (ctypes.c_int, [_PP, _P, _P, _P, _P, _P]),
    "moe_aux_free_bias_update": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_float, _P, _P]),
    "moe_permute_noalloc": (ctypes.c_int, [_PP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_expert_ffn": (ctypes.c_int, [_PP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                      ctypes.c_size_t, _P]),
    "moe_shared_expert_ffn": (ctypes.c_int, [_PP, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_combine": (ctypes.c_int, [_PP, _P, _P, _P, _P, _P, _P]),
    "moe_layer_forward": (ctypes.c_int, [_PP] + [_P] * 18 + [ctypes.c_size_t, _P]),
    "moe_layer_forward_host": (ctypes.c_int, [_PP] + [_P] * 15 + [ctypes.c_size_t, _P]),
    "moe_layer_forward_host_batches": (ctypes.c_int, [_PP, ctypes.c_int32] + [_P] * 15 + [ctypes.c_size_t, _P]),
    "moe_get_device_status": (ctypes.c_int, [_P, _P, ctypes.POINTER(ctypes.c_int32)]),
    "moe_clear_device_status": (ctypes.c_int, [_P, _P]),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_abi_version": (ctypes.c_int32, []),
    "moe_prepare_fp4_scales": (ctypes.c_int, [_P, ctypes.c_int64, ctypes.c_int32, _P, _P]),
    "moe_selftest_bounded_wait": (ctypes.c_int, [_P, ctypes.c_int32, _P]),
    "moe_trace_enable": (ctypes.c_int, [ctypes.c_uint32, ctypes.c_int32]),
    "moe_trace_disable": (ctypes.c_int, []),
    "moe_trace_collect": (ctypes.c_int32, [ctypes.POINTER(ctypes.c_int32),
                                           ctypes.POINTER(ctypes.c_float), ctypes.c_int32]),
    "moe_layer_launch_count": (ctypes.c_int32, [_PP]),
}

EXPORTED = sorted(_SIGS)


def lib(require_gpu: bool = True):
    """The loaded CUDA library.  Raises if it is not built or (by default) no GPU."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise MoEError(f"CUDA library not built: {_LIB_PATH} (run "
                           "python -m mixture_experts_ffn_08_b200.build)")
        l = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    if require_gpu and not torch.cuda.is_available():
        raise MoEError("no CUDA device: the MoE layer runs only in its CUDA kernels")
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        return t.data_ptr()
    return int(t)


def _stream(s):
    if s is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, torch.cuda.Stream):
        return s.cuda_stream
    return int(s)


def check(status: int, what: str = "moe call"):
    if status != MOE_OK:
        msg = lib(require_gpu=False).moe_status_string(status).decode()
        raise MoEError(f"{what} failed: {msg} ({status})")
    return status


# ------------------------------------------------------------------ sizes
def moe_workspace_size(p: MoeParams) -> int:
    return lib(require_gpu=False).moe_workspace_size(ctypes.byref(p))


def moe_workspace_size_host(p: MoeParams) -> int:
    return lib(require_gpu=False).moe_workspace_size_host(ctypes.byref(p))


def moe_max_padded_rows(p: MoeParams) -> int:
    return lib(require_gpu=False).moe_max_padded_rows(ctypes.byref(p))


def moe_effective_block_m(p: MoeParams) -> int:
    return lib(require_gpu=False).moe_effective_block_m(ctypes.byref(p))


def moe_layer_launch_count(p: MoeParams) -> int:
    return lib(require_gpu=False).moe_layer_launch_count(ctypes.byref(p))


# ------------------------------------------------------------------ stages
def moe_route(p, x, x_scale, w_r, bias, topk_ids, topk_w, ws, ws_bytes, stream=None) -> int:
    return lib().moe_route(ctypes.byref(p), _ptr(x), _ptr(x_scale), _ptr(w_r), _ptr(bias),
                           _ptr(topk_ids), _ptr(topk_w), _ptr(ws), ws_bytes, _stream(stream))


def moe_grouped_topk(p, logits, bias, topk_ids, topk_w, stream=None) -> int:
    return lib().moe_grouped_topk(ctypes.byref(p), _ptr(logits), _ptr(bias), _ptr(topk_ids),
                                  _ptr(topk_w), _stream(stream))


def moe_aux_free_bias_update(counts, E, gamma, bias, stream=None) -> int:
    return lib().moe_aux_free_bias_update(_ptr(counts), E, gamma, _ptr(bias), _stream(stream))


def moe_permute(p, topk_ids, x, x_scale, counts, offsets_padded, row_of_pair, pair_of_row,
                x_perm, x_perm_scale, ws, ws_bytes, stream=None) -> int:
    return lib().moe_permute(ctypes.byref(p), _ptr(topk_ids), _ptr(x), _ptr(x_scale), _ptr(counts),
                             _ptr(offsets_padded), _ptr(row_of_pair), _ptr(pair_of_row),
                             _ptr(x_perm), _ptr(x_perm_scale), _ptr(ws), ws_bytes, _stream(stream))


def moe_permute_noalloc(p, topk_ids, x, x_scale, counts, offsets_padded, row_of_pair,
                        pair_of_row, x_perm, x_perm_scale, device_status, stream=None) -> int:
    """moe_permute without a workspace, for callers that cannot allocate device memory
    for the library; its scratch is a fixed device array inside the library."""
    return lib().moe_permute_noalloc(ctypes.byref(p), _ptr(topk_ids), _ptr(x), _ptr(x_scale),
                                     _ptr(counts), _ptr(offsets_padded), _ptr(row_of_pair),
                                     _ptr(pair_of_row), _ptr(x_perm), _ptr(x_perm_scale),
                                     _ptr(device_status), _stream(stream))


def moe_expert_ffn(p, x_perm, x_perm_scale, offsets_padded, counts, w_gate, w_up, w_down,
                   w_gate_scale, w_up_scale, w_down_scale, y_perm, ws, ws_bytes, stream=None) -> int:
    return lib().moe_expert_ffn(ctypes.byref(p), _ptr(x_perm), _ptr(x_perm_scale),
                                _ptr(offsets_padded), _ptr(counts), _ptr(w_gate), _ptr(w_up),
                                _ptr(w_down),
                                _ptr(w_gate_scale), _ptr(w_up_scale), _ptr(w_down_scale),
                                _ptr(y_perm), _ptr(ws), ws_bytes, _stream(stream))


def moe_shared_expert_ffn(p, x, ws_gate, ws_up, ws_down, y_shared, ws, ws_bytes, stream=None) -> int:
    return lib().moe_shared_expert_ffn(ctypes.byref(p), _ptr(x), _ptr(ws_gate), _ptr(ws_up),
                                       _ptr(ws_down), _ptr(y_shared), _ptr(ws), ws_bytes,
                                       _stream(stream))


def moe_combine(p, y_perm, row_of_pair, topk_w, y_shared, out, stream=None) -> int:
    return lib().moe_combine(ctypes.byref(p), _ptr(y_perm), _ptr(row_of_pair), _ptr(topk_w),
                             _ptr(y_shared), _ptr(out), _stream(stream))


def moe_layer_forward(p, x, x_scale, w_r, bias, w_gate, w_up, w_down, w_gate_scale, w_up_scale,
                      w_down_scale, ws_gate, ws_up, ws_down, out, topk_ids_out, topk_w_out,
                      counts_out, ws, ws_bytes, stream=None) -> int:
    return lib().moe_layer_forward(
        ctypes.byref(p), _ptr(x), _ptr(x_scale), _ptr(w_r), _ptr(bias), _ptr(w_gate), _ptr(w_up),
        _ptr(w_down), _ptr(w_gate_scale), _ptr(w_up_scale), _ptr(w_down_scale), _ptr(ws_gate),
        _ptr(ws_up), _ptr(ws_down), _ptr(out), _ptr(topk_ids_out), _ptr(topk_w_out),
        _ptr(counts_out), _ptr(ws), ws_bytes, _stream(stream))


def moe_layer_forward_host(p, x_host, x_scale_host, w_r, bias, w_gate, w_up, w_down, w_gate_scale,
                           w_up_scale, w_down_scale, ws_gate, ws_up, ws_down, out_host, ws,
                           ws_bytes, stream=None) -> int:
    return lib().moe_layer_forward_host(
        ctypes.byref(p), _ptr(x_host), _ptr(x_scale_host), _ptr(w_r), _ptr(bias), _ptr(w_gate),
        _ptr(w_up), _ptr(w_down), _ptr(w_gate_scale), _ptr(w_up_scale), _ptr(w_down_scale),
        _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), _ptr(out_host), _ptr(ws), ws_bytes,
        _stream(stream))


def _ptr_array(items):
    """ctypes array of void* from tensors / addresses / None (NULL), or NULL if items is None."""
    if items is None:
        return None
    arr = (ctypes.c_void_p * len(items))(*[_ptr(t) for t in items])
    return ctypes.cast(arr, ctypes.c_void_p).value, arr


def moe_layer_forward_host_batches(p, x_host, x_scale_host, w_r, bias, w_gate, w_up, w_down, w_gate_scale,
                                   w_up_scale, w_down_scale, ws_gate, ws_up, ws_down, out_host, ws,
                                   ws_bytes, stream=None) -> int:
    """x_host, x_scale_host (or None) and out_host are lists of host tensors, one per batch."""
    n = len(x_host)
    if len(out_host) != n or (x_scale_host is not None and len(x_scale_host) != n):
        raise ValueError("one x, x_scale and out buffer per batch")
    xs = _ptr_array(x_host)
    ss = _ptr_array(x_scale_host)
    os_ = _ptr_array(out_host)
    return lib().moe_layer_forward_host_batches(
        ctypes.byref(p), n, xs[0], ss[0] if ss else None, _ptr(w_r), _ptr(bias), _ptr(w_gate), _ptr(w_up),
        _ptr(w_down), _ptr(w_gate_scale), _ptr(w_up_scale), _ptr(w_down_scale), _ptr(ws_gate), _ptr(ws_up),
        _ptr(ws_down), os_[0], _ptr(ws), ws_bytes, _stream(stream))


# ------------------------------------------------------------------ status, tracing
def moe_get_device_status(ws, stream=None) -> int:
    v = ctypes.c_int32(0)
    check(lib().moe_get_device_status(_ptr(ws), _stream(stream), ctypes.byref(v)), "status read")
    return v.value


def moe_clear_device_status(ws, stream=None) -> int:
    return lib().moe_clear_device_status(_ptr(ws), _stream(stream))


def moe_status_string(s: int) -> str:
    return lib(require_gpu=False).moe_status_string(s).decode()


def moe_abi_version() -> int:
    return lib(require_gpu=False).moe_abi_version()


def moe_selftest_bounded_wait(ws, limit_ms: int, stream=None) -> int:
    return lib().moe_selftest_bounded_wait(_ptr(ws), limit_ms, _stream(stream))


def moe_prepare_fp4_scales(scale_bytes, rows: int, K: int, atoms, stream=None) -> int:
    """scale_bytes: UE8M0 bytes [rows, K/32] (read as [rows, K/128] 32-bit words);
    atoms: rows*K/32 bytes, written."""
    return lib().moe_prepare_fp4_scales(_ptr(scale_bytes), rows, K, _ptr(atoms), _stream(stream))


def moe_trace_enable(kernel_mask: int, capacity: int) -> int:
    return lib().moe_trace_enable(kernel_mask, capacity)


def moe_trace_disable() -> int:
    return lib().moe_trace_disable()


def moe_trace_collect(max_out: int = 4096):
    ids = (ctypes.c_int32 * max_out)()
    ms = (ctypes.c_float * max_out)()
    n = lib().moe_trace_collect(ids, ms, max_out)
    return [(ids[i], ms[i]) for i in range(n)]
