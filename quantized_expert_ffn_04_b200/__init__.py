"""Python binding of the Strata MoE layer library (libstrata_moe.so).

Argument marshalling only: every function forwards to the C entry point of
the same name declared in include/strata_moe.h, and every step of the layer
runs in the library's CUDA kernels.  PyTorch is used only for device memory
and streams in the `Layer` convenience wrapper.  There is no fallback: if the
shared library has not been built, importing this package raises.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# STRATA_MOE_CHECKED=1 loads the checked build instead (every device-side
# gather/scatter index tested; a bad one reports STRATA_ERR_BOUNDS)
LIB_PATH = os.path.join(_HERE, "libstrata_moe_checked.so" if os.environ.get("STRATA_MOE_CHECKED") == "1"
                        else "libstrata_moe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: the CUDA library must be built first "
        "(python quantized_expert_ffn_04_b200/build.py, or __graft_entry__.build())")

_lib = C.CDLL(LIB_PATH)

STRATA_OK, STRATA_ERR_INVALID_ARG, STRATA_ERR_UNSUPPORTED, STRATA_ERR_OOM, STRATA_ERR_CUDA, \
    STRATA_ERR_TIMEOUT, STRATA_ERR_BOUNDS = range(7)
STRATA_OPT_PATH, STRATA_OPT_WAIT_BUDGET, STRATA_OPT_DECODE_MAX_T = 1, 2, 3

# every symbol the header declares
SYMBOLS = ("strata_moe_create", "strata_moe_destroy", "strata_moe_route", "strata_moe_forward",
           "strata_moe_forward_host", "strata_moe_rmsnorm", "strata_moe_stack_forward",
           "strata_moe_sync_status", "strata_moe_last_error", "strata_moe_debug_dequant",
           "strata_moe_set_option", "strata_moe_selftest_wait", "strata_moe_version",
           "strata_moe_set_probe", "strata_moe_launch_count", "strata_moe_route_noalloc",
           "strata_moe_debug_fail_alloc", "strata_moe_debug_live_allocs",
           "strata_ep_expert_range", "strata_ep_plan", "strata_ep_gather_rows",
           "strata_moe_expert_rows", "strata_moe_combine_rows", "strata_moe_debug_screen")


class strata_moe_config(C.Structure):
    _fields_ = [("hidden", C.c_int32), ("n_experts", C.c_int32), ("top_k", C.c_int32),
                ("inter", C.c_int32), ("quant_bits", C.c_int32), ("block", C.c_int32),
                ("max_tokens", C.c_int32), ("has_router_bias", C.c_int32)]


class strata_moe_weights(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("scales", C.c_void_p), ("router_w", C.c_void_p),
                ("router_b", C.c_void_p), ("shared_codes", C.c_void_p),
                ("shared_scales", C.c_void_p)]


class StrataError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"strata status {status}: {message}")
        self.status = status


_P, _I, _I64 = C.c_void_p, C.c_int, C.c_int64
_sig = {
    "strata_moe_create": [C.POINTER(strata_moe_config), C.POINTER(strata_moe_weights), _I,
                          C.POINTER(C.c_void_p)],
    "strata_moe_route": [_P, _P, _I, _P, _P, _P, _P, _P],
    "strata_moe_forward": [_P, _P, _I, _P, _P],
    "strata_moe_forward_host": [_P, _P, _I, _P, _P],
    "strata_moe_rmsnorm": [_P, _P, _I, _I, _P],
    "strata_moe_stack_forward": [C.POINTER(C.c_void_p), _I, _P, _I, _P, _P],
    "strata_moe_sync_status": [_P, _P],
    "strata_moe_debug_dequant": [_P, _I, _I, _I, _I, _I, _P],
    "strata_moe_set_option": [_P, _I, _I64],
    "strata_moe_selftest_wait": [_I, _I64],
    "strata_moe_set_probe": [_P, _I, _P, _P],
    "strata_moe_launch_count": [_P, _I],
    "strata_moe_route_noalloc": [_P, _I, _I, _P, _P, _I, _I, _P, _P, _P, _P, _P],
    "strata_moe_debug_fail_alloc": [_I64],
    "strata_moe_debug_screen": [_P, _P, _I, _P, _P],
    "strata_ep_expert_range": [_I, _I, _I, _P, _P],
    "strata_ep_plan": [_P, _I, _I, _I, _I, _P, _P, _P],
    "strata_ep_gather_rows": [_P, _P, _I, _I, _I, _P, _P],
    "strata_moe_expert_rows": [_P, _P, _P, _I, _I, _I, _P, _P, _P],
    "strata_moe_combine_rows": [_P, _P, _I, _P, _P, _P, _P, _I, _P, _P],
}
for _name, _args in _sig.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = C.c_int
_lib.strata_moe_destroy.argtypes = [_P]
_lib.strata_moe_destroy.restype = None
_lib.strata_moe_last_error.restype = C.c_char_p
_lib.strata_moe_version.restype = C.c_char_p
_lib.strata_moe_debug_live_allocs.argtypes = []
_lib.strata_moe_debug_live_allocs.restype = C.c_int64


def _check(status: int):
    if status != STRATA_OK:
        raise StrataError(status, strata_moe_last_error())


def strata_moe_last_error() -> str:
    return _lib.strata_moe_last_error().decode()


def strata_moe_version() -> str:
    return _lib.strata_moe_version().decode()


def strata_moe_create(cfg: strata_moe_config, weights: strata_moe_weights, device: int = 0):
    h = C.c_void_p()
    _check(_lib.strata_moe_create(C.byref(cfg), C.byref(weights), device, C.byref(h)))
    return h


def strata_moe_destroy(h) -> None:
    _lib.strata_moe_destroy(h)


def strata_moe_route(h, x, T, idx, w, offsets=None, lst=None, stream=None) -> None:
    _check(_lib.strata_moe_route(h, x, T, idx, w, offsets, lst, stream))


def strata_moe_forward(h, x, T, y, stream=None) -> None:
    _check(_lib.strata_moe_forward(h, x, T, y, stream))


def strata_moe_forward_host(h, x_host, T, y_host, stream=None) -> None:
    _check(_lib.strata_moe_forward_host(h, x_host, T, y_host, stream))


def strata_moe_rmsnorm(h_dev, xn_dev, T, H, stream=None) -> None:
    _check(_lib.strata_moe_rmsnorm(h_dev, xn_dev, T, H, stream))


def strata_moe_stack_forward(layers, h_dev, T, h_trace=None, stream=None) -> None:
    arr = (C.c_void_p * len(layers))(*[l.value if isinstance(l, C.c_void_p) else l
                                       for l in layers])
    _check(_lib.strata_moe_stack_forward(arr, len(layers), h_dev, T, h_trace, stream))


def strata_moe_sync_status(h, stream=None) -> None:
    _check(_lib.strata_moe_sync_status(h, stream))


def strata_moe_debug_dequant(h, expert, mat, row0, nrows, kind, out_host) -> None:
    _check(_lib.strata_moe_debug_dequant(h, expert, mat, row0, nrows, kind, out_host))


def strata_moe_set_option(h, option, value) -> None:
    _check(_lib.strata_moe_set_option(h, option, int(value)))


def strata_ep_expert_range(rank, n_ranks, n_experts) -> tuple[int, int]:
    b, e = C.c_int32(), C.c_int32()
    _check(_lib.strata_ep_expert_range(rank, n_ranks, n_experts, C.byref(b), C.byref(e)))
    return b.value, e.value


def strata_ep_plan(idx, n_experts, n_ranks):
    """idx: int32 numpy [T][k] (host).  Returns (send_counts [n_ranks],
    send_pick [T*k], slot [T*k]) as int32 numpy arrays."""
    import numpy as np
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    counts = np.zeros(n_ranks, dtype=np.int32)
    pick = np.zeros(T * k, dtype=np.int32)
    slot = np.zeros(T * k, dtype=np.int32)
    _check(_lib.strata_ep_plan(idx.ctypes.data, T, k, n_experts, n_ranks, counts.ctypes.data,
                               pick.ctypes.data, slot.ctypes.data))
    return counts, pick, slot


def strata_ep_gather_rows(src, rows, n, n_src, row_bytes, dst, stream=None) -> None:
    _check(_lib.strata_ep_gather_rows(src, rows, n, n_src, row_bytes, dst, stream))


def strata_moe_expert_rows(h, x, ids, n, n_shared, prefill, y, yshared, stream=None) -> None:
    _check(_lib.strata_moe_expert_rows(h, x, ids, n, n_shared, int(prefill), y, yshared, stream))


def strata_moe_combine_rows(h, x, T, idx, w, slot, y, prefill, out, stream=None) -> None:
    _check(_lib.strata_moe_combine_rows(h, x, T, idx, w, slot, y, int(prefill), out, stream))


def strata_moe_debug_screen(h, x, T, a_host, eps_host) -> None:
    _check(_lib.strata_moe_debug_screen(h, x, T, a_host, eps_host))


def strata_moe_debug_fail_alloc(n) -> None:
    _check(_lib.strata_moe_debug_fail_alloc(int(n)))


def strata_moe_debug_live_allocs() -> int:
    return int(_lib.strata_moe_debug_live_allocs())


def strata_moe_selftest_wait(device, budget_cycles) -> None:
    _check(_lib.strata_moe_selftest_wait(device, int(budget_cycles)))


def strata_moe_set_probe(h, stage, ev_begin, ev_end) -> None:
    _check(_lib.strata_moe_set_probe(h, stage, ev_begin, ev_end))


def strata_moe_launch_count(h, T) -> int:
    return _lib.strata_moe_launch_count(h, T)


def strata_moe_route_noalloc(x, T, H, router_w, router_b, E, k, idx, w, offsets=None, lst=None,
                             stream=None) -> None:
    _check(_lib.strata_moe_route_noalloc(x, T, H, router_w, router_b, E, k, idx, w, offsets, lst,
                                         stream))


# ----------------------------------------------------------------- convenience
def make_config(shape, max_tokens: int) -> strata_moe_config:
    """Config from any object with hidden/n_experts/top_k/inter/bits/router_bias."""
    return strata_moe_config(shape.hidden, shape.n_experts, shape.top_k, shape.inter, shape.bits,
                             32, max_tokens, 1 if shape.router_bias else 0)


def make_weights(layer) -> tuple[strata_moe_weights, list]:
    """Weights struct from numpy arrays (any object with codes, scales, router_w,
    router_b, shared_codes, shared_scales).  Returns the struct and the arrays
    it points into (keep them alive until create returns)."""
    import numpy as np
    keep = [np.ascontiguousarray(layer.codes, dtype=np.uint8),
            np.ascontiguousarray(layer.scales, dtype=np.uint16),
            np.ascontiguousarray(layer.router_w, dtype=np.float32),
            None if layer.router_b is None else np.ascontiguousarray(layer.router_b,
                                                                    dtype=np.float32),
            np.ascontiguousarray(layer.shared_codes, dtype=np.uint8),
            np.ascontiguousarray(layer.shared_scales, dtype=np.uint16)]
    ptr = [None if a is None else a.ctypes.data for a in keep]
    return strata_moe_weights(*ptr), keep


def _stream_ptr(stream):
    return None if stream is None else stream.cuda_stream


class Layer:
    """One MoE layer on a CUDA device; torch tensors in and out."""

    def __init__(self, layer, max_tokens: int, device: int = 0):
        self.shape = layer.shape
        self.device = device
        cfg = make_config(layer.shape, max_tokens)
        w, keep = make_weights(layer)
        self.handle = strata_moe_create(cfg, w, device)
        del keep

    def close(self):
        if self.handle is not None:
            strata_moe_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_option(self, option, value):
        strata_moe_set_option(self.handle, option, value)

    def forward(self, x, out=None, stream=None):
        import torch
        T = x.shape[0]
        if out is None:
            out = torch.empty_like(x)
        strata_moe_forward(self.handle, x.data_ptr(), T, out.data_ptr(), _stream_ptr(stream))
        return out

    def route(self, x, stream=None):
        import torch
        T, k, E = x.shape[0], self.shape.top_k, self.shape.n_experts
        dev = x.device
        idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        w = torch.empty((T, k), dtype=torch.float32, device=dev)
        off = torch.empty(E + 1, dtype=torch.int32, device=dev)
        lst = torch.empty(T * k, dtype=torch.int32, device=dev)
        strata_moe_route(self.handle, x.data_ptr(), T, idx.data_ptr(), w.data_ptr(),
                         off.data_ptr(), lst.data_ptr(), _stream_ptr(stream))
        return idx, w, off, lst

    def sync_status(self, stream=None):
        strata_moe_sync_status(self.handle, _stream_ptr(stream))

    def debug_dequant(self, expert, mat, row0, nrows, kind=0):
        import numpy as np
        cols = self.shape.hidden if mat < 2 else self.shape.inter
        out = np.empty((nrows, cols), dtype=np.float32)
        strata_moe_debug_dequant(self.handle, expert, mat, row0, nrows, kind,
                                 out.ctypes.data)
        return out
