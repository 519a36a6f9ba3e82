"""CPU oracle of the Strata MoE layer forward -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package.  The product path (the CUDA library and its Python
binding) never imports, loads or calls it, and the two share no code: this
package only loads ``strata_oracle.c`` (plain C, built here with gcc) through
ctypes and marshals numpy arrays.

Every function below forwards to the C function of the same name; the C file's
header states the layer definition, the precision of each step and the sources.

Parity status: every function is pinned by the ``-m "not gpu"`` tests (worked
blocks, closed forms, textbook special cases, brute force, invariants); none is
"parity unpinned".
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "strata_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_strata_oracle.so")
_lib = None
_lock = threading.Lock()


def _cpu_has_fma() -> bool:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("flags"):
                    return " fma " in f" {line.split(':', 1)[1].strip()} "
    except OSError:
        pass
    return False


def build(force: bool = False) -> str:
    """Compile strata_oracle.c into a shared library (idempotent)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    flags = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c99", "-shared", "-fPIC"]
    if _cpu_has_fma():
        flags.append("-mfma")  # explicit fmaf() becomes one instruction; no contraction
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *flags, "-o", tmp, _SRC, "-lm"], check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = C.CDLL(build())
            P = C.c_void_p
            i32, sz = C.c_int, C.c_size_t
            L.orc_f16_to_f64.restype = C.c_double
            L.orc_f16_to_f64.argtypes = [C.c_uint16]
            L.orc_bf16_to_f32.restype = C.c_float
            L.orc_bf16_to_f32.argtypes = [C.c_uint16]
            L.orc_f64_to_bf16.restype = C.c_uint16
            L.orc_f64_to_bf16.argtypes = [C.c_double]
            L.orc_f64_to_f16.restype = C.c_uint16
            L.orc_f64_to_f16.argtypes = [C.c_double]
            L.orc_code.restype = i32
            L.orc_code.argtypes = [P, i32, i32]
            L.orc_weight.restype = C.c_double
            L.orc_weight.argtypes = [P, P, i32, i32, i32, i32]
            L.orc_dequant_rows.restype = None
            L.orc_dequant_rows.argtypes = [P, P, i32, i32, i32, i32, P]
            L.orc_router_logits.restype = None
            L.orc_router_logits.argtypes = [P, i32, i32, P, P, i32, P]
            L.orc_route.restype = None
            L.orc_route.argtypes = [P, i32, i32, i32, P, P]
            L.orc_dispatch.restype = None
            L.orc_dispatch.argtypes = [P, i32, i32, i32, P, P, P, P]
            L.orc_expert_ffn.restype = None
            L.orc_expert_ffn.argtypes = [P, P, i32, i32, i32, P, P]
            L.orc_moe_forward.restype = i32
            L.orc_moe_forward.argtypes = [i32, i32, i32, i32, i32, P, P, P, P, P, P, P, i32, P,
                                          i32, P, P, P, P]
            L.orc_rmsnorm.restype = None
            L.orc_rmsnorm.argtypes = [P, i32, i32, P]
            L.orc_residual_add.restype = None
            L.orc_residual_add.argtypes = [P, P, sz]
            _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- formats
def f16_to_f64(bits: int) -> float:
    return lib().orc_f16_to_f64(int(bits))


def f64_to_bf16(v: float) -> int:
    return lib().orc_f64_to_bf16(float(v))


def f64_to_f16(v: float) -> int:
    return lib().orc_f64_to_f16(float(v))


def code(block: np.ndarray, bits: int, j: int) -> int:
    block = _c(block, np.uint8)
    return lib().orc_code(_p(block), bits, j)


# ---------------------------------------------------------------- dequant
def mat_slices(shape, codes_e: np.ndarray, scales_e: np.ndarray, m: int):
    """Packed codes/scales of matrix m (0 gate, 1 up, 2 down) of one expert."""
    cb, sb = shape.mat_code_bytes, shape.mat_scales
    return codes_e[m * cb:(m + 1) * cb], scales_e[m * sb:(m + 1) * sb]


def expert_slices(shape, codes: np.ndarray, scales: np.ndarray, e: int):
    cb, sb = 3 * shape.mat_code_bytes, 3 * shape.mat_scales
    return codes[e * cb:(e + 1) * cb], scales[e * sb:(e + 1) * sb]


def dequant_rows(codes_m, scales_m, bits: int, cols: int, row0: int, nrows: int) -> np.ndarray:
    codes_m, scales_m = _c(codes_m, np.uint8), _c(scales_m, np.uint16)
    out = np.empty((nrows, cols), dtype=np.float64)
    lib().orc_dequant_rows(_p(codes_m), _p(scales_m), bits, cols, row0, nrows, _p(out))
    return out


# ---------------------------------------------------------------- routing
def router_logits(x_bits: np.ndarray, W: np.ndarray, b: np.ndarray | None,
                  threads: int = 1) -> np.ndarray:
    """fp32 logits [T, E]; `threads` > 1 splits the tokens across threads."""
    x_bits, W = _c(x_bits, np.uint16), _c(W, np.float32)
    T, H = x_bits.shape
    E = W.shape[0]
    b = None if b is None else _c(b, np.float32)
    out = np.empty((T, E), dtype=np.float32)
    L = lib()

    def run(lo, hi):
        if hi > lo:
            L.orc_router_logits(_p(x_bits[lo:hi]), hi - lo, H, _p(W), _p(b), E, _p(out[lo:hi]))

    threads = max(1, min(threads, T))
    bounds = np.linspace(0, T, threads + 1).astype(int)
    if threads == 1:
        run(0, T)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda i: run(bounds[i], bounds[i + 1]), range(threads)))
    return out


def route(logits: np.ndarray, k: int):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    lib().orc_route(_p(logits), T, E, k, _p(idx), _p(w))
    return idx, w


def dispatch(idx: np.ndarray, E: int):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    cnt = np.empty(E, dtype=np.int32)
    off = np.empty(E + 1, dtype=np.int32)
    lst = np.empty(T * k, dtype=np.int32)
    slot = np.empty((T, k), dtype=np.int32)
    lib().orc_dispatch(_p(idx), T, k, E, _p(cnt), _p(off), _p(lst), _p(slot))
    return cnt, off, lst, slot


# ---------------------------------------------------------------- experts
def expert_ffn(codes_e, scales_e, bits: int, H: int, I: int, x: np.ndarray) -> np.ndarray:
    codes_e, scales_e = _c(codes_e, np.uint8), _c(scales_e, np.uint16)
    x = _c(x, np.float64)
    y = np.empty(H, dtype=np.float64)
    lib().orc_expert_ffn(_p(codes_e), _p(scales_e), bits, H, I, _p(x), _p(y))
    return y


def moe_forward(layer, x_bits: np.ndarray, sel=None, threads: int = 1):
    """Layer forward for tokens `sel` (default: all).

    `layer` is any object with the attributes of gen.LayerWeights.  Returns
    (y_bf16 bits [n,H], y_f64 [n,H], idx [n,k], w [n,k]).  `threads` > 1 splits
    the token list across threads (each thread runs the same C code on its own
    tokens; tokens do not interact in this layer)."""
    s = layer.shape
    x_bits = _c(x_bits, np.uint16)
    T, H = x_bits.shape
    sel = np.arange(T, dtype=np.int32) if sel is None else _c(sel, np.int32)
    n = len(sel)
    yb = np.empty((n, H), dtype=np.uint16)
    yf = np.empty((n, H), dtype=np.float64)
    idx = np.empty((n, s.top_k), dtype=np.int32)
    w = np.empty((n, s.top_k), dtype=np.float64)
    codes, scales = _c(layer.codes, np.uint8), _c(layer.scales, np.uint16)
    rw = _c(layer.router_w, np.float32)
    rb = None if layer.router_b is None else _c(layer.router_b, np.float32)
    sc, ss = _c(layer.shared_codes, np.uint8), _c(layer.shared_scales, np.uint16)
    L = lib()

    def run(lo, hi):
        if hi <= lo:
            return
        sub = np.ascontiguousarray(sel[lo:hi])
        rc = L.orc_moe_forward(s.hidden, s.n_experts, s.top_k, s.inter, s.bits, _p(codes),
                               _p(scales), _p(rw), _p(rb), _p(sc), _p(ss), _p(x_bits), T,
                               _p(sub), hi - lo, _p(yb[lo:hi]), _p(yf[lo:hi]), _p(idx[lo:hi]),
                               _p(w[lo:hi]))
        if rc != 0:
            raise ValueError(f"orc_moe_forward failed: {rc}")

    threads = max(1, min(threads, n))
    if threads == 1:
        run(0, n)
    else:
        bounds = np.linspace(0, n, threads + 1).astype(int)
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda i: run(bounds[i], bounds[i + 1]), range(threads)))
    return yb, yf, idx, w


# ---------------------------------------------------------------- stack pieces
def rmsnorm(h_bits: np.ndarray) -> np.ndarray:
    h_bits = _c(h_bits, np.uint16)
    T, H = h_bits.shape
    out = np.empty_like(h_bits)
    lib().orc_rmsnorm(_p(h_bits), T, H, _p(out))
    return out


def residual_add(h_bits: np.ndarray, y_bits: np.ndarray) -> np.ndarray:
    h = np.array(h_bits, dtype=np.uint16, copy=True, order="C")
    y = _c(y_bits, np.uint16)
    lib().orc_residual_add(_p(h), _p(y), h.size)
    return h


def stack_forward(layers, h_bits: np.ndarray, sel=None, threads: int = 1):
    """h <- h + MoE_l(RMSNorm(h)) for every layer, for tokens `sel`.

    Returns (h_final [n,H] bits, per-layer inputs [L, n, H] bits)."""
    h_bits = _c(h_bits, np.uint16)
    if sel is not None:
        h = np.ascontiguousarray(h_bits[np.asarray(sel)])
    else:
        h = h_bits.copy()
    ins = []
    for layer in layers:
        ins.append(h.copy())
        xn = rmsnorm(h)
        yb, _, _, _ = moe_forward(layer, xn, threads=threads)
        h = residual_add(h, yb)
    return h, np.stack(ins)
