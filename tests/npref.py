"""Independent numpy restatements used to pin the oracle.

These are written separately from the oracle's C code (different language,
different structure: whole-matrix numpy operations and library routines such as
np.unpackbits, np.lexsort and matrix products) so that a mistake in one is not
repeated in the other.  Test-only.
"""
import numpy as np


def f16_bits_to_f64(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def bf16_bits_to_f64(bits):
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def unpack_codes(codes_m, bits, rows, cols):
    """Codes of a packed matrix as an int array [rows, cols] (bit-serial reading:
    element j of a block occupies bits bits*j .. bits*j+bits-1, LSB first)."""
    nb = cols // 32
    raw = np.asarray(codes_m, dtype=np.uint8).reshape(rows, nb, 4 * bits)
    b = np.unpackbits(raw, axis=2, bitorder="little").reshape(rows, nb, 32, bits)
    weights = (1 << np.arange(bits)).astype(np.int64)
    return (b.astype(np.int64) * weights).sum(axis=3).reshape(rows, cols)


def dequant(codes_m, scales_m, bits, rows, cols):
    q = unpack_codes(codes_m, bits, rows, cols).astype(np.float64)
    d = f16_bits_to_f64(scales_m).reshape(rows, cols // 32)
    centre = (2 ** bits - 1) / 2.0
    return (q - centre) * np.repeat(d, 32, axis=1)


def expert_mats(shape, codes_e, scales_e):
    H, I, bits = shape.hidden, shape.inter, shape.bits
    cb, sb = shape.mat_code_bytes, shape.mat_scales
    dims = [(I, H), (I, H), (H, I)]
    return [dequant(codes_e[m * cb:(m + 1) * cb], scales_e[m * sb:(m + 1) * sb], bits, *dims[m])
            for m in range(3)]


def swiglu(mats, x):
    """Textbook SwiGLU FFN: Wd @ (silu(Wg @ x) * (Wu @ x)) for x [H] or [T, H]."""
    Wg, Wu, Wd = mats
    g = x @ Wg.T
    u = x @ Wu.T
    a = g / (1.0 + np.exp(-g)) * u
    return a @ Wd.T


def topk_softmax(logits, k):
    """Softmax over all experts, top-k (lower id wins ties), renormalised."""
    logits = np.asarray(logits, dtype=np.float64)
    T, E = logits.shape
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    idx = np.empty((T, k), dtype=np.int64)
    w = np.empty((T, k))
    for t in range(T):
        order = np.lexsort((np.arange(E), -p[t]))  # primary: -p, secondary: id
        idx[t] = order[:k]
        w[t] = p[t, order[:k]] / p[t, order[:k]].sum()
    return idx, w


def round_bf16_rne(v):
    """Round doubles to bf16 (round to nearest even) by brute force over the two
    bf16 neighbours of the value (finite, normal range)."""
    v = np.asarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    for i, x in np.ndenumerate(v):
        f = np.float32(x)  # nearest float; its bf16 neighbours bracket x
        u = int(np.array(f).view(np.uint32)) >> 16
        cands = [(u - 1) & 0xFFFF, u, (u + 1) & 0xFFFF]
        vals = [float(np.array(c << 16, dtype=np.uint32).view(np.float32)) for c in cands]
        best = min(range(3), key=lambda j: (abs(vals[j] - x), cands[j] & 1))
        out[i] = cands[best]
    return out
