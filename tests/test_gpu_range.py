"""The fp16 token operand across bf16's range (needs a B200).

The expert kernels multiply in fp16, whose range (65504 largest, 2^-14
smallest normal) is far narrower than bf16's.  Every token row is scaled by an
exact power of two before the conversion (the token prescale), and the layer
output is scaled back after the combine.  These cases put rows outside fp16's
range through every path and compare each token row with the oracle's fp64
output on its own scale: max |err| <= 2e-2 max |ref| and sum |err| <= 5e-3
sum |ref| per row, and a row whose exact output rounds to zero in bf16 must
come out zero.

Rows (H = 2560, the Flash-Next-shaped layer):
  normal   ~N(0, 1)
  big      ~N(0, 1) * 3e5: entries from ~6.6e4 up to ~1e6 (fp16 overflows)
  spiky    ~N(0, 1) with a few entries of 1e5 .. 1e6
  small    ~N(0, 1) * 1e-10 (fp16 flushes every entry to zero)
  subnorm  bf16 subnormals (~1e-39): the exact output rounds to zero
"""
import numpy as np
import pytest

import gen
import oracle
from tests import npref
from tests.gpu_util import THREADS, from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import quantized_expert_ffn_04_b200 as qe  # noqa: E402

KINDS = ("normal", "big", "spiky", "small", "subnorm")


def range_rows(T, H, seed):
    """T rows cycling through KINDS; returns (bf16 bits [T][H], kinds [T])."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H)).astype(np.float64)
    kinds = []
    for t in range(T):
        kind = KINDS[t % len(KINDS)]
        kinds.append(kind)
        if kind == "big":
            x[t] *= 3e5
        elif kind == "spiky":
            pos = rng.choice(H, size=4, replace=False)
            x[t, pos] = rng.uniform(1e5, 1e6, size=4) * rng.choice([-1.0, 1.0], size=4)
        elif kind == "small":
            x[t] *= 1e-10
        elif kind == "subnorm":
            x[t] *= 2.0 ** -130  # below bf16's smallest normal (2^-126)
    bits = gen.f32_to_bf16_bits(x.astype(np.float32))
    return bits, kinds


def check_rows(y_bits, ref, kinds, label):
    y = npref.bf16_bits_to_f64(y_bits)
    assert np.all(np.isfinite(y)), f"{label}: non-finite output"
    for t, kind in enumerate(kinds):
        r = ref[t]
        scale = np.abs(r).max()
        err = np.abs(y[t] - r)
        if scale == 0.0 or scale < 2.0 ** -133:
            # the exact output rounds to zero in bf16
            assert np.all(np.abs(y[t]) <= 2.0 ** -126), f"{label}: row {t} ({kind}) not ~0"
            continue
        assert err.max() <= 2e-2 * scale, \
            f"{label}: row {t} ({kind}) max err {err.max() / scale:.3e} of its max"
        assert err.sum() <= 5e-3 * np.abs(r).sum(), \
            f"{label}: row {t} ({kind}) mean rel err {err.sum() / np.abs(r).sum():.3e}"


CASES = [  # name, shape, T, path (0 auto, 1 decode chain, 2 prefill GEMM, 3 fused decode)
    ("fused-T5", gen.FLASH2, 5, 3),
    ("fused-T15", gen.FLASH2, 15, 3),
    ("chain-T10", gen.FLASH2, 10, 1),
    ("prefill-T20", gen.FLASH2, 20, 2),
    ("prefill-T300", gen.FLASH2, 300, 2),
    ("fused3-T10", gen.FLASH3, 10, 3),
    ("prefill3-T40", gen.FLASH3, 40, 2),
]


@pytest.mark.parametrize("name,shape,T,path", CASES, ids=[c[0] for c in CASES])
def test_out_of_fp16_range_rows(name, shape, T, path):
    w = gen.layer_weights(shape, seed=0)
    x, kinds = range_rows(T, shape.hidden, seed=11)
    L = qe.Layer(w, max_tokens=T)
    L.set_option(qe.STRATA_OPT_PATH, path)
    y = from_dev_bf16(L.forward(to_dev_bf16(x)))
    L.sync_status()
    L.close()
    sel = np.arange(T, dtype=np.int32) if T <= 40 else np.arange(0, T, 7, dtype=np.int32)
    _, ref, _, _ = oracle.moe_forward(w, x, sel=sel, threads=THREADS)
    check_rows(y[sel], ref, [kinds[i] for i in sel], name)

