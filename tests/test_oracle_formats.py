"""Pins for the oracle's number-format helpers and the packed weight format.

The packed block formats (2-bit w = d*(q-1.5), 3-bit w = d*(q-3.5), blocks of
32 along the input dimension, fp16 scale) are the layer specification's; the
pages only name the 2-3 bit builds ("Strata Runs 125B Qwen3.8-Flash-Next on a
12GB Gaming GPU at Up to 94 Tokens/s", sections "The numbers, measured by the
author" and "Caveats").
"""
import numpy as np
import pytest

import gen
import oracle
from tests.conftest import golden
from tests import npref


def _golden_blocks():
    rows = []
    for line in open(golden("dequant_blocks.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        bits, scale, data, expect = [s.strip() for s in line.split("|")]
        rows.append((int(bits), int(scale, 16), bytes(int(h, 16) for h in data.split()),
                     [float(v) for v in expect.split()]))
    return rows


@pytest.mark.parametrize("bits,scale,data,expect", _golden_blocks())
def test_worked_blocks(bits, scale, data, expect):
    codes = np.frombuffer(data, dtype=np.uint8)
    scales = np.array([scale], dtype=np.uint16)
    got = oracle.dequant_rows(codes, scales, bits, 32, 0, 1)[0]
    assert list(got) == expect


def test_f16_decode_ieee_values():
    # IEEE 754 binary16 definitions
    cases = {0x3C00: 1.0, 0x3800: 0.5, 0xC000: -2.0, 0x7BFF: 65504.0, 0x0400: 2.0 ** -14,
             0x0001: 2.0 ** -24, 0x03FF: 1023 * 2.0 ** -24, 0x3555: 0.333251953125,
             0x0000: 0.0}
    for bits, v in cases.items():
        assert oracle.f16_to_f64(bits) == v
    # every finite pattern agrees with numpy's float16
    pats = np.arange(0x10000, dtype=np.uint32).astype(np.uint16)
    ref = npref.f16_bits_to_f64(pats)
    fin = np.isfinite(ref)
    got = np.array([oracle.f16_to_f64(int(p)) for p in pats[fin][::7]])
    assert np.array_equal(got, ref[fin][::7])


def test_f16_rounding_matches_numpy():
    rng = np.random.default_rng(5)
    v = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.integers(-8, 5, 3000),
                        [65519.99, 65520.0, 2.0 ** -25, 3 * 2.0 ** -26, 1 + 2.0 ** -11]])
    ref = v.astype(np.float16).view(np.uint16)  # numpy rounds double -> half directly, RNE
    got = np.array([oracle.f64_to_f16(x) for x in v], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_rounding_worked_and_brute_force():
    # halfway cases round to even
    assert oracle.f64_to_bf16(1.0 + 2.0 ** -8) == 0x3F80
    assert oracle.f64_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82
    assert oracle.f64_to_bf16(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81  # no float detour
    assert oracle.f64_to_bf16(-2.0) == 0xC000
    rng = np.random.default_rng(7)
    v = rng.standard_normal(400) * 10.0 ** rng.integers(-6, 6, 400)
    got = np.array([oracle.f64_to_bf16(x) for x in v], dtype=np.uint16)
    assert np.array_equal(got, npref.round_bf16_rne(v))


@pytest.mark.parametrize("bits", [1, 2, 3])
def test_code_extraction_matches_bit_serial_reader(bits):
    rng = np.random.default_rng(bits)
    rows, cols = 8, 128
    codes = rng.integers(0, 256, rows * cols * bits // 8, dtype=np.uint8)
    ref = npref.unpack_codes(codes, bits, rows, cols)
    for r in range(rows):
        for b in range(cols // 32):
            blk = codes[(r * (cols // 32) + b) * 4 * bits:][:4 * bits]
            got = [oracle.code(blk, bits, j) for j in range(32)]
            assert got == list(ref[r, b * 32:(b + 1) * 32])


@pytest.mark.parametrize("bits", [1, 2, 3])
def test_dequant_matrix_matches_numpy_decoder(bits):
    shape = gen.LayerShape(hidden=256, n_experts=2, top_k=1, inter=64, bits=bits)
    w = gen.layer_weights(shape, seed=11)
    ce, se = oracle.expert_slices(shape, w.codes, w.scales, 1)
    for m, (rows, cols) in enumerate([(64, 256), (64, 256), (256, 64)]):
        cm, sm = oracle.mat_slices(shape, ce, se, m)
        ref = npref.dequant(cm, sm, bits, rows, cols)
        got = oracle.dequant_rows(cm, sm, bits, cols, 0, rows)
        assert np.array_equal(got, ref)


@pytest.mark.parametrize("bits", [2, 3])
def test_dequant_is_exact_in_fp32(bits):
    """d*(q-c) needs <= 11+3 significant bits, so fp32 holds every weight exactly:
    any correct fp32 implementation reproduces the oracle's value bit for bit."""
    d = np.arange(0x10000, dtype=np.uint32).astype(np.uint16).view(np.float16)
    d = d[np.isfinite(d)]
    c = (2 ** bits - 1) / 2.0
    for q in range(2 ** bits):
        w32 = d.astype(np.float32) * np.float32(q - c)
        w64 = d.astype(np.float64) * (q - c)
        assert np.array_equal(w32.astype(np.float64), w64)
