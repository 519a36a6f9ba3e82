"""Pins for the oracle's expert FFN, combine and 48-layer stack pieces.

Layer as specified: SwiGLU experts (g = Wg x, u = Wu x, a = silu(g) u,
y = Wd a), 10 routed + 1 always-on shared expert per token ("Strata Runs 125B
Qwen3.8-Flash-Next on a 12GB Gaming GPU at Up to 94 Tokens/s", section "What it
is"), shared expert added with weight 1, routed experts weighted by the
renormalised top-k softmax, one rounding to bf16.  Stack: h <- h +
MoE(RMSNorm(h)), RMSNorm weight 1, eps 1e-6.
"""
import copy

import numpy as np
import pytest

import gen
import oracle
from tests import npref

TINY = gen.TINY


def _dense_reference(layer, x_bits):
    """Brute force: evaluate every expert densely, weight by a vector that is zero
    off the top-k (softmax from fp64 logits), add the shared expert."""
    s = layer.shape
    xf = npref.bf16_bits_to_f64(x_bits)
    logits = xf @ layer.router_w.astype(np.float64).T
    if layer.router_b is not None:
        logits = logits + layer.router_b
    idx, w = npref.topk_softmax(logits, s.top_k)
    T = xf.shape[0]
    gate = np.zeros((T, s.n_experts))
    for t in range(T):
        gate[t, idx[t]] = w[t]
    y = npref.swiglu(npref.expert_mats(s, layer.shared_codes, layer.shared_scales), xf)
    for e in range(s.n_experts):
        ce, se = oracle.expert_slices(s, layer.codes, layer.scales, e)
        y = y + gate[:, e:e + 1] * npref.swiglu(npref.expert_mats(s, ce, se), xf)
    return y, idx, logits


def _logit_gaps(logits, k):
    srt = -np.sort(-logits, axis=1)
    return srt[:, k - 1] - srt[:, k]


@pytest.mark.parametrize("shape", [TINY, gen.LayerShape(hidden=128, n_experts=6, top_k=3,
                                                        inter=32, bits=3, router_bias=True),
                                   gen.TINY1])
def test_brute_force_dense_masked(shape):
    layer = gen.layer_weights(shape, seed=0)
    x = gen.hidden(8, shape.hidden, seed=0)
    yb, yf, idx, w = oracle.moe_forward(layer, x)
    ref, ridx, logits = _dense_reference(layer, x)
    assert np.min(_logit_gaps(logits, shape.top_k)) > 1e-4  # selection well separated
    assert np.array_equal(np.sort(idx, axis=1), np.sort(ridx, axis=1))
    # fp32 vs fp64 logits move the weights by ~1e-7 relative
    assert np.max(np.abs(yf - ref)) <= 1e-6 * np.max(np.abs(ref))
    assert np.array_equal(yb, npref.round_bf16_rne(yf))


def test_identical_experts_reduce_to_two_dense_swiglus():
    layer = copy.copy(gen.layer_weights(TINY, seed=2))
    s = TINY
    ce, se = oracle.expert_slices(s, layer.codes, layer.scales, 3)
    layer.codes = np.tile(ce, s.n_experts)
    layer.scales = np.tile(se, s.n_experts)
    x = gen.hidden(8, s.hidden, seed=2)
    _, yf, _, _ = oracle.moe_forward(layer, x)
    xf = npref.bf16_bits_to_f64(x)
    ref = (npref.swiglu(npref.expert_mats(s, ce, se), xf)
           + npref.swiglu(npref.expert_mats(s, layer.shared_codes, layer.shared_scales), xf))
    assert np.allclose(yf, ref, rtol=1e-12, atol=1e-13)
    # and with the shared expert equal too, the layer is 2 * SwiGLU(x)
    layer.shared_codes, layer.shared_scales = ce, se
    _, yf2, _, _ = oracle.moe_forward(layer, x)
    assert np.allclose(yf2, 2 * npref.swiglu(npref.expert_mats(s, ce, se), xf), rtol=1e-12,
                       atol=1e-13)


def test_single_expert_top1():
    s = gen.LayerShape(hidden=256, n_experts=1, top_k=1, inter=64, bits=2)
    layer = gen.layer_weights(s, seed=4)
    x = gen.hidden(5, 256, seed=4)
    _, yf, idx, w = oracle.moe_forward(layer, x)
    assert np.all(idx == 0) and np.all(w == 1.0)
    xf = npref.bf16_bits_to_f64(x)
    ref = (npref.swiglu(npref.expert_mats(s, layer.codes, layer.scales), xf)
           + npref.swiglu(npref.expert_mats(s, layer.shared_codes, layer.shared_scales), xf))
    assert np.allclose(yf, ref, rtol=1e-12, atol=1e-13)


def test_constant_codes_closed_form():
    """All 2-bit codes q = 2 (byte 0xAA): every weight is d/2, so
    g_r = u_r = 1/2 sum_b d[r,b] S_b with S_b the sum of x over block b."""
    s = gen.LayerShape(hidden=128, n_experts=1, top_k=1, inter=32, bits=2)
    rng = np.random.default_rng(0)
    codes = np.full(3 * s.mat_code_bytes, 0xAA, dtype=np.uint8)
    scales = gen._scales(3 * s.mat_scales, 8, 0, 5)
    x = np.array([1.0, -0.5, 2.0, 0.25] * 32)
    y = oracle.expert_ffn(codes, scales, 2, 128, 32, x)
    d = npref.f16_bits_to_f64(scales)
    dg = d[:s.mat_scales].reshape(32, 4)
    du = d[s.mat_scales:2 * s.mat_scales].reshape(32, 4)
    dd = d[2 * s.mat_scales:].reshape(128, 1)
    S = x.reshape(4, 32).sum(axis=1)            # block sums of x (each 2.75*8)
    g = 0.5 * dg @ S
    u = 0.5 * du @ S
    a = g / (1 + np.exp(-g)) * u
    ref = 0.5 * dd[:, 0] * a.sum()              # every down weight of row c is d[c]/2
    assert np.allclose(y, ref, rtol=1e-13)
    del rng


def test_token_subset_equals_full_batch():
    layer = gen.layer_weights(TINY, seed=5)
    x = gen.hidden(8, TINY.hidden, seed=5)
    yb, yf, idx, w = oracle.moe_forward(layer, x)
    sel = np.array([6, 1, 3])
    yb2, yf2, idx2, w2 = oracle.moe_forward(layer, x, sel=sel, threads=2)
    assert np.array_equal(yb2, yb[sel]) and np.array_equal(yf2, yf[sel])
    assert np.array_equal(idx2, idx[sel]) and np.array_equal(w2, w[sel])


def test_rmsnorm_constant_rows_and_bound():
    H = 256
    h = np.full((2, H), 0x4000, dtype=np.uint16)  # 2.0
    h[1] = 0xC040                                 # -3.0
    xn = oracle.rmsnorm(h)
    assert np.all(xn[0] == 0x3F80) and np.all(xn[1] == 0xBF80)  # +-1.0 after RNE
    x = gen.hidden(16, 2560, seed=8)
    xf = npref.bf16_bits_to_f64(x)
    r = 1.0 / np.sqrt((xf ** 2).mean(axis=1, keepdims=True) + 1e-6)
    ref = xf * r
    got = npref.bf16_bits_to_f64(oracle.rmsnorm(x))
    # one bf16 rounding of a value within ~1e-6 relative: at most 1 ulp apart
    ulp = 2.0 ** (np.floor(np.log2(np.abs(ref) + 1e-300)) - 7)
    assert np.all(np.abs(got - ref) <= ulp)


def test_rmsnorm_canonical_order():
    # squares: lane 0 holds 4096^2 = 2^24 then 1; lane 1 holds 1, 1 (H = 64)
    h = np.zeros((1, 64), dtype=np.uint16)
    h[0, 0], h[0, 32], h[0, 1], h[0, 33] = 0x4580, 0x3F80, 0x3F80, 0x3F80  # 4096, 1, 1, 1
    xn = oracle.rmsnorm(h)
    ss = np.float32(2.0 ** 24 + 2)  # canonical: p0 = 2^24 (tie), p1 = 2, sum exact
    r = np.float32(1.0) / np.sqrt(ss / np.float32(64) + np.float32(1e-6))
    assert xn[0, 0] == npref.round_bf16_rne(np.float64(np.float32(4096.0) * r))


def test_residual_add_worked():
    h = np.array([[0x3F80, 0x3F80, 0x4000]], dtype=np.uint16)  # 1, 1, 2
    y = np.array([[0x3B80, 0x3C00, 0xBF80]], dtype=np.uint16)  # 2^-8, 2^-7, -1
    out = oracle.residual_add(h, y)
    assert list(out[0]) == [0x3F80, 0x3F81, 0x3F80]  # tie->even, exact, exact


def test_stack_is_composition():
    layers = [gen.layer_weights(TINY, seed=0, layer=l) for l in range(3)]
    h0 = gen.hidden(4, TINY.hidden, seed=0)
    hf, ins = oracle.stack_forward(layers, h0)
    h = h0.copy()
    for l, layer in enumerate(layers):
        assert np.array_equal(ins[l], h)
        yb, _, _, _ = oracle.moe_forward(layer, oracle.rmsnorm(h))
        hb = npref.bf16_bits_to_f64(h) + npref.bf16_bits_to_f64(yb)
        h = npref.round_bf16_rne(hb.astype(np.float32).astype(np.float64))
    assert np.array_equal(hf, h)
