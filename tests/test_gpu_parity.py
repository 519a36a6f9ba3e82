"""GPU-vs-oracle parity through the C ABI (needs a B200).

Bit-exact: routing indices, per-expert offsets and token lists, dequantised
weights.  Tolerance (layer specification): bf16 outputs within
max |err| <= 2e-2 max |ref| and mean relative error <= 5e-3 of the oracle's
fp64 layer output.  Workloads: the tiny layer (H 256, E 16, k 2, I 64, T 8), the
Flash-Next-shaped layer (H 2560, E 512, k 10, I 640; the pages' shape: "Strata
Runs 125B Qwen3.8-Flash-Next on a 12GB Gaming GPU at Up to 94 Tokens/s",
section "What it is") at decode T = 1, 4 (2-bit), T = 64 (3-bit) and prefill
T = 8192 (2-bit, sampled outputs), the pruned 256-expert build of the same
layer ("Strata Runs 125B Qwen3.8-Flash-Next on a 12GB Gaming GPU at Up to 94
Tokens/s", section "The Coder build: half the experts, most of the skill"), plus
ragged and degenerate cases.
"""
import numpy as np
import pytest

import gen
import oracle
from tests import npref
from tests.gpu_util import THREADS, W_RTOL, check_output, from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import quantized_expert_ffn_04_b200 as qe  # noqa: E402

_layers = {}


def layer_of(shape, seed=0, layer=0):
    key = (shape, seed, layer)
    if key not in _layers:
        _layers[key] = gen.layer_weights(shape, seed=seed, layer=layer)
    return _layers[key]


def gpu_layer(shape, T, seed=0, path=0):
    L = qe.Layer(layer_of(shape, seed), max_tokens=max(T, 1))
    if path:
        L.set_option(qe.STRATA_OPT_PATH, path)
    return L


def check_route(L, w, x_bits, T, label):
    s = w.shape
    xt = to_dev_bf16(x_bits)
    idx, wts, off, lst = L.route(xt)
    L.sync_status()
    logits = oracle.router_logits(x_bits, w.router_w, w.router_b, threads=THREADS)
    ridx, rw = oracle.route(logits, s.top_k)
    cnt, roff, rlst, rslot = oracle.dispatch(ridx, s.n_experts)
    gi = idx.cpu().numpy()
    assert np.array_equal(gi, ridx), f"{label}: routing indices differ"
    np.testing.assert_allclose(wts.cpu().numpy(), rw, rtol=W_RTOL, atol=0)
    assert np.array_equal(off.cpu().numpy(), roff), f"{label}: offsets differ"
    assert np.array_equal(lst.cpu().numpy(), rlst), f"{label}: token lists differ"
    return ridx, roff


CASES = [
    ("tiny", gen.TINY, 8),
    ("flash2-T1", gen.FLASH2, 1),
    ("flash2-T4", gen.FLASH2, 4),
    ("flash2-T13", gen.FLASH2, 13),
    ("flash3-T64", gen.FLASH3, 64),
    ("pruned256-T4", gen.PRUNED256, 4),
    ("pruned256-T300", gen.PRUNED256, 300),
    ("tiny1-T8", gen.TINY1, 8),
    ("coder1-T4", gen.CODER1, 4),
    ("coder1-T13", gen.CODER1, 13),
    ("coder1-T300", gen.CODER1, 300),
]


@pytest.mark.parametrize("name,shape,T", CASES, ids=[c[0] for c in CASES])
def test_route_and_forward_parity(name, shape, T):
    w = layer_of(shape)
    x = gen.hidden(T, shape.hidden, seed=1)
    L = gpu_layer(shape, T)
    check_route(L, w, x, T, name)
    y = from_dev_bf16(L.forward(to_dev_bf16(x)))
    L.sync_status()
    _, ref, _, _ = oracle.moe_forward(w, x, threads=THREADS)
    check_output(y, ref, name)


@pytest.mark.parametrize("shape", [gen.TINY, gen.FLASH2, gen.FLASH3, gen.CODER1],
                         ids=["tiny", "f2", "f3", "c1"])
def test_dequant_bit_exact(shape):
    w = layer_of(shape)
    L = gpu_layer(shape, 1)
    E = shape.n_experts
    for e in (0, E // 2, E - 1, -1):
        if e >= 0:
            ce, se = oracle.expert_slices(shape, w.codes, w.scales, e)
        else:
            ce, se = w.shared_codes, w.shared_scales
        for m in range(3):
            rows, cols = (shape.inter, shape.hidden) if m < 2 else (shape.hidden, shape.inter)
            cm, sm = oracle.mat_slices(shape, ce, se, m)
            r0, nr = (rows // 2 - 8, 24) if rows > 48 else (0, rows)
            exact = oracle.dequant_rows(cm, sm, shape.bits, cols, r0, nr)
            got = L.debug_dequant(e, m, r0, nr, kind=0)
            assert np.array_equal(got.astype(np.float64), exact), (e, m)
            got16 = L.debug_dequant(e, m, r0, nr, kind=1)
            assert np.array_equal(got16, exact.astype(np.float16).astype(np.float32)), (e, m)


def test_prefill_route_exact_and_sampled_outputs():
    shape, T = gen.FLASH2, 8192
    w = layer_of(shape)
    x = gen.hidden(T, shape.hidden, seed=2)
    L = gpu_layer(shape, T)
    ridx, roff = check_route(L, w, x, T, "prefill")
    y = from_dev_bf16(L.forward(to_dev_bf16(x)))
    L.sync_status()
    cnt = np.diff(roff)
    hot, cold = int(np.argmax(cnt)), int(np.argmin(np.where(cnt > 0, cnt, 1 << 30)))
    rng = np.random.default_rng(0)
    sel = set(rng.choice(T, 16, replace=False).tolist()) | {0, T - 1}
    sel |= set(np.nonzero((ridx == cold).any(axis=1))[0][:4].tolist())
    sel |= set(np.nonzero((ridx == hot).any(axis=1))[0][:4].tolist())
    sel = np.array(sorted(sel), dtype=np.int32)
    _, ref, _, _ = oracle.moe_forward(w, x, sel=sel, threads=THREADS)
    check_output(y[sel], ref, "prefill sampled")
    assert np.all(np.isfinite(npref.bf16_bits_to_f64(y)))


PATH_CASES = [
    ("f2-T200-gemv", gen.FLASH2, 200, 1, 7),
    ("f2-T200-gemm", gen.FLASH2, 200, 2, 7),
    ("tiny-T8-gemm", gen.TINY, 8, 2, 1),
    ("tiny-T300-gemm", gen.TINY, 300, 2, 1),
    ("f2-T65-auto", gen.FLASH2, 65, 0, 4),
    ("f3-T160-gemm", gen.FLASH3, 160, 2, 9),
    ("f3-T64-gemm", gen.FLASH3, 64, 2, 5),
    ("c1-T20-gemv", gen.CODER1, 20, 1, 3),
    ("c1-T200-gemm", gen.CODER1, 200, 2, 7),
]


@pytest.mark.parametrize("name,shape,T,path,stride", PATH_CASES, ids=[c[0] for c in PATH_CASES])
def test_paths_agree_with_oracle(name, shape, T, path, stride):
    """Decode (1) and tensor-core (2) paths at sizes spanning several tiles with a
    ragged last tile; every `stride`-th token is checked against the oracle."""
    w = layer_of(shape)
    x = gen.hidden(T, shape.hidden, seed=3)
    L = gpu_layer(shape, T, path=path)
    y = from_dev_bf16(L.forward(to_dev_bf16(x)))
    L.sync_status()
    sel = np.arange(0, T, stride, dtype=np.int32)
    _, ref, _, _ = oracle.moe_forward(w, x, sel=sel, threads=THREADS)
    check_output(y[sel], ref, name)


def test_paths_agree_with_each_other():
    """Both paths on the same input: within tolerance of each other, and the
    routing (shared by both) is identical."""
    shape, T = gen.FLASH2, 96
    x = to_dev_bf16(gen.hidden(T, shape.hidden, seed=12))
    y1 = from_dev_bf16(gpu_layer(shape, T, path=1).forward(x))
    y2 = from_dev_bf16(gpu_layer(shape, T, path=2).forward(x))
    check_output(y2, npref.bf16_bits_to_f64(y1), "gemm vs gemv")


def test_deterministic_across_calls_and_streams():
    shape, T = gen.FLASH2, 4
    L = gpu_layer(shape, T)
    xt = to_dev_bf16(gen.hidden(T, shape.hidden, seed=4))
    y1 = from_dev_bf16(L.forward(xt))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y2 = L.forward(xt, stream=s)
    s.synchronize()
    y3 = from_dev_bf16(L.forward(xt))
    assert np.array_equal(y1, from_dev_bf16(y2)) and np.array_equal(y1, y3)


def test_forward_host_matches_device():
    shape, T = gen.FLASH2, 4
    L = gpu_layer(shape, T)
    x = gen.hidden(T, shape.hidden, seed=5)
    yd = from_dev_bf16(L.forward(to_dev_bf16(x)))
    yh = np.empty_like(x)
    qe.strata_moe_forward_host(L.handle, x.ctypes.data, T, yh.ctypes.data, None)
    assert np.array_equal(yd, yh)


def test_forward_host_pinned():
    # pinned (page-locked) host buffers, as a serving loop holds them: new
    # contents in the same buffers, other buffers, another T and a path
    # change all give the device forward's bits
    shape = gen.FLASH2
    L = gpu_layer(shape, 8)
    s = torch.cuda.Stream()

    def pinned(a):
        return torch.from_numpy(a.view(np.int16).copy()).pin_memory()

    xa, xb = pinned(gen.hidden(8, shape.hidden, seed=7)), pinned(gen.hidden(8, shape.hidden, seed=8))
    ya, yb = torch.empty_like(xa).pin_memory(), torch.empty_like(xb).pin_memory()

    def device_ref(xp, T):
        xd = to_dev_bf16(xp.numpy().view(np.uint16)[:T])
        return from_dev_bf16(L.forward(xd))

    def host(xp, yp, T):
        qe.strata_moe_forward_host(L.handle, xp.data_ptr(), T, yp.data_ptr(), s.cuda_stream)
        return yp.numpy().view(np.uint16)[:T].copy()

    for T in (4, 1):
        for xp, yp in ((xa, ya), (xb, yb)):
            first = host(xp, yp, T)
            again = host(xp, yp, T)
            assert np.array_equal(first, device_ref(xp, T)) and np.array_equal(again, first)
    host(xa, ya, 4)
    xa.copy_(pinned(gen.hidden(8, shape.hidden, seed=9)))
    assert np.array_equal(host(xa, ya, 4), device_ref(xa, 4))
    qe.strata_moe_set_option(L.handle, qe.STRATA_OPT_PATH, 1)  # the decode kernel chain
    y_chain = host(xa, ya, 4)
    assert np.array_equal(y_chain, device_ref(xa, 4))
    qe.strata_moe_set_option(L.handle, qe.STRATA_OPT_PATH, 0)  # back to the fused kernel
    y_fused = host(xa, ya, 4)
    assert np.array_equal(y_fused, device_ref(xa, 4))
    close_outputs(y_fused, y_chain, "host forward, fused vs chain")


def test_zero_and_oversized_batches():
    shape = gen.TINY
    L = gpu_layer(shape, 8)
    xt = to_dev_bf16(gen.hidden(8, shape.hidden, seed=6))
    y = torch.zeros_like(xt)
    qe.strata_moe_forward(L.handle, xt.data_ptr(), 0, y.data_ptr(), None)  # no-op
    assert int((y.view(torch.int16) != 0).sum()) == 0
    with pytest.raises(qe.StrataError) as ei:
        qe.strata_moe_forward(L.handle, xt.data_ptr(), 9, y.data_ptr(), None)
    assert ei.value.status == qe.STRATA_ERR_INVALID_ARG
    with pytest.raises(qe.StrataError) as ei:
        qe.strata_moe_forward(L.handle, xt.data_ptr(), 8, xt.data_ptr() + 64, None)  # overlap
    assert ei.value.status == qe.STRATA_ERR_INVALID_ARG


def test_bounded_waits_report_timeout_and_recover():
    with pytest.raises(qe.StrataError) as ei:
        qe.strata_moe_selftest_wait(0, 200000)
    assert ei.value.status == qe.STRATA_ERR_TIMEOUT
    shape, T = gen.TINY, 8
    L = gpu_layer(shape, T)
    xt = to_dev_bf16(gen.hidden(T, shape.hidden, seed=7))
    L.set_option(qe.STRATA_OPT_WAIT_BUDGET, 0)
    L.forward(xt)
    with pytest.raises(qe.StrataError) as ei:
        L.sync_status()
    assert ei.value.status == qe.STRATA_ERR_TIMEOUT
    L.set_option(qe.STRATA_OPT_WAIT_BUDGET, 4_000_000_000)
    y = from_dev_bf16(L.forward(xt))
    L.sync_status()
    _, ref, _, _ = oracle.moe_forward(layer_of(shape), gen.hidden(T, shape.hidden, seed=7))
    check_output(y, ref, "after timeout")


def test_rmsnorm_bit_exact():
    x = gen.hidden(37, 2560, seed=8)
    xt = to_dev_bf16(x)
    out = torch.empty_like(xt)
    qe.strata_moe_rmsnorm(xt.data_ptr(), out.data_ptr(), 37, 2560, None)
    torch.cuda.synchronize()
    assert np.array_equal(from_dev_bf16(out), oracle.rmsnorm(x))


def _route_case(layer, T, seed, label):
    L = qe.Layer(layer, max_tokens=T)
    x = gen.hidden(T, layer.shape.hidden, seed=seed)
    check_route(L, layer, x, T, label)


@pytest.mark.parametrize("T", [300, 1000], ids=["T300", "T1000"])
def test_screened_router_ties_and_near_ties(T):
    """Above 256 tokens the router screens on the tensor cores and recomputes
    candidates exactly; picks must still be the oracle's bit for bit when logits
    tie exactly (duplicated router rows, lower id first), when every logit ties
    (zero router: all experts are candidates) and when rows differ by one ulp."""
    import copy
    shape = gen.LayerShape(hidden=256, n_experts=512, top_k=10, inter=64, bits=2,
                           router_bias=True)
    base = gen.layer_weights(shape, seed=31)
    dup = copy.copy(base)
    W = base.router_w.copy()
    W[1::2] = W[0::2]
    b = base.router_b.copy()
    b[1::2] = b[0::2]
    dup.router_w, dup.router_b = W, b
    _route_case(dup, T, 5, "duplicated rows")
    near = copy.copy(base)
    W2 = base.router_w.copy()
    W2[1::2] = np.nextafter(W2[0::2], np.float32(np.inf))
    near.router_w, near.router_b = W2, b
    _route_case(near, T, 6, "one-ulp rows")
    zero = copy.copy(base)
    zero.router_w = np.zeros_like(base.router_w)
    zero.router_b = np.zeros_like(base.router_b)
    _route_case(zero, T, 7, "zero router")


def _tie_layers(shape, seed):
    """The layer plus three router variants: duplicated rows (exact ties, the
    lower id wins), rows one ulp apart, and an all-zero router (every logit
    ties)."""
    import copy
    base = gen.layer_weights(shape, seed=seed)
    out = [("base", base)]
    dup = copy.copy(base)
    W = base.router_w.copy()
    W[1::2] = W[0::2]
    b = base.router_b.copy() if base.router_b is not None else None
    if b is not None:
        b[1::2] = b[0::2]
    dup.router_w, dup.router_b = W, b
    out.append(("duplicated rows", dup))
    near = copy.copy(base)
    W2 = base.router_w.copy()
    W2[1::2] = np.nextafter(W2[0::2], np.float32(np.inf))
    near.router_w, near.router_b = W2, b
    out.append(("one-ulp rows", near))
    zero = copy.copy(base)
    zero.router_w = np.zeros_like(base.router_w)
    zero.router_b = None if base.router_b is None else np.zeros_like(base.router_b)
    out.append(("zero router", zero))
    return out


def close_outputs(a_bits, b_bits, label):
    """Two bf16 layer outputs of the same input that differ only by rounding:
    every element within 2^-8 of the largest magnitude (about one bf16 unit in
    the last place of the largest element) and the mean difference within
    1e-3 of the mean magnitude."""
    a, b = npref.bf16_bits_to_f64(a_bits), npref.bf16_bits_to_f64(b_bits)
    err = np.abs(a - b)
    assert err.max() <= 2.0 ** -8 * np.abs(b).max(), f"{label}: max diff {err.max():.3e}"
    assert err.sum() <= 1e-3 * np.abs(b).sum(), f"{label}: mean diff {err.sum() / np.abs(b).sum():.3e}"


@pytest.mark.parametrize("T", [1, 4, 13, 64])
def test_fused_decode_agrees_with_gemv_chain(T):
    """The fused decode kernel (router, top-k, dispatch, gate/up, down and
    combine in one launch) against the chain of decode kernels on exact ties,
    one-ulp near-ties and an all-zero router: the same routing (both equal to
    the oracle's, bit for bit), both outputs within the layer tolerance of the
    oracle, and the two outputs equal up to rounding (the fused kernel's
    gate/up products use the magic-offset form and sum its K splits in its own
    fixed order, so the fp32 values may round to neighbouring bf16 values)."""
    shape = gen.LayerShape(hidden=512, n_experts=512, top_k=10, inter=128, bits=2,
                           router_bias=True)
    for label, w in _tie_layers(shape, seed=41):
        x = gen.hidden(T, shape.hidden, seed=42)
        xt = to_dev_bf16(x)
        fused = qe.Layer(w, max_tokens=T)
        fused.set_option(qe.STRATA_OPT_PATH, 3)
        chain = qe.Layer(w, max_tokens=T)
        chain.set_option(qe.STRATA_OPT_PATH, 1)
        assert qe.strata_moe_launch_count(fused.handle, T) == 1
        yf = from_dev_bf16(fused.forward(xt))
        yc = from_dev_bf16(chain.forward(xt))
        fused.sync_status()
        chain.sync_status()
        check_route(fused, w, x, T, f"fused T={T} {label}")
        _, ref, _, _ = oracle.moe_forward(w, x, threads=THREADS)
        check_output(yf, ref, f"fused T={T} {label}")
        check_output(yc, ref, f"chain T={T} {label}")
        close_outputs(yf, yc, f"fused vs chain T={T} {label}")


def test_fused_decode_3bit_batch():
    """3-bit weights at the batched-decode size: fused against the chain and
    the oracle."""
    shape, T = gen.FLASH3, 64
    xh = gen.hidden(T, shape.hidden, seed=43)
    x = to_dev_bf16(xh)
    fused = gpu_layer(shape, T, path=3)
    chain = gpu_layer(shape, T, path=1)
    yf = from_dev_bf16(fused.forward(x))
    yc = from_dev_bf16(chain.forward(x))
    fused.sync_status()
    chain.sync_status()
    close_outputs(yf, yc, "fused vs chain 3-bit T=64")
    sel = np.arange(0, T, 3, dtype=np.int32)
    _, ref, _, _ = oracle.moe_forward(layer_of(shape), xh, sel=sel, threads=THREADS)
    check_output(yf[sel], ref, "fused 3-bit T=64")


@pytest.mark.parametrize("shape", [gen.FLASH2, gen.FLASH3, gen.CODER1], ids=["2bit", "3bit", "1bit"])
def test_prefill_full_tiles(shape):
    """T = 8192 at full tile sizes: the oracle checks the tokens of the hottest
    expert's ragged last tile, the tokens on each side of every interior tile
    boundary of that expert (positions 256 u - 2 .. 256 u + 1 in its token
    list), every token of two mid-load experts, and the shared expert's tile
    boundaries (tokens 256 u - 1, 256 u)."""
    T, tile = 8192, 256
    w = layer_of(shape)
    x = gen.hidden(T, shape.hidden, seed=12)
    L = gpu_layer(shape, T)
    ridx, roff = check_route(L, w, x, T, "prefill full tiles")
    y = from_dev_bf16(L.forward(to_dev_bf16(x)))
    L.sync_status()
    cnt = np.diff(roff)
    hot = int(np.argmax(cnt))
    assert cnt[hot] > tile, "the hottest expert must span several tiles"
    hot_tokens = np.nonzero((ridx == hot).any(axis=1))[0]  # ascending = its list order
    sel = set(hot_tokens[(len(hot_tokens) // tile) * tile:].tolist())  # ragged last tile
    for u in range(1, (len(hot_tokens) + tile - 1) // tile):
        sel |= set(hot_tokens[max(0, u * tile - 2):u * tile + 2].tolist())
    order = np.argsort(cnt, kind="stable")
    nz = order[cnt[order] > 0]
    for e in (nz[len(nz) // 2], nz[len(nz) // 2 + 1]):   # two mid-load experts
        sel |= set(np.nonzero((ridx == e).any(axis=1))[0].tolist())
    for u in range(1, T // tile):
        sel |= {u * tile - 1, u * tile}
    sel = np.array(sorted(sel), dtype=np.int32)
    _, ref, _, _ = oracle.moe_forward(w, x, sel=sel, threads=THREADS)
    check_output(y[sel], ref, f"prefill full tiles ({len(sel)} tokens)")
