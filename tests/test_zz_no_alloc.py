"""The allocation-free routing entry point (needs a GPU).

strata_moe_route_noalloc serves callers that cannot call cudaMalloc (code
inside another framework's memory pool, on a fixed memory budget, or on a path
that must not synchronise).  It keeps its intermediates in a static device
array, so this test calls it twice in a row through the C ABI and checks both
results against the handle-based strata_moe_route on the same input and against
the CPU oracle's routing: picks, per-expert offsets and token lists bit for bit,
weights within the routing weight tolerance.  Further cases leave out the
optional outputs (offsets and lists then stay in the static array) and run at
the largest sizes the entry point accepts.  It lives in its own file, collected
last, and runs the same alone in a fresh process.
"""
import numpy as np
import pytest

import gen
import oracle
from tests.gpu_util import THREADS, W_RTOL, to_dev_bf16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import quantized_expert_ffn_04_b200 as qe  # noqa: E402


@pytest.mark.parametrize("shape,T", [(gen.FLASH2, 4), (gen.FLASH3, 64), (gen.TINY, 8)],
                         ids=["flash-T4", "flash-T64", "tiny-T8"])
def test_noalloc_route_matches_handle_route_twice(shape, T):
    layer = gen.layer_weights(shape, seed=21)
    L = qe.Layer(layer, max_tokens=T)
    E, k, H = shape.n_experts, shape.top_k, shape.hidden
    W = torch.from_numpy(layer.router_w).cuda()
    b = None if layer.router_b is None else torch.from_numpy(layer.router_b).cuda()
    for call in range(2):
        x = to_dev_bf16(gen.hidden(T, H, seed=30 + call))
        ridx, rw, roff, rlst = L.route(x)
        idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
        w = torch.zeros((T, k), dtype=torch.float32, device="cuda")
        off = torch.full((E + 1,), -1, dtype=torch.int32, device="cuda")
        lst = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
        qe.strata_moe_route_noalloc(x.data_ptr(), T, H, W.data_ptr(),
                                    None if b is None else b.data_ptr(), E, k, idx.data_ptr(),
                                    w.data_ptr(), off.data_ptr(), lst.data_ptr(), None)
        torch.cuda.synchronize()
        assert torch.equal(idx, ridx), f"call {call}: picks differ"
        assert torch.equal(off, roff), f"call {call}: offsets differ"
        assert torch.equal(lst, rlst), f"call {call}: token lists differ"
        np.testing.assert_allclose(w.cpu().numpy(), rw.cpu().numpy(), rtol=W_RTOL, atol=0)
        check_with_oracle(x, layer.router_w, layer.router_b, k, idx, w, off, lst,
                          f"call {call}")


def check_with_oracle(x, W, b, k, idx, w, off, lst, label):
    """The routing of the oracle (fp32 logits in the fixed order, top-k with the
    lower id winning a tie, stable dispatch) on the same bits."""
    xb = x.cpu().view(torch.int16).numpy().view(np.uint16)
    logits = oracle.router_logits(xb, W, b, threads=THREADS)
    oidx, ow = oracle.route(logits, k)
    _, ooff, olst, _ = oracle.dispatch(oidx, W.shape[0])
    assert np.array_equal(idx.cpu().numpy(), oidx), f"{label}: picks differ from the oracle"
    np.testing.assert_allclose(w.cpu().numpy(), ow, rtol=W_RTOL, atol=0)
    if off is not None:
        assert np.array_equal(off.cpu().numpy(), ooff), f"{label}: offsets differ from the oracle"
        assert np.array_equal(lst.cpu().numpy(), olst), f"{label}: lists differ from the oracle"


def test_noalloc_route_without_offsets_and_lists():
    """offsets and lists left out (NULL): they stay in the static array, and the
    picks and weights still match the oracle on two calls in a row."""
    shape, T = gen.FLASH2, 16
    layer = gen.layer_weights(shape, seed=22)
    E, k, H = shape.n_experts, shape.top_k, shape.hidden
    W = torch.from_numpy(layer.router_w).cuda()
    b = torch.from_numpy(layer.router_b).cuda()
    for call in range(2):
        x = to_dev_bf16(gen.hidden(T, H, seed=40 + call))
        idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
        w = torch.zeros((T, k), dtype=torch.float32, device="cuda")
        qe.strata_moe_route_noalloc(x.data_ptr(), T, H, W.data_ptr(), b.data_ptr(), E, k,
                                    idx.data_ptr(), w.data_ptr(), None, None, None)
        torch.cuda.synchronize()
        check_with_oracle(x, layer.router_w, layer.router_b, k, idx, w, None, None,
                          f"call {call}")


def test_noalloc_route_at_its_largest_sizes():
    """T = 64 tokens, E = 1024 experts, k = 32 picks, H = 6144: the sizes the
    static array and the dispatch scan are sized for, against the oracle."""
    shape = gen.LayerShape(hidden=6144, n_experts=1024, top_k=32, inter=32, bits=2,
                           router_bias=True)
    T, E, k, H = 64, shape.n_experts, shape.top_k, shape.hidden
    Wn = gen.router_weight(shape, seed=23)
    bn = gen.router_bias(shape, seed=23)
    W = torch.from_numpy(Wn).cuda()
    b = torch.from_numpy(bn).cuda()
    for call in range(2):
        x = to_dev_bf16(gen.hidden(T, H, seed=50 + call))
        idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
        w = torch.zeros((T, k), dtype=torch.float32, device="cuda")
        off = torch.full((E + 1,), -1, dtype=torch.int32, device="cuda")
        lst = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
        qe.strata_moe_route_noalloc(x.data_ptr(), T, H, W.data_ptr(), b.data_ptr(), E, k,
                                    idx.data_ptr(), w.data_ptr(), off.data_ptr(),
                                    lst.data_ptr(), None)
        torch.cuda.synchronize()
        check_with_oracle(x, Wn, bn, k, idx, w, off, lst, f"call {call}")


def test_noalloc_route_rejects_sizes_beyond_its_limits():
    x = torch.zeros((65, 256), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((16, 256), dtype=torch.float32, device="cuda")
    idx = torch.empty((65, 2), dtype=torch.int32, device="cuda")
    w = torch.empty((65, 2), dtype=torch.float32, device="cuda")
    for T, H, E, k in [(65, 256, 16, 2), (8, 200, 16, 2), (8, 256, 2048, 2), (8, 256, 16, 33)]:
        with pytest.raises(qe.StrataError) as ei:
            qe.strata_moe_route_noalloc(x.data_ptr(), T, H, W.data_ptr(), None, E, k,
                                        idx.data_ptr(), w.data_ptr())
        assert ei.value.status == qe.STRATA_ERR_INVALID_ARG
