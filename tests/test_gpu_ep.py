"""Expert parallelism's GPU steps on one device (needs a B200).

This run has one GPU, so the ranks are emulated in one process: each rank's
routing, plan, expert rows and combine run through the C ABI on the device,
and the all-to-alls are replaced by host-side copies in the order
torch.distributed's all_to_all_single delivers (by source rank).  Each
emulated rank's output must be the same bits as the one-GPU forward of its
tokens on the same kernels: the decode GEMV chain at T = 4 (path 1; the
fused decode kernel sums its K partials in another order, so it agrees with
these only within the layer tolerance) and the tensor-core prefill at
T = 300.  The
multi-process exchange itself is covered by tests/test_ep_gloo.py.
"""
import numpy as np
import pytest

import gen
from tests.gpu_util import from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import quantized_expert_ffn_04_b200 as qe  # noqa: E402
from quantized_expert_ffn_04_b200.ep import GpuBackend  # noqa: E402


def emulated_ep(L, xs, n_ranks, prefill):
    be = GpuBackend(L)
    s = L.shape
    E, k, H = s.n_experts, s.top_k, s.hidden
    plans = []
    for x in xs:
        idx, w = be.route(x)
        idx_h = idx.cpu().numpy()
        counts, pick, slot = qe.strata_ep_plan(idx_h, E, n_ranks)
        tok = torch.from_numpy((pick // k).astype(np.int32)).cuda()
        rows = be.gather_rows(x, tok)
        ids = torch.from_numpy(idx_h.reshape(-1)[pick].astype(np.int32)).cuda()
        offs = np.concatenate([[0], np.cumsum(counts)])
        plans.append(dict(idx=idx, w=w, slot=slot, rows=rows, ids=ids, offs=offs, T=x.shape[0]))
    yd = be.y_dtype(prefill)
    backs = [torch.empty((p["T"] * k, H), dtype=yd, device="cuda") for p in plans]
    shared = []
    for d in range(n_ranks):
        T = xs[d].shape[0]
        parts = [(src, p["offs"][d], p["offs"][d + 1]) for src, p in enumerate(plans)]
        recv_rows = torch.cat([plans[src]["rows"][a:b] for src, a, b in parts])
        recv_ids = torch.cat([plans[src]["ids"][a:b] for src, a, b in parts])
        lo, hi = qe.strata_ep_expert_range(d, n_ranks, E)
        assert bool(((recv_ids >= lo) & (recv_ids < hi)).all())
        rows = torch.cat([xs[d], recv_rows])
        ids = torch.cat([torch.full((T,), -1, dtype=torch.int32, device="cuda"), recv_ids])
        y_rows = torch.empty((rows.shape[0], H), dtype=yd, device="cuda")
        ysh = torch.empty((T, H), dtype=yd, device="cuda")
        be.expert_rows(rows, ids, T, prefill, y_rows, ysh)
        shared.append(ysh)
        pos = T
        for src, a, b in parts:  # outputs back to their sources, in plan order
            backs[src][a:b] = y_rows[pos:pos + (b - a)]
            pos += b - a
    outs = []
    for r, p in enumerate(plans):
        Y = torch.cat([backs[r], shared[r]])
        slot = torch.from_numpy(p["slot"]).cuda()
        outs.append(be.combine(xs[r], p["idx"], p["w"], slot, Y, prefill))
    torch.cuda.synchronize()
    L.sync_status()
    return outs


@pytest.mark.parametrize("T,n_ranks", [(4, 2), (4, 3), (300, 2)], ids=["t4-n2", "t4-n3", "t300-n2"])
def test_emulated_expert_parallel_equals_one_gpu(T, n_ranks):
    shape = gen.FLASH2
    layer = gen.layer_weights(shape, seed=0)
    prefill = T > 64
    L = qe.Layer(layer, max_tokens=T + n_ranks * T * shape.top_k)
    xs = [to_dev_bf16(gen.hidden(T, shape.hidden, seed=60 + r)) for r in range(n_ranks)]
    outs = emulated_ep(L, xs, n_ranks, prefill)
    if not prefill:
        L.set_option(qe.STRATA_OPT_PATH, 1)  # the decode GEMV chain
    for r in range(n_ranks):
        ref = from_dev_bf16(L.forward(xs[r]))
        L.sync_status()
        assert np.array_equal(from_dev_bf16(outs[r]), ref), f"rank {r}: differs from one GPU"
    L.close()
