"""Expert parallelism over torch.distributed: the experts of one layer split
across ranks, one process per GPU.

Rank r of N owns the experts [ceil(r E / N), ceil((r + 1) E / N)) and keeps
the router and the shared expert.  A forward of the rank's own T tokens:

  1. route its tokens (fp32 router, top-k, lower id on ties);
  2. plan the exchange: every pick (t, j) goes to the owner of its expert,
     grouped by rank, then expert id, then token (strata_ep_plan);
  3. all-to-all of the picked token rows and their expert ids;
  4. the owner runs each received row through its expert, and every rank runs
     its own rows through the shared expert (strata_moe_expert_rows);
  5. all-to-all of the expert outputs back, in the order they came;
  6. the fixed-order combine: shared first, then the picks in ascending
     expert id, fp32, one rounding to bf16 (strata_moe_combine_rows).

Each expert output depends on one token row and one expert only, and the
combine is the one-GPU combine on the same values, so the result is the same
bits as the one-GPU forward of the rank's tokens on the same kernels (the
decode GEMV chain up to 64 tokens, the tensor-core prefill above; the fused
decode kernel sums its K partials in another order and agrees within the
layer tolerance).  The exchange is
torch.distributed's all_to_all_single (NCCL on GPUs, gloo on CPU).

The compute steps go through a backend; GpuBackend calls the library's
kernels through the C ABI.  Any object with the same methods works (the
tests drive the exchange logic on CPU ranks with a numpy backend).
"""
from __future__ import annotations

import numpy as np

from . import (Layer, strata_ep_expert_range, strata_ep_gather_rows, strata_ep_plan,
               strata_moe_combine_rows, strata_moe_expert_rows)

# decode (the GEMV kernels, fp32 expert outputs) up to this many tokens, like
# the one-GPU forward's default; the tensor-core kernels (fp16 outputs) above
DECODE_MAX_T = 64


class GpuBackend:
    """The library's kernels on one CUDA device (torch tensors in and out)."""

    def __init__(self, layer: Layer):
        self.layer = layer
        self.h = layer.handle
        s = layer.shape
        self.H, self.E, self.k = s.hidden, s.n_experts, s.top_k

    def route(self, x):
        idx, w, _, _ = self.layer.route(x)
        return idx, w

    def gather_rows(self, src, rows):
        import torch
        n = rows.numel()
        dst = torch.empty((n,) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
        row_bytes = src[0].numel() * src.element_size() if src.shape[0] else 16
        if n:
            strata_ep_gather_rows(src.data_ptr(), rows.data_ptr(), n, src.shape[0], row_bytes,
                                  dst.data_ptr())
        return dst

    def expert_rows(self, rows, ids, n_shared, prefill, y_out, yshared_out):
        n = rows.shape[0]
        strata_moe_expert_rows(self.h, rows.data_ptr(), ids.data_ptr(), n, n_shared, prefill,
                               y_out.data_ptr(), yshared_out.data_ptr() if n_shared else None)

    def combine(self, x, idx, w, slot, Y, prefill):
        import torch
        out = torch.empty_like(x)
        strata_moe_combine_rows(self.h, x.data_ptr(), x.shape[0], idx.data_ptr(), w.data_ptr(),
                                slot.data_ptr(), Y.data_ptr(), prefill, out.data_ptr())
        return out

    def y_dtype(self, prefill):
        import torch
        return torch.float16 if prefill else torch.float32


def _a2a(out, inp, out_splits, in_splits, group):
    """all_to_all_single that moves bits: 2-byte rows (bf16) travel as fp16,
    which every backend carries (nothing is computed on them)."""
    import torch
    import torch.distributed as dist
    if out.dtype == torch.bfloat16:
        out, inp = out.view(torch.float16), inp.view(torch.float16)
    dist.all_to_all_single(out, inp, out_splits, in_splits, group=group)


class ExpertParallel:
    """One rank of an expert-parallel layer.  `backend` does the compute; the
    process group (default: the world) does the exchange."""

    def __init__(self, backend, n_experts: int, top_k: int, hidden: int, group=None,
                 decode_max_t: int = DECODE_MAX_T):
        import torch.distributed as dist
        self.be = backend
        self.E, self.k, self.H = n_experts, top_k, hidden
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.e_begin, self.e_end = strata_ep_expert_range(self.rank, self.world, n_experts)
        self.decode_max_t = decode_max_t

    def forward(self, x):
        import torch
        import torch.distributed as dist
        T, k, H = x.shape[0], self.k, self.H
        prefill = T > self.decode_max_t
        dev = x.device
        idx, w = self.be.route(x)
        idx_h = idx.cpu().numpy().reshape(T, k)
        counts, pick, slot = strata_ep_plan(idx_h, self.E, self.world)
        send_counts = torch.from_numpy(counts.astype(np.int64))
        recv_counts = torch.empty_like(send_counts)
        if dev.type == "cuda":
            send_counts, recv_counts = send_counts.to(dev), recv_counts.to(dev)
        dist.all_to_all_single(recv_counts, send_counts, group=self.group)
        sc = [int(c) for c in send_counts.cpu()]
        rc = [int(c) for c in recv_counts.cpu()]
        n_recv = sum(rc)
        tok_t = torch.from_numpy((pick // k).astype(np.int32)).to(dev)
        # the picked rows and their expert ids, in plan order
        send_rows = self.be.gather_rows(x, tok_t)
        send_ids = torch.from_numpy(idx_h.reshape(-1)[pick].astype(np.int32)).to(dev)
        # own rows first (the shared expert, no routed pick: id -1), then the
        # rows received for this rank's experts
        rows = torch.empty((T + n_recv, H), dtype=x.dtype, device=dev)
        ids = torch.full((T + n_recv,), -1, dtype=torch.int32, device=dev)
        rows[:T].copy_(x)
        _a2a(rows[T:], send_rows, rc, sc, self.group)
        _a2a(ids[T:], send_ids, rc, sc, self.group)
        yd = self.be.y_dtype(prefill)
        y_rows = torch.empty((T + n_recv, H), dtype=yd, device=dev)
        # combine layout: the picks in plan order, then the shared rows
        Y = torch.empty((T * k + T, H), dtype=yd, device=dev)
        self.be.expert_rows(rows, ids, T, prefill, y_rows, Y[T * k:])
        _a2a(Y[:T * k], y_rows[T:], sc, rc, self.group)
        slot_t = torch.from_numpy(slot).to(dev)
        return self.be.combine(x, idx, w, slot_t, Y, prefill)
