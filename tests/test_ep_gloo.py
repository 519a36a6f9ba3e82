"""Expert parallelism on CPU ranks (gloo, world_size 2 and 3): the exchange
plan, the all-to-alls and the fixed-order combine of
quantized_expert_ffn_04_b200.ep, driven by a float64 numpy backend (oracle
routing, textbook dequantised SwiGLU experts).  Each rank's expert-parallel
output must be the same bits as the same backend's forward of the rank's
tokens without any exchange, and agree with the oracle's layer output."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import gen
import oracle
from tests import npref


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bits(x):
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


class NumpyBackend:
    """The layer's steps in float64 on the host (test-only)."""

    def __init__(self, layer):
        self.w = layer
        s = layer.shape
        self.s = s
        self.mats = {}

    def _expert(self, e):
        if e not in self.mats:
            s, w = self.s, self.w
            if e == s.n_experts:
                self.mats[e] = npref.expert_mats(s, w.shared_codes, w.shared_scales)
            else:
                cb, sb = 3 * s.mat_code_bytes, 3 * s.mat_scales
                self.mats[e] = npref.expert_mats(s, w.codes[e * cb:(e + 1) * cb],
                                                 w.scales[e * sb:(e + 1) * sb])
        return self.mats[e]

    def route(self, x):
        logits = oracle.router_logits(_bits(x), self.w.router_w, self.w.router_b)
        idx, w = oracle.route(logits, self.s.top_k)
        return torch.from_numpy(idx), torch.from_numpy(w)

    def gather_rows(self, src, rows):
        return src.index_select(0, rows.long())

    def y_dtype(self, prefill):
        return torch.float64

    def expert_rows(self, rows, ids, n_shared, prefill, y_out, yshared_out):
        xf = npref.bf16_bits_to_f64(_bits(rows))
        ids = ids.numpy()
        for i in range(rows.shape[0]):
            if ids[i] >= 0:
                y_out[i] = torch.from_numpy(npref.swiglu(self._expert(int(ids[i])), xf[i]))
            if i < n_shared:
                yshared_out[i] = torch.from_numpy(npref.swiglu(self._expert(self.s.n_experts), xf[i]))

    def combine(self, x, idx, w, slot, Y, prefill):
        T, k = idx.shape
        idx, w, slot, Y = idx.numpy(), w.numpy(), slot.numpy(), Y.numpy()
        out = np.empty((T, self.s.hidden))
        for t in range(T):
            acc = Y[T * k + t].copy()
            for j in np.argsort(idx[t], kind="stable"):  # ascending expert id
                acc += w[t, j] * Y[slot[t * k + j]]
            out[t] = acc
        bits = gen.f32_to_bf16_bits(out.astype(np.float32))
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)

    def forward_local(self, x):
        """The same steps on one rank, no exchange: the reference."""
        T, k = x.shape[0], self.s.top_k
        idx, w = self.route(x)
        picks = idx.numpy().reshape(-1)
        Y = torch.empty((T * k + T, self.s.hidden), dtype=torch.float64)
        rows = x.repeat_interleave(k, dim=0)
        self.expert_rows(rows, torch.from_numpy(picks.astype(np.int32)), 0, False, Y[:T * k], None)
        self.expert_rows(x, torch.full((T,), -1, dtype=torch.int32), T, False,
                         torch.empty((T, self.s.hidden), dtype=torch.float64), Y[T * k:])
        slot = torch.arange(T * k, dtype=torch.int32)
        return self.combine(x, idx, w, slot, Y, False)


def _tokens(shape, T, rank):
    x = gen.hidden(T, shape.hidden, seed=40 + rank)
    return torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16)


def _worker(rank, world, port, shape_name, T, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    from quantized_expert_ffn_04_b200.ep import ExpertParallel
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        shape = getattr(gen, shape_name)
        layer = gen.layer_weights(shape, seed=0)
        be = NumpyBackend(layer)
        ep = ExpertParallel(be, shape.n_experts, shape.top_k, shape.hidden)
        x = _tokens(shape, T, rank)
        y = ep.forward(x)
        out[rank] = (_bits(y).copy(), (ep.e_begin, ep.e_end))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,shape_name,T", [(2, "TINY", 8), (3, "TINY", 5), (2, "TINY", 70)])
def test_expert_parallel_matches_one_rank(world, shape_name, T):
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, shape_name, T, out), nprocs=world, join=True)
        res = dict(out)
    shape = getattr(gen, shape_name)
    layer = gen.layer_weights(shape, seed=0)
    be = NumpyBackend(layer)
    ranges = [res[r][1] for r in range(world)]
    # the expert ranges tile [0, E) in rank order
    assert ranges[0][0] == 0 and ranges[-1][1] == shape.n_experts
    assert all(ranges[r][1] == ranges[r + 1][0] for r in range(world - 1))
    for r in range(world):
        x = _tokens(shape, T, r)
        ref = _bits(be.forward_local(x))
        assert np.array_equal(res[r][0], ref), f"rank {r}: expert-parallel output differs"
        _, oref, _, _ = oracle.moe_forward(layer, _bits(x))
        y = npref.bf16_bits_to_f64(res[r][0])
        assert np.abs(y - oref).max() <= 2e-2 * np.abs(oref).max()


def test_plan_groups_by_rank_then_expert_then_token():
    import quantized_expert_ffn_04_b200 as qe
    rng = np.random.default_rng(1)
    T, k, E, N = 37, 5, 40, 3
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, pick, slot = qe.strata_ep_plan(idx, E, N)
    flat = idx.reshape(-1)
    owner = (flat * N) // E
    assert counts.tolist() == [int((owner == r).sum()) for r in range(N)]
    # a permutation, slot its inverse
    assert sorted(pick.tolist()) == list(range(T * k))
    assert np.array_equal(slot[pick], np.arange(T * k))
    key = np.stack([owner[pick], flat[pick], pick // k], axis=1)
    assert all(tuple(key[i]) <= tuple(key[i + 1]) for i in range(len(key) - 1))
    for r in range(N):
        b, e = qe.strata_ep_expert_range(r, N, E)
        assert all(((x * N) // E == r) == (b <= x < e) for x in range(E))
