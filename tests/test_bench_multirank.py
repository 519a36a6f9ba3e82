"""bench.py's multi-rank host logic on CPU (gloo, world_size 2): the timing is
the max over ranks, the value is every rank's tokens over that time (weak
scaling: one independent replica per GPU, no data-path collective), and the
reference arm works on rank 0 only."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank           # rank 1 is the slow one
        ms = bench.reduce_max(local_ms, dist, "cpu")
        value = bench.weak_scaling_value(1000, world, ms)
        out[rank] = (ms, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_gloo():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    assert res[0][1] == res[1][1] == pytest.approx(2 * 1000 / 0.015)


def test_single_rank_identity():
    assert bench.reduce_max(3.5, None, "cpu") == 3.5
    assert bench.weak_scaling_value(4 * 100, 1, 2.0) == pytest.approx(200000.0)


def test_reference_arm_is_rank0_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), dict(layers=1, warmup=3, steps=1, ref_budget=1.0, gpus=2))()
    bench.run_reference(args, "tiny-t8")       # must return at once, without work
    assert capsys.readouterr().out == ""
