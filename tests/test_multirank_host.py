"""Multi-rank host logic of the benchmark on CPU ranks (gloo, world size 2).

With N GPUs every rank runs its own independent message (weak scaling, no
collective on the data path); the only cross-rank steps are the barrier and
the max-over-ranks of the timed region. The reference arm runs on rank 0 only.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        m = bench.max_over_ranks(local_ms, world, "cpu")
        v = bench.weak_scaling_gbs(world, 8 << 30, m)
        dist.barrier()
        q.put((rank, m, v))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_value():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, m, v in got:
        assert m == 15.0                                  # the slowest rank's time
        assert v == pytest.approx(2 * (8 << 30) / 15e-3 / 1e9)


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), {"steps": 1, "warmup": 0, "gpus": 2})()
    bench.run_reference(args)                              # returns without work or output
    assert capsys.readouterr().out == ""
