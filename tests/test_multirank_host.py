"""Multi-rank host logic of the benchmark on CPU ranks (gloo, world sizes 2
and 3).

With N GPUs the one message is split by group columns (rank k takes columns
[floor(kG/N), floor((k+1)G/N))) and each rank runs the call on its window, or
(``--split messages``) every rank runs its own message; either way there is
no collective on the data path, and the only cross-rank steps are the
barrier and the max-over-ranks of the timed region. The reference arm runs on
rank 0 only. Here the windows are checked to tile [0, G) for awkward G, and
the oracle run window by window on the ranks (standing in for each GPU's
call) gives, gathered, exactly the whole-message call.
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


def _window_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import numpy as np
    import oracle as O
    from bit_error_compensated_group_b200.echo import column_window
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        # 1. the windows of every rank, gathered, tile [0, G) in rank order
        tilings = {}
        for G in (1, 2, 3, 7, 64, 1000, 4194304, 4194303):
            mine = column_window(rank, world, G)
            allw = [None] * world
            dist.all_gather_object(allw, mine)
            tilings[G] = allw
        # 2. one message, P = 3 ranks of the all-reduce, 1000 elements in groups
        #    of 32 (G = 32, partial last group): this rank's window through the
        #    oracle with its own EMA rows, two calls in a row
        P, n, group = 3, 1000, 32
        G = -(-n // group)
        rng = np.random.default_rng(5)
        x = (rng.standard_normal((P, G * group)) * 2).astype(np.float32)
        xb = (x.view(np.uint32) >> 16).astype(np.uint16)         # truncate to bf16 bit patterns
        xb[:, n:] = 0
        c0, c1 = column_window(rank, world, G)
        ys = []
        el = np.zeros((P, (c1 - c0) * group), np.float32)
        es = np.zeros_like(el)
        for _ in range(2):
            if c1 > c0:
                res = O.echo_allreduce(np.ascontiguousarray(xb[:, c0 * group:c1 * group]), n_total=n, group=group,
                                       bits=4, e_long=el, e_short=es, j0=c0, jc=c1 - c0)
                ys.append((c0, c1, res.y.copy(), el.copy(), es.copy()))
            else:
                ys.append((c0, c1, None, None, None))
        gathered = [None] * world
        dist.all_gather_object(gathered, ys)
        dist.barrier()
        q.put((rank, tilings, gathered if rank == 0 else None))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_column_split_tiles_the_message_and_matches_the_whole_call(world):
    import numpy as np
    import oracle as O
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_window_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    got = sorted((q.get(timeout=5) for _ in range(world)), key=lambda t: t[0])
    for rank, tilings, _ in got:
        for G, wins in tilings.items():
            assert wins[0][0] == 0 and wins[-1][1] == G, (G, wins)
            for a, b in zip(wins, wins[1:]):
                assert a[1] == b[0], (G, wins)                 # contiguous, no overlap, no gap
            assert all(c1 >= c0 for c0, c1 in wins)
            if G >= world:                                    # none empty once there is a column per rank
                assert all(c1 > c0 for c0, c1 in wins)
    gathered = got[0][2]
    P, n, group = 3, 1000, 32
    G = -(-n // group)
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((P, G * group)) * 2).astype(np.float32)
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    xb[:, n:] = 0
    el = np.zeros((P, G * group), np.float32)
    es = np.zeros_like(el)
    for call in range(2):
        full = O.echo_allreduce(xb, n_total=n, group=group, bits=4, e_long=el, e_short=es)
        for per_rank in gathered:
            c0, c1, y, gl, gs = per_rank[call]
            if y is None:
                continue
            sl = slice(c0 * group, c1 * group)
            assert np.array_equal(y, full.y[:, sl]), (call, c0, c1)
            assert np.array_equal(gl, el[:, sl]) and np.array_equal(gs, es[:, sl]), (call, c0, c1)
