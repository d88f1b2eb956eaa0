"""The exchanges of a multi-GPU call on CPU ranks (gloo): the all-to-all and
all-gather that EchoRank.allreduce runs between its kernels, over the
workspace views and split sizes of ExchangePlan (the library's rank
layout). Every byte a rank sends is tagged with (sender, group, byte), so
the test checks that each owner receives exactly the payload of its segment
from every rank, in rank order, and every rank every owner's requantized
segment. No kernel runs here; the kernels' side of the same layout is
checked against the oracle on the GPU (tests/test_gpu_ranks.py).

The chunked call's exchanges (exchange_chunk: point-to-point pieces of every
owner's part of a chunk, in the order the chunked schedule issues them) must
deliver the same bytes, chunk after chunk, as the whole exchanges."""
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


def _tag_codes(r, j, cb):
    """Codes byte b of group j sent by rank r."""
    return (torch.arange(cb, dtype=torch.int64) * 7 + 31 * j + 101 * r) % 251


def _tag_param(r, j):
    return 1_000_000 * (r + 1) + j


def _worker(rank, world, port, n, group, bits, chunks, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bit_error_compensated_group_b200 as E
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        P = world
        L = E.echo_query_rank_layout(n, P, rank, group, 8, bits)
        ws = torch.zeros(int(L.workspace_bytes), dtype=torch.uint8)
        plan = E.ExchangePlan(ws, n, P, rank, group, 8, bits)
        G, cb = int(L.groups), int(L.code_bytes)
        lay = [E.echo_query_rank_layout(n, P, s, group, 8, bits) for s in range(P)]
        # this rank's send row: every group j
        for j in range(G):
            plan.send_codes[j * cb:(j + 1) * cb] = _tag_codes(rank, j, cb).to(torch.uint8)
            plan.send_params[j] = _tag_param(rank, j)
        seg, b0, sm = int(L.seg_groups), int(L.seg_begin), int(L.seg_max)
        for k in range(seg):
            plan.gsend_codes[k * cb:(k + 1) * cb] = _tag_codes(rank, b0 + k, cb).to(torch.uint8) ^ 0x55
            plan.gsend_params[k] = -_tag_param(rank, b0 + k)
        if chunks == 1:
            E.exchange_all_to_all(plan)
            E.exchange_all_gather(plan)
        else:
            # the order of the chunked schedule: all-to-all of chunk t, then
            # all-gather of chunk t - 1
            for t in range(chunks + 1):
                if t < chunks:
                    for req in E.exchange_chunk(plan, "all_to_all", t, chunks, rank):
                        req.wait()
                if t >= 1:
                    for req in E.exchange_chunk(plan, "all_gather", t - 1, chunks, rank):
                        req.wait()
        bad = []
        for r in range(P):
            if chunks > 1 and r == rank:
                continue          # the chunked exchange does not send an owner its own row (never read)
            for k in range(seg):
                j = b0 + k
                got = plan.recv_codes[(r * seg + k) * cb:(r * seg + k + 1) * cb].to(torch.int64)
                if not torch.equal(got, _tag_codes(r, j, cb)):
                    bad.append(("a2a codes", r, j))
                if int(plan.recv_params[r * seg + k]) != _tag_param(r, j):
                    bad.append(("a2a params", r, j))
        for s in range(P):
            sb, ss = int(lay[s].seg_begin), int(lay[s].seg_groups)
            for k in range(ss):
                got = plan.grecv_codes[(s * sm + k) * cb:(s * sm + k + 1) * cb].to(torch.int64)
                if not torch.equal(got, _tag_codes(s, sb + k, cb) ^ 0x55):
                    bad.append(("gather codes", s, sb + k))
                if int(plan.grecv_params[s * sm + k]) != -_tag_param(s, sb + k):
                    bad.append(("gather params", s, sb + k))
        q.put((rank, bad[:5], seg))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,n,group,bits,chunks", [
    (3, 1000, 64, 4, 1),        # G = 16: segments of 5, 5 and 6 groups
    (2, 777, 32, 8, 1),         # partial last group
    (4, 3 * 128, 128, 4, 1),    # G = 3 < P: one rank owns nothing
    (2, 777, 32, 8, 3),         # chunked: parts of 8 and 9 groups in thirds
    (3, 1000, 64, 4, 4),        # chunked: more chunks than some parts have groups
    (4, 5000, 32, 4, 5),
    (4, 3 * 128, 128, 4, 2),    # chunked with an empty segment
])
def test_exchange_delivers_each_segment(world, n, group, bits, chunks):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, n, group, bits, chunks, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    assert [g[0] for g in got] == list(range(world))
    for rank, bad, seg in got:
        assert bad == [], (rank, bad)


def _subgroup_worker(rank, world, port, q):
    """Ranks 2 and 3 of 4 form the Echo group; their chunked exchange names
    peers by group rank and must reach the right global ranks."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bit_error_compensated_group_b200 as E
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        sub = dist.new_group([2, 3])
        bad = []
        if rank in (2, 3):
            P, me, n, group, bits, chunks = 2, rank - 2, 777, 32, 4, 3
            L = E.echo_query_rank_layout(n, P, me, group, 4, bits)
            ws = torch.zeros(int(L.workspace_bytes), dtype=torch.uint8)
            plan = E.ExchangePlan(ws, n, P, me, group, 4, bits)
            G, cb = int(L.groups), int(L.code_bytes)
            for j in range(G):
                plan.send_codes[j * cb:(j + 1) * cb] = _tag_codes(me, j, cb).to(torch.uint8)
                plan.send_params[j] = _tag_param(me, j)
            seg, b0 = int(L.seg_groups), int(L.seg_begin)
            for t in range(chunks):
                for req in E.exchange_chunk(plan, "all_to_all", t, chunks, me, sub):
                    req.wait()
            other = 1 - me
            for k in range(seg):
                got = plan.recv_codes[(other * seg + k) * cb:(other * seg + k + 1) * cb].to(torch.int64)
                if not torch.equal(got, _tag_codes(other, b0 + k, cb)):
                    bad.append(("a2a codes", other, b0 + k))
        dist.barrier()
        q.put((rank, bad[:5]))
    finally:
        dist.destroy_process_group()


def test_chunked_exchange_in_a_subgroup():
    world = 4
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_subgroup_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, bad in got:
        assert bad == [], (rank, bad)
