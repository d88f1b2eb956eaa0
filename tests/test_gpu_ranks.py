"""One rank per handle (the multi-GPU call's kernels) against the oracle, on
one GPU.

P EchoRank objects stand for the P GPUs. The two exchanges are emulated
in-process with stream-ordered copies that follow the same ExchangePlan
views and split sizes that torch.distributed receives on real GPUs
(all_to_all_single: chunk `dst` of the sender's input goes to chunk `src` of
the receiver's output; all_gather_into_tensor: rank order). Kernels run one
after another on one stream; none waits on another. Checked bit for bit
against the oracle's whole call: every rank's output, its EMA rows, its
all-to-all send row (non-owned groups) and every owner's requantized
segment, over two calls with carried state.
"""
import numpy as np
import pytest
import torch

import oracle as O
import bit_error_compensated_group_b200 as E
from parity import Params, padded, random_inputs, seeded_state, u16

pytestmark = pytest.mark.gpu


def emulate_all_to_all(plans):
    E.exchange_in_process(plans, "all_to_all")


def emulate_all_gather(plans):
    E.exchange_in_process(plans, "all_gather")


CASES = [
    # P, n, group, bits, feedback, quantizer
    (2, 4096, 128, 4, True, O.Q_DIRECTED),
    (3, 1000, 64, 8, True, O.Q_DIRECTED),
    (8, 8192 * 3 + 77, 128, 4, True, O.Q_DIRECTED),    # partial last group
    (8, 8192 * 3 + 77, 128, 4, False, O.Q_DIRECTED),
    (4, 3 * 128, 128, 4, True, O.Q_DIRECTED),          # G < P: a rank owns nothing
    (1, 5000, 128, 4, True, O.Q_DIRECTED),             # one rank: nothing exchanged
    (5, 148 * 8 * 256 + 37, 256, 8, True, O.Q_DIRECTED),
    (8, 50000, 32, 4, True, O.Q_NEAREST),
    (6, 70001, 64, 4, True, O.Q_INT_ZERO),
    (16, 50000, 128, 4, True, O.Q_DIRECTED),
    (64, 3 * 64 * 128 + 17, 128, 4, True, O.Q_DIRECTED),   # largest P
    # without feedback, P <= 8: the owners' pass stages the received rows in shared memory
    (2, 4096, 128, 4, False, O.Q_DIRECTED),
    (3, 1000, 64, 8, False, O.Q_DIRECTED),
    (8, 50000, 32, 4, False, O.Q_NEAREST),             # 64-group tiles
    (5, 148 * 8 * 256 + 37, 256, 8, False, O.Q_INT_ZERO),
    (16, 50000, 128, 4, False, O.Q_DIRECTED),          # P > 8: the rows are read from global memory
]


@pytest.mark.parametrize("P,n,group,bits,feedback,quantizer", CASES)
def test_ranks_match_the_oracle(P, n, group, bits, feedback, quantizer):
    p = Params(bits=bits, group=group, w=0.3, alpha_long=0.1, alpha_short=0.6, quantizer=quantizer)
    fb = (p.eta, p.alpha_long, p.alpha_short, p.w)
    G = -(-n // group)
    ld = G * group
    ranks = [E.EchoRank(n, P, r, group, max(bits, 4), feedback, quantizer=quantizer) for r in range(P)]
    try:
        x = random_inputs(P, n, 17 * P + n, 2.0)
        xs = [x[r].cuda() for r in range(P)]
        outs = [torch.empty_like(t) for t in xs]
        el = es = None
        if feedback:
            el0, es0 = seeded_state(P, n, n + 5 * P)
            for r in range(P):
                L, S = ranks[r].ema_views()
                L.copy_(torch.from_numpy(el0[r]))
                S.copy_(torch.from_numpy(es0[r]))
            el, es = padded(el0, ld), padded(es0, ld)
        plans = [rk.plan(bits) for rk in ranks]
        xb = padded(u16(x), ld)
        for call in range(2):
            for r in range(P):
                ranks[r].quantize(xs[r], bits, *fb)
            emulate_all_to_all(plans)
            for r in range(P):
                ranks[r].reduce(xs[r], outs[r], bits, *fb)
            emulate_all_gather(plans)
            for r in range(P):
                ranks[r].decode(outs[r], bits)
            orc = O.echo_allreduce(xb, n_total=n, group=group, bits=bits, e_long=el, e_short=es, eta=p.eta,
                                   alpha_long=p.alpha_long, alpha_short=p.alpha_short, w=p.w, quantizer=quantizer)
            flags = 0
            for rk in ranks:
                flags |= rk.status()[1]
            assert flags == orc.flags
            for r in range(P):
                assert np.array_equal(u16(outs[r]), orc.y[r, :n]), f"call {call}: output of rank {r}"
                if feedback:
                    L, S = ranks[r].ema_views()
                    assert np.array_equal(L.cpu().numpy(), el[r, :n]), f"call {call}: e_long of rank {r}"
                    assert np.array_equal(S.cpu().numpy(), es[r, :n]), f"call {call}: e_short of rank {r}"
            cb = group * bits // 8
            for r in range(P):
                pl = plans[r]
                send_c = pl.send_codes.cpu().numpy().reshape(G, cb)
                send_p = pl.send_params.cpu().numpy().view(np.uint16).reshape(G, 2)
                owned = [O.owner(j, G, P) == r for j in range(G)]
                for j in range(G):
                    if not owned[j]:
                        assert np.array_equal(send_c[j], orc.a2a_codes[r, j]), f"a2a codes r={r} j={j}"
                        assert np.array_equal(send_p[j], orc.a2a_params[r, j]), f"a2a params r={r} j={j}"
                if P >= 2:
                    b0, seg = int(pl.layout.seg_begin), int(pl.layout.seg_groups)
                    g_c = pl.gsend_codes.cpu().numpy()[:seg * cb].reshape(seg, cb)
                    g_p = pl.gsend_params.cpu().numpy()[:seg].view(np.uint16).reshape(seg, 2)
                    assert np.array_equal(g_c, orc.gather_codes[b0:b0 + seg]), f"gather codes of owner {r}"
                    assert np.array_equal(g_p, orc.gather_params[b0:b0 + seg]), f"gather params of owner {r}"
            # the next call reduces the result again
            xs = [o.clone() for o in outs]
            xb = padded(orc.y[:, :n].copy(), ld)
    finally:
        for rk in ranks:
            rk.close()


def test_rank_and_simulation_handles_do_not_mix():
    rk = E.EchoRank(4096, 2, 0)
    ar = E.EchoAllReduce(4096, 2)
    try:
        x = torch.zeros(4096, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(E.EchoError) as ei:
            E.echo_allreduce_sim([x, x], [x, x], rk.handle, 4096, 2, 4, 128, 1.0, 0.05, 0.5, 0.5)
        assert ei.value.status == E.ECHO_EINVAL
        with pytest.raises(E.EchoError) as ei:
            E.echo_rank_quantize(x, ar.handle, 4, 1.0, 0.05, 0.5, 0.5)
        assert ei.value.status == E.ECHO_EINVAL
    finally:
        rk.close()
        ar.close()


@pytest.mark.parametrize("bad", [1e6, float("nan")])
@pytest.mark.parametrize("rank", [0, 1])
def test_rank_range_flag(bad, rank):
    """A value outside the fp16 parameter range (or a NaN) on one rank sets
    ECHO_FLAG_RANGE on the handle whose kernel met it -- the non-owner's
    quantize pass or the owner's sum -- and echo_get_status clears it."""
    P, n = 2, 4096
    x = random_inputs(P, n, 10)
    x[rank, 100] = bad            # group 0: owned by rank 0
    ranks = [E.EchoRank(n, P, r, 128, 4, True) for r in range(P)]
    try:
        xs = [x[r].cuda() for r in range(P)]
        outs = [torch.empty_like(t) for t in xs]
        plans = [rk.plan(4) for rk in ranks]
        for r in range(P):
            ranks[r].quantize(xs[r], 4)
        emulate_all_to_all(plans)
        for r in range(P):
            ranks[r].reduce(xs[r], outs[r], 4)
        emulate_all_gather(plans)
        for r in range(P):
            ranks[r].decode(outs[r], 4)
        flags = [rk.status()[1] for rk in ranks]
        assert flags[0] & E.ECHO_FLAG_RANGE          # the owner's sum holds the bad value
        if rank == 1:
            assert flags[1] & E.ECHO_FLAG_RANGE      # and rank 1 quantized it
        assert [rk.status()[1] for rk in ranks] == [0, 0]   # cleared
    finally:
        for rk in ranks:
            rk.close()


CHUNK_CASES = [
    # P, n, group, bits, feedback, chunks
    (2, 4096 * 3 + 5, 128, 4, True, 3),                # partial last group
    (3, 1000, 64, 8, True, 2),
    (8, 8192 * 3 + 77, 128, 4, True, 4),               # partial last group, owner parts of unequal size
    (8, 8192 * 3 + 77, 128, 4, False, 7),
    (8, 50000, 32, 4, True, 16),
    (4, 3 * 128, 128, 4, True, 3),                     # G < P: empty segments and empty parts
    (64, 3 * 64 * 128 + 17, 128, 4, True, 2),          # largest P
    (64, 200 * 128, 128, 4, True, 5),                  # more chunks than some owners have groups
]


@pytest.mark.parametrize("P,n,group,bits,feedback,chunks", CHUNK_CASES)
def test_chunked_ranks_match_the_oracle(P, n, group, bits, feedback, chunks):
    """The chunked schedule (run_chunked): chunk c's exchanges, emulated by
    copies of the chunk's pieces on a second stream, overlap the kernels of
    the neighbouring chunks on the compute stream, ordered by events only.
    Every rank's output and EMA rows match the oracle's whole call bit for
    bit over two calls."""
    p = Params(bits=bits, group=group, w=0.3, alpha_long=0.1, alpha_short=0.6)
    fb = (p.eta, p.alpha_long, p.alpha_short, p.w)
    G = -(-n // group)
    ld = G * group
    ranks = [E.EchoRank(n, P, r, group, max(bits, 4), feedback) for r in range(P)]
    try:
        x = random_inputs(P, n, 29 * P + n, 2.0)
        xs = [x[r].cuda() for r in range(P)]
        outs = [torch.full_like(t, 3.0) for t in xs]
        el = es = None
        if feedback:
            el0, es0 = seeded_state(P, n, n + 7 * P)
            for r in range(P):
                L, S = ranks[r].ema_views()
                L.copy_(torch.from_numpy(el0[r]))
                S.copy_(torch.from_numpy(es0[r]))
            el, es = padded(el0, ld), padded(es0, ld)
        plans = [rk.plan(bits) for rk in ranks]
        comm_stream = torch.cuda.Stream()

        def comm(step, c):
            E.exchange_chunk_in_process(plans, step, c, chunks)

        xb = padded(u16(x), ld)
        for call in range(2):
            E.run_chunked(ranks, xs, outs, bits, fb, chunks, comm, comm_stream)
            orc = O.echo_allreduce(xb, n_total=n, group=group, bits=bits, e_long=el, e_short=es, eta=p.eta,
                                   alpha_long=p.alpha_long, alpha_short=p.alpha_short, w=p.w)
            flags = 0
            for rk in ranks:
                flags |= rk.status()[1]
            assert flags == orc.flags
            for r in range(P):
                assert np.array_equal(u16(outs[r]), orc.y[r, :n]), f"call {call}: output of rank {r}"
                if feedback:
                    L, S = ranks[r].ema_views()
                    assert np.array_equal(L.cpu().numpy(), el[r, :n]), f"call {call}: e_long of rank {r}"
                    assert np.array_equal(S.cpu().numpy(), es[r, :n]), f"call {call}: e_short of rank {r}"
    finally:
        for rk in ranks:
            rk.close()


def test_chunk_arguments_are_checked():
    rk = E.EchoRank(4096, 2, 0)
    try:
        x = torch.zeros(4096, dtype=torch.bfloat16, device="cuda")
        for chunk, chunks in ((0, 0), (2, 2), (-1, 3), (0, E.ECHO_MAX_CHUNKS + 1)):
            with pytest.raises(E.EchoError) as ei:
                rk.quantize_chunk(x, chunk, chunks)
            assert ei.value.status == E.ECHO_EINVAL
            with pytest.raises(E.EchoError) as ei:
                rk.decode_chunk(x, chunk, chunks)
            assert ei.value.status == E.ECHO_EINVAL
    finally:
        rk.close()
