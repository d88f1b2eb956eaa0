"""The background-traffic study's two kernels through the C ABI.

* echo_bf16_allreduce_sim, the 16-bit baseline simulated over P virtual
  ranks, against the oracle's bf16_allreduce bit for bit: every rank's
  output, for P = 1 .. 64, lengths that are not a multiple of eight (the
  scalar tail) and in place;
* echo_background_traffic ends by itself after its duration, copies src to
  dst (a full pass at 100 % duty), counts the bytes it moved, moves less at
  lower duty, and launches nothing at 0 %.
"""
import time

import numpy as np
import pytest
import torch

import oracle as O
import bit_error_compensated_group_b200 as E
from parity import random_inputs, u16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("P,n", [(1, 1000), (2, 4096 + 3), (3, 77), (8, 1 << 20), (8, 8 * 148 * 256 * 3 + 5),
                                 (16, 10007), (64, 4099)])
def test_bf16_baseline_matches_the_oracle(P, n):
    x = random_inputs(P, n, 900 + P, 3.0)
    xs = [x[r].cuda() for r in range(P)]
    outs = [torch.full_like(t, 5.0) for t in xs]
    E.echo_bf16_allreduce_sim(xs, outs, n, P)
    want = O.bf16_allreduce(u16(x))
    for r in range(P):
        assert np.array_equal(u16(outs[r]), want[r]), f"rank {r}"
    # in place: outputs are the inputs
    E.echo_bf16_allreduce_sim(xs, xs, n, P)
    for r in range(P):
        assert np.array_equal(u16(xs[r]), want[r]), f"in place, rank {r}"


def test_bf16_baseline_rank_order():
    """The hand-worked sums of the oracle's rank-order pin, on the GPU."""
    v = torch.tensor([[2.0 ** -14, 32768.0], [32768.0, -32768.0], [-32768.0, 2.0 ** -14]]).to(torch.bfloat16)
    xs = [v[r].contiguous().cuda() for r in range(3)]
    outs = [torch.empty_like(t) for t in xs]
    E.echo_bf16_allreduce_sim(xs, outs, 2, 3)
    for o in outs:
        assert u16(o).tolist() == [0, 0x3880]


def test_background_traffic_runs_for_its_duration_and_copies():
    nbytes = 256 << 20
    src = torch.randint(0, 255, (nbytes,), dtype=torch.uint8, device="cuda")
    dst = torch.zeros_like(src)
    moved = torch.zeros(1, dtype=torch.int64, device="cuda")
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    E.echo_background_traffic(src, dst, 1000, 100, 60_000, moved, stream=s)   # 60 ms at full duty
    s.synchronize()
    dt = time.perf_counter() - t0
    assert 0.055 < dt < 2.0
    full = int(moved.item())
    assert full >= 2 * nbytes                     # at least one full pass (read + written)
    assert torch.equal(dst, src)
    moved.zero_()
    E.echo_background_traffic(src, dst, 250, 100, 60_000, moved, stream=s)    # a quarter of each period
    s.synchronize()
    quarter = int(moved.item())
    assert 0 < quarter < 0.6 * full
    moved.zero_()
    E.echo_background_traffic(src, dst, 0, 100, 60_000, moved, stream=s)      # nothing launched
    s.synchronize()
    assert int(moved.item()) == 0
