"""Pins of the two evaluation orders the oracle fixes.

1. The owner's binary32 sum runs in rank order 0, 1, ..., P-1, its own
   unquantized x' entering at its own rank (the explainer's "Echoの仕組み①":
   the owner sums the P partial results at high precision; the fixed rank
   order is the reading this build states for it).
2. The EMA update is evaluated as u = (1 - alpha) * e, v = alpha * rho,
   e = u + v (the explainer's "Echoの仕組み②": two moving averages of the
   exposed error; the update formula is the reading this build states).

Each expected value below is worked out by hand in exact binary arithmetic,
so a different order -- reversed ranks, the owner's term first or last, the
incremental form e + alpha * (rho - e) -- gives different bits.
"""
import numpy as np

import oracle as O

# binary32 / bf16 / fp16 values used below
TINY = 2.0 ** -14      # smallest normal fp16; bf16 bits 0x3880
BIG = 32768.0          # 2^15, exact in bf16 and fp16; bf16 bits 0x4700
BF16 = {0.0: 0x0000, TINY: 0x3880, BIG: 0x4700, -BIG: 0xC700}


def test_owner_sum_runs_in_rank_order():
    """P = 3, groups of 32, n = 96: three groups, group j owned by rank j.
    Every group is constant on every rank, so each non-owner's quantized term
    is its value exactly (s = 0, x_hat = z = the value, which is an fp16
    number) and no feedback is applied (no state: x' = x).

    Terms per group (rank 0, rank 1, rank 2; the owner's in brackets):

      group 0: [TINY], BIG, -BIG
        rank order  (TINY + BIG) + (-BIG): TINY + 2^15 needs 30 significant
                    bits, rounds to 2^15; then 0.                     -> 0
        owner last  (BIG - BIG) + TINY                                -> TINY
      group 1: BIG, [-BIG], TINY
        rank order  (BIG - BIG) + TINY = TINY                         -> TINY
        reversed    (TINY - BIG) rounds to -BIG; + BIG = 0            -> 0
      group 2: BIG, -BIG, [TINY]
        rank order  (BIG - BIG) + TINY = TINY                         -> TINY
        owner first (TINY + BIG) rounds to BIG; - BIG = 0             -> 0

    Each sum is constant over its group, so requantization is exact
    (z = fp16 value, s = 0) and every rank's bf16 output is the sum itself.
    """
    P, group, n = 3, 32, 96
    terms = [(TINY, BIG, -BIG), (BIG, -BIG, TINY), (BIG, -BIG, TINY)]
    x = np.zeros((P, n), np.uint16)
    for j, col in enumerate(terms):
        for r in range(P):
            x[r, j * group:(j + 1) * group] = BF16[col[r]]
    assert [O.owner(j, 3, P) for j in range(3)] == [0, 1, 2]
    res = O.echo_allreduce(x, n_total=n, group=group, bits=4)
    want = [0.0, TINY, TINY]
    for j in range(3):
        assert np.all(res.y[:, j * group:(j + 1) * group] == BF16[want[j]]), f"group {j}"
    assert res.flags == 0


def test_ema_update_evaluation_order():
    """alpha = 0.25 (so 1 - alpha = 0.75 exactly), e = 1, rho = -(1 + 2^-23).

      u = 0.75 * 1 = 0.75
      v = 0.25 * rho = -(0.25 + 2^-25)                (exact)
      u + v = 0.5 - 2^-25, exact in binary32 (the spacing in [0.25, 0.5)
              is 2^-25)                                -> 0x3EFFFFFF

    The incremental form e + alpha * (rho - e) rounds rho - e = -(2 + 2^-23)
    to -2 (a tie in [2, 4), spacing 2^-22, to even), then 1 - 0.5 = 0.5
    (0x3F000000): one ulp away.
    """
    e = np.array([1.0], np.float32)
    rho = np.array([-(1.0 + 2.0 ** -23)], np.float32)
    O.ema_update(e, rho, 0.25)
    assert e.view(np.uint32)[0] == 0x3EFFFFFF
    assert float(e[0]) == 0.5 - 2.0 ** -25
