"""Pins of the 16-bit baseline all-reduce (the comparison the Echo abstract
and the explainer's results table make against a 16-bit all-reduce), as the
oracle simulates it over P virtual ranks: every rank receives bf16_rn of the
binary32 sum of the P bf16 inputs in rank order.

Checked against what arithmetic fixes, not against a retyped formula:
  * P = 1 returns the input exactly;
  * sums of values whose exact sum is a bf16 number come back exactly
    (integers k/8 with |sum| < 2^8 have at most 8 significant bits);
  * the rank order: the hand-worked sums of the owner-order pin, where
    reversed order gives different bits;
  * a sum of two bf16 numbers rounds once to nearest-even: brute force over
    pairs in fp64 (exact for such sums), compared with numpy's own
    binary32 -> bfloat16 rounding through torch;
  * every rank receives the same result.
"""
import numpy as np
import torch

import oracle as O


def _bits(v):
    return torch.tensor(v, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_single_rank_is_identity():
    rng = np.random.default_rng(1)
    x = _bits(rng.standard_normal((1, 1000)) * 3)
    assert np.array_equal(O.bf16_allreduce(x), x)


def test_representable_sums_are_exact():
    rng = np.random.default_rng(2)
    P, n = 8, 4096
    k = rng.integers(-15, 16, size=(P, n))             # each term k/8 with |k| <= 15
    # every partial sum is a multiple of 1/8 of magnitude <= 15: at most 7 significant bits
    x = _bits(k / 8.0)
    y = O.bf16_allreduce(x)
    want = _bits(k.sum(axis=0, keepdims=True) / 8.0)
    assert np.array_equal(y, np.repeat(want, P, axis=0))


def test_rank_order_is_pinned():
    """TINY = 2^-14, BIG = 2^15 as in the owner-order pin:
    (TINY + BIG) + (-BIG) = 0 in rank order (TINY + 2^15 rounds to 2^15),
    while the reverse order gives TINY; (BIG - BIG) + TINY = TINY."""
    x = _bits([[2.0 ** -14, 32768.0], [32768.0, -32768.0], [-32768.0, 2.0 ** -14]])
    y = O.bf16_allreduce(x)
    assert y[:, 0].tolist() == [0, 0, 0]
    assert y[:, 1].tolist() == [0x3880] * 3


def test_two_term_sums_round_once_to_nearest_even():
    rng = np.random.default_rng(3)
    a = _bits(rng.standard_normal(20000) * 10)
    b = _bits(rng.standard_normal(20000) * 0.1)
    y = O.bf16_allreduce(np.stack([a, b]))
    fa = (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    fb = (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    exact = fa + fb                                     # exact in fp64 (8-bit significands)
    # the binary32 sum is exact here too (exponents within 24 bits of each other) -- skip the rest
    ok = np.abs(np.log2(np.abs(fa) + 1e-300) - np.log2(np.abs(fb) + 1e-300)) < 15
    want = _bits(exact.astype(np.float32))              # binary32 value exact, then one RN to bf16
    assert np.array_equal(y[0][ok], want[ok]) and np.array_equal(y[1], y[0])
    assert ok.sum() > 15000
