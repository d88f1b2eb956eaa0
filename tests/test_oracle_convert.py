"""Pins for the oracle's own bf16 / fp16 converters.

The oracle rounds binary32 to binary16 to nearest-even (for the bf16 outputs'
sibling format), toward -inf (the zero-point z) and toward +inf (the scale s),
and to bfloat16 to nearest-even (the reduced outputs). These tests check them
against things that are not the oracle:
  * numpy's float16 conversion (IEEE round-to-nearest-even) and decoding;
  * torch's CPU bfloat16 conversion (round-to-nearest-even) and decoding;
  * brute force over the table of all finite binary16 values for the two
    directed modes (the largest value <= x, the smallest value >= x).
"""
import numpy as np
import pytest
import torch

import oracle as O


def _f32_samples(rng, count):
    """float32 values spread over every binade binary16 touches, plus ties."""
    sign = rng.choice([-1.0, 1.0], size=count)
    e = rng.integers(-30, 18, size=count)
    frac = rng.random(count)
    x = (sign * np.ldexp(1.0 + frac, e)).astype(np.float32)
    # exact midpoints between neighbouring binary16 values (ties)
    h = rng.integers(0, 0x7BFF, size=count // 4).astype(np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    mid = ((lo + hi) / 2).astype(np.float32)
    assert np.all(mid.astype(np.float64) == (lo + hi) / 2)   # representable in binary32
    special = np.array([0.0, -0.0, 65504.0, 65519.0, 65520.0, 65535.9, 65536.0, 70000.0,
                        -65520.0, -70000.0, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26,
                        2.0 ** -14, 2.0 ** -14 - 2.0 ** -25, 1e-30, -1e-30, 3e38, -3e38],
                       dtype=np.float32)
    return np.concatenate([x, mid, -mid, special])


def _bits16(v):
    return np.array([v], dtype=np.float16).view(np.uint16)[0]


def test_f16_decode_all_patterns(oracle_lib):
    for b in range(65536):
        ref = np.array([b], dtype=np.uint16).view(np.float16).astype(np.float32)[0]
        got = O.f16_to_f32(b)
        if np.isnan(ref):
            assert np.isnan(got)
        else:
            assert np.float32(got).view(np.uint32) == ref.view(np.uint32), hex(b)


def test_f16_round_nearest_even_matches_numpy(oracle_lib):
    rng = np.random.default_rng(1)
    for x in _f32_samples(rng, 4000):
        with np.errstate(over="ignore"):
            ref = int(_bits16(np.float16(x)))
        got = O.f32_to_f16(float(x), O.RN)
        assert got == ref, (float(x), hex(got), hex(ref))


@pytest.fixture(scope="module")
def f16_table():
    vals = np.arange(65536, dtype=np.uint16).view(np.float16).astype(np.float64)
    return np.unique(vals[np.isfinite(vals)])


@pytest.mark.parametrize("mode", [O.RD, O.RU])
def test_f16_directed_rounding_brute_force(oracle_lib, f16_table, mode):
    rng = np.random.default_rng(2 + mode)
    for x in _f32_samples(rng, 3000):
        xd = float(x)
        if mode == O.RD:
            idx = np.searchsorted(f16_table, xd, side="right") - 1
            ref = f16_table[idx] if idx >= 0 else -np.inf
        else:
            idx = np.searchsorted(f16_table, xd, side="left")
            ref = f16_table[idx] if idx < len(f16_table) else np.inf
        bits = O.f32_to_f16(xd, mode)
        got = float(np.array([bits], dtype=np.uint16).view(np.float16)[0])
        assert got == ref, (xd, mode, got, ref)
        if got == 0.0:
            # a zero result keeps the sign of its input under IEEE rounding
            assert (bits >> 15) == (1 if np.signbit(x) else 0), (xd, hex(bits))


def test_f16_directed_overflow_and_zero_signs(oracle_lib):
    assert O.f32_to_f16(70000.0, O.RD) == 0x7BFF        # stays at 65504
    assert O.f32_to_f16(70000.0, O.RU) == 0x7C00        # +inf
    assert O.f32_to_f16(-70000.0, O.RD) == 0xFC00       # -inf
    assert O.f32_to_f16(-70000.0, O.RU) == 0xFBFF       # -65504
    assert O.f32_to_f16(1e-30, O.RD) == 0x0000
    assert O.f32_to_f16(1e-30, O.RU) == 0x0001          # smallest subnormal
    assert O.f32_to_f16(-1e-30, O.RU) == 0x8000         # -0
    assert O.f32_to_f16(-1e-30, O.RD) == 0x8001


def test_bf16_decode_all_patterns(oracle_lib):
    bits = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    for b in range(0, 65536, 7):
        got = O.bf16_to_f32(b)
        if np.isnan(ref[b]):
            assert np.isnan(got)
        else:
            assert np.float32(got).view(np.uint32) == ref[b].view(np.uint32)


def test_bf16_round_nearest_even_matches_torch(oracle_lib):
    rng = np.random.default_rng(5)
    raw = rng.integers(0, 2 ** 32, size=6000, dtype=np.uint64).astype(np.uint32)
    ties = (raw & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    special = np.array([0x7F7F8000, 0x7F7FFFFF, 0xFF7F8000, 0x00008000, 0x00018000,
                        0x80008000, 0x3F808000, 0x3F818000, 0x00000001], dtype=np.uint32)
    u = np.concatenate([raw, ties, special])
    f = u.view(np.float32)
    f = f[~np.isnan(f)]
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for x, r in zip(f, ref):
        got = O.f32_to_bf16(float(x))
        assert got == int(r), (hex(np.float32(x).view(np.uint32)), hex(got), hex(int(r)))
