"""Pins for the oracle's two other quantizer forms (the ablations of the
quantizer's parameter rounding and of its zero point).

The Echo explainer (section "Echoの仕組み①", mechanism 1) names an
asymmetric, zero-point-aware group quantizer and (section "よくある質問",
FAQ) half-precision parameters, without fixing how the parameters round or
whether the zero is a float or an integer. Besides the default form (fp16
zero rounded down, step rounded up; pinned in test_oracle_quantizer.py) the
oracle has:
  * nearest: zero and step both rounded to the nearest binary16, codes
    clamped to [0, Q];
  * integer zero point: range widened to include 0, step rounded up, zero
    point zp = the integer nearest to -lo/s, codes rint(v/s) + zp clamped,
    dequantization (code - zp) * s.
The checks use facts independent of how the oracle computes: the binary16
table searched by brute force, the nearest grid point by brute force over all
codes in float64, covering and error bounds, exact special cases, and at
call level the residual invariant and a two-rank composition.
"""
import numpy as np
import pytest

import oracle as O

QUANTIZERS = [O.Q_NEAREST, O.Q_INT_ZERO]


def _h(bits):
    return float(np.array([bits], dtype=np.uint16).view(np.float16)[0])


@pytest.fixture(scope="module")
def f16_table():
    vals = np.arange(65536, dtype=np.uint16).view(np.float16).astype(np.float64)
    return np.unique(vals[np.isfinite(vals)])


def _groups(rng, count):
    for i in range(count):
        m = int(rng.choice([1, 2, 3, 5, 8, 16, 31, 32, 64, 100, 128, 256]))
        kind = i % 7
        if kind == 0:
            v = rng.standard_normal(m)
        elif kind == 1:
            v = rng.standard_normal(m) * 0.01 + 30.0          # small range, large offset
        elif kind == 2:
            v = rng.standard_t(3, m) * 50.0                  # heavy tails
        elif kind == 3:
            v = -np.abs(rng.standard_normal(m)) * 1e-3        # all negative, tiny
        elif kind == 4:
            v = rng.uniform(-30000, 30000, m)                # wide
        elif kind == 5:
            v = np.abs(rng.standard_normal(m)) + 5.0          # all positive, away from 0
        else:
            v = rng.standard_normal(m) * 1e-6                 # binary16-subnormal scale
        yield v.astype(np.float32)


def _grid(gq, quantizer, Q):
    """float64 grid points of a quantized group and its (s, offset)."""
    s = _h(gq.s_bits)
    ks = np.arange(Q + 1, dtype=np.float64)
    if quantizer == O.Q_INT_ZERO:
        zp = gq.z_bits
        assert 0 <= zp <= Q
        return (ks - zp) * s, s
    return _h(gq.z_bits) + ks * s, s


# ------------------------------------------------------------------ nearest


@pytest.mark.parametrize("bits", [4, 8])
def test_nearest_params_are_nearest_binary16(f16_table, bits):
    Q = (1 << bits) - 1
    rng = np.random.default_rng(110 + bits)
    for v in _groups(rng, 500):
        gq = O.quantize_group(v, bits, O.Q_NEAREST)
        assert gq.flag == 0
        mn = float(v.min()) + 0.0
        mx = float(v.max()) + 0.0
        z, s = _h(gq.z_bits), _h(gq.s_bits)
        # z: a binary16 value nearest to the minimum (ties either way)
        d = np.abs(f16_table - mn).min()
        assert abs(z - mn) == d, (mn, z)
        assert gq.z_bits != 0x8000
        # s: nearest to (max - min) / Q, up to one binary32 rounding of the quotient
        ratio = (mx - mn) / Q
        dd = np.abs(f16_table - ratio)
        best = dd.min()
        assert abs(s - ratio) <= best + 2.0 ** -22 * ratio + 1e-45, (ratio, s)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("quantizer", QUANTIZERS)
def test_codes_are_nearest_grid_points(bits, quantizer):
    Q = (1 << bits) - 1
    rng = np.random.default_rng(120 + bits + 7 * quantizer)
    for v in _groups(rng, 400):
        gq = O.quantize_group(v, bits, quantizer)
        grid, s = _grid(gq, quantizer, Q)
        assert np.all(gq.codes <= Q)
        if s == 0.0:
            assert np.all(gq.codes == (gq.z_bits if quantizer == O.Q_INT_ZERO else 0))
            continue
        v64 = v.astype(np.float64)
        dist = np.abs(v64[:, None] - grid[None, :])
        best = dist.min(axis=1)
        mine = dist[np.arange(v.size), gq.codes.astype(np.int64)]
        slack = 2.0 ** -21 * (np.abs(v64) + np.abs(grid).max())
        assert np.all(mine <= best + slack), (quantizer, (mine - best).max())


@pytest.mark.parametrize("bits", [4, 8])
def test_nearest_error_bound(bits):
    """Inside [z, z + Q s] the error is at most s/2; outside, the clamp costs
    at most the distance to the nearer end of the grid."""
    Q = (1 << bits) - 1
    rng = np.random.default_rng(130 + bits)
    for v in _groups(rng, 400):
        gq = O.quantize_group(v, bits, O.Q_NEAREST)
        z, s = _h(gq.z_bits), _h(gq.s_bits)
        v64 = v.astype(np.float64)
        over = np.maximum(z - v64, 0.0) + np.maximum(v64 - (z + Q * s), 0.0)
        err = np.abs(v64 - gq.vhat.astype(np.float64))
        bound = s / 2 + over + 2.0 ** -22 * (abs(z) + Q * s + np.abs(v64))
        assert np.all(err <= bound)
        exact = (z + gq.codes.astype(np.float64) * s).astype(np.float32)
        assert np.array_equal(exact.view(np.uint32), gq.vhat.view(np.uint32))


@pytest.mark.parametrize("bits", [4, 8])
def test_nearest_constant_group(bits):
    for c in [0.0, -0.0, 1.0, -2.5, 1000.3, -12345.6, 3.0e-6]:
        v = np.full(29, c, np.float32)
        gq = O.quantize_group(v, bits, O.Q_NEAREST)
        want = np.float32(np.float16(np.float32(c) + np.float32(0.0)))   # numpy: nearest, ties to even
        assert gq.s_bits == 0 and np.all(gq.codes == 0)
        assert np.all(gq.vhat == want), (c, gq.vhat[0], want)


# --------------------------------------------------------- integer zero point


@pytest.mark.parametrize("bits", [4, 8])
def test_int_zero_scale_and_zero_point(f16_table, bits):
    Q = (1 << bits) - 1
    rng = np.random.default_rng(140 + bits)
    for v in _groups(rng, 500):
        gq = O.quantize_group(v, bits, O.Q_INT_ZERO)
        assert gq.flag == 0
        lo = min(float(v.min()), 0.0)
        hi = max(float(v.max()), 0.0)
        s, zp = _h(gq.s_bits), gq.z_bits
        span = hi - lo
        # s: the smallest binary16 step with Q*s >= span (one binary32 rounding)
        assert Q * s >= span * (1 - 2.0 ** -22)
        if s > 0:
            k = np.searchsorted(f16_table, s, side="left")
            assert Q * f16_table[k - 1] < span * (1 + 2.0 ** -22)
            # zp: the integer nearest to -lo/s (one binary32 rounding of the ratio)
            assert abs(zp - (-lo / s)) <= 0.5 + 2.0 ** -20 * Q
            # the grid (k - zp) s covers [lo, hi] to within half a step
            assert -zp * s <= lo + s / 2 * (1 + 2.0 ** -20)
            assert (Q - zp) * s >= hi - s / 2 * (1 + 2.0 ** -20)
        else:
            assert span == 0.0 and zp == 0


@pytest.mark.parametrize("bits", [4, 8])
def test_int_zero_error_and_exact_zero(bits):
    Q = (1 << bits) - 1
    rng = np.random.default_rng(150 + bits)
    for v in _groups(rng, 400):
        v = v.copy()
        v[rng.integers(0, v.size)] = 0.0                  # a zero in every group
        gq = O.quantize_group(v, bits, O.Q_INT_ZERO)
        s, zp = _h(gq.s_bits), gq.z_bits
        v64 = v.astype(np.float64)
        err = np.abs(v64 - gq.vhat.astype(np.float64))
        assert np.all(err <= s / 2 * (1 + 2.0 ** -20) + 2.0 ** -22 * np.abs(v64))
        # zero is on the grid and decodes to exactly 0
        assert np.all(gq.vhat[v == 0.0] == 0.0)
        # dequantization is the exact product (code - zp) * s
        exact = ((gq.codes.astype(np.float64) - zp) * s)
        assert np.array_equal(exact.astype(np.float32), gq.vhat)
        assert np.array_equal(exact, gq.vhat.astype(np.float64))


@pytest.mark.parametrize("bits", [4, 8])
def test_int_zero_special_groups(bits):
    Q = (1 << bits) - 1
    # all zero: no step, zero point 0
    gq = O.quantize_group(np.zeros(40, np.float32), bits, O.Q_INT_ZERO)
    assert gq.s_bits == 0 and gq.z_bits == 0 and np.all(gq.codes == 0) and np.all(gq.vhat == 0)
    # all positive: the range starts at 0, zp = 0
    v = np.linspace(2.0, 7.0, 33).astype(np.float32)
    gq = O.quantize_group(v, bits, O.Q_INT_ZERO)
    assert gq.z_bits == 0
    # all negative: the range ends at 0, zp = Q
    gq = O.quantize_group(-v, bits, O.Q_INT_ZERO)
    assert gq.z_bits == Q
    # a grid of exact multiples of a binary16 step round-trips exactly
    step = 0.25
    k = np.arange(-5, Q - 5 + 1)
    v = (k * step).astype(np.float32)
    gq = O.quantize_group(v, bits, O.Q_INT_ZERO)
    assert _h(gq.s_bits) == step and gq.z_bits == 5
    assert np.array_equal(gq.vhat, v)


# --------------------------------------------------------------- whole call


def _rand_bf16(rng, shape, scale=1.0):
    v = (rng.standard_normal(shape) * scale).astype(np.float32)
    return (v.view(np.uint32) >> 16).astype(np.uint16)     # truncation: any bf16 values do


def _f32(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


CASES = [(2, 1000, 128, 4), (3, 777, 64, 8), (5, 4096, 32, 4), (8, 3000, 128, 4), (1, 500, 128, 4)]


@pytest.mark.parametrize("P,n,group,bits", CASES)
@pytest.mark.parametrize("quantizer", QUANTIZERS)
@pytest.mark.parametrize("feedback", [False, True])
def test_residuals_sum_to_minus_injected_error(P, n, group, bits, quantizer, feedback):
    rng = np.random.default_rng(17 * P + n + feedback + 5 * quantizer)
    G = -(-n // group)
    ld = G * group
    x = np.zeros((P, ld), np.uint16)
    x[:, :n] = _rand_bf16(rng, (P, n), 2.0)
    el = es = None
    if feedback:
        el = (rng.standard_normal((P, ld)) * 0.05).astype(np.float32)
        es = (rng.standard_normal((P, ld)) * 0.05).astype(np.float32)
    res = O.echo_allreduce(x, n_total=n, group=group, bits=bits, e_long=el, e_short=es, w=0.3,
                           debug=True, quantizer=quantizer)
    assert res.flags == 0
    for r in range(1, P):
        assert np.array_equal(res.y[r, :n], res.y[0, :n])
    y = _f32(res.y[0, :n]).astype(np.float64)
    xp = res.xprime[:, :n].astype(np.float64)
    rho = res.rho[:, :n].astype(np.float64)
    injected = y - xp.sum(axis=0)
    bound = (P + 2) * 2.0 ** -23 * (np.abs(xp).sum(axis=0) + np.abs(y) + np.abs(rho).sum(axis=0))
    assert np.all(np.abs(rho.sum(axis=0) + injected) <= bound + 1e-30)
    assert res.passes.max() <= 2


@pytest.mark.parametrize("quantizer", QUANTIZERS)
def test_single_rank_is_identity(quantizer):
    rng = np.random.default_rng(160 + quantizer)
    x = _rand_bf16(rng, (1, 512))
    res = O.echo_allreduce(x, n_total=512, group=128, bits=4, quantizer=quantizer)
    assert np.array_equal(res.y, x)


@pytest.mark.parametrize("quantizer", QUANTIZERS)
@pytest.mark.parametrize("bits", [4, 8])
def test_two_rank_composition(quantizer, bits):
    """P = 2: the owner's output is the group quantizer of (own x + the
    other rank's dequantized payload), decoded with the same form."""
    Q = (1 << bits) - 1
    rng = np.random.default_rng(170 + quantizer + bits)
    group, n = 64, 256
    x = _rand_bf16(rng, (2, n), 1.5)
    res = O.echo_allreduce(x, n_total=n, group=group, bits=bits, quantizer=quantizer)
    G = n // group
    for j in range(G):
        o = O.owner(j, G, 2)
        other = 1 - o
        sl = slice(j * group, (j + 1) * group)
        sent = O.quantize_group(_f32(x[other, sl]), bits, quantizer)
        got_codes = O.unpack_codes(res.a2a_codes[other, j], group, bits)
        assert np.array_equal(got_codes, sent.codes)
        assert tuple(res.a2a_params[other, j]) == (sent.s_bits, sent.z_bits)
        # rank order 0, 1: the owner's own term enters unquantized
        terms = [None, None]
        terms[o] = _f32(x[o, sl])
        terms[other] = sent.vhat
        acc = (terms[0] + terms[1]).astype(np.float32)
        back = O.quantize_group(acc, bits, quantizer)
        assert np.array_equal(O.unpack_codes(res.gather_codes[j], group, bits), back.codes)
        want = (back.vhat.view(np.uint32) + 0x7FFF + ((back.vhat.view(np.uint32) >> 16) & 1)) >> 16
        assert np.array_equal(res.y[0, sl], want.astype(np.uint16))
        assert np.all(back.codes <= Q)


@pytest.mark.parametrize("quantizer", QUANTIZERS)
def test_forms_differ_from_the_default(quantizer):
    """The forms are really different quantizers (a dropped mode switch would
    make them all the default)."""
    rng = np.random.default_rng(180 + quantizer)
    diff = 0
    for v in _groups(rng, 60):
        a = O.quantize_group(v, 4, O.Q_DIRECTED)
        b = O.quantize_group(v, 4, quantizer)
        diff += int((a.s_bits, a.z_bits) != (b.s_bits, b.z_bits) or not np.array_equal(a.codes, b.codes))
    assert diff > 20
