"""Pins for the oracle's group quantizer, packing and segment table.

The quantizer is the zero-point-aware asymmetric group quantizer of the Echo
explainer (section "Echoの仕組み①", mechanism 1) carrying half-precision
parameters (section "よくある質問", FAQ). The checks below use only facts
that do not depend on how the oracle computes:
  * z is the largest binary16 value <= the group minimum (brute force over the
    binary16 table);
  * s is the smallest binary16 step whose grid z + k*s (k <= Q) reaches the
    group maximum, up to one binary32 rounding;
  * each code is the nearest grid point (brute force over all 2^bits codes in
    float64), ties within binary32 rounding accepted;
  * |v - x_hat| <= s/2 (+ binary32 rounding);
  * constant groups of binary16-representable values round-trip exactly.
"""
import numpy as np
import pytest

import oracle as O


def _h(bits):
    return float(np.array([bits], dtype=np.uint16).view(np.float16)[0])


@pytest.fixture(scope="module")
def f16_table():
    vals = np.arange(65536, dtype=np.uint16).view(np.float16).astype(np.float64)
    return np.unique(vals[np.isfinite(vals)])


def _groups(rng, count):
    for i in range(count):
        m = int(rng.choice([1, 2, 3, 5, 8, 16, 31, 32, 64, 100, 128, 256]))
        kind = i % 6
        if kind == 0:
            v = rng.standard_normal(m)
        elif kind == 1:
            v = rng.standard_normal(m) * 0.01 + 30.0          # small range, large offset
        elif kind == 2:
            v = rng.standard_t(3, m) * 50.0                  # heavy tails
        elif kind == 3:
            v = -np.abs(rng.standard_normal(m)) * 1e-3        # all negative, tiny
        elif kind == 4:
            v = rng.uniform(-60000, 60000, m)                # near the fp16 edge
        else:
            v = rng.standard_normal(m) * 1e-6                 # binary16-subnormal scale
        yield v.astype(np.float32)


@pytest.mark.parametrize("bits", [4, 8])
def test_params_are_directed_fp16_roundings(f16_table, bits):
    Q = (1 << bits) - 1
    rng = np.random.default_rng(10 + bits)
    for v in _groups(rng, 600):
        gq = O.quantize_group(v, bits)
        assert gq.flag == 0
        mn = float(v.min()) + 0.0
        mx = float(v.max()) + 0.0
        z = _h(gq.z_bits)
        s = _h(gq.s_bits)
        # z: the largest binary16 value not above the minimum
        idx = np.searchsorted(f16_table, mn, side="right") - 1
        assert z == f16_table[idx], (mn, z)
        assert gq.z_bits != 0x8000                       # -0 is canonicalized away
        # s: the grid reaches the maximum, and one binary16 step less would not
        span = mx - z
        assert Q * s >= span * (1 - 2.0 ** -22), (span, s)
        if s > 0:
            k = np.searchsorted(f16_table, s, side="left")
            s_prev = f16_table[k - 1]
            assert Q * s_prev < span * (1 + 2.0 ** -22), (span, s, s_prev)
        else:
            assert span == 0.0


@pytest.mark.parametrize("bits", [4, 8])
def test_codes_are_nearest_grid_points(bits):
    Q = (1 << bits) - 1
    rng = np.random.default_rng(20 + bits)
    ks = np.arange(Q + 1, dtype=np.float64)
    for v in _groups(rng, 400):
        gq = O.quantize_group(v, bits)
        z = _h(gq.z_bits)
        s = _h(gq.s_bits)
        if s == 0.0:
            assert np.all(gq.codes == 0)
            continue
        grid = z + ks * s                                      # exact in float64
        dist = np.abs(v.astype(np.float64)[:, None] - grid[None, :])
        best = dist.min(axis=1)
        mine = dist[np.arange(v.size), gq.codes.astype(np.int64)]
        slack = 2.0 ** -21 * (np.abs(v.astype(np.float64)) + abs(z) + Q * s)
        assert np.all(mine <= best + slack)
        assert np.all(gq.codes <= Q)


@pytest.mark.parametrize("bits", [4, 8])
def test_error_within_half_step(bits):
    Q = (1 << bits) - 1
    rng = np.random.default_rng(30 + bits)
    for v in _groups(rng, 400):
        gq = O.quantize_group(v, bits)
        z = _h(gq.z_bits)
        s = _h(gq.s_bits)
        err = np.abs(v.astype(np.float64) - gq.vhat.astype(np.float64))
        bound = s / 2 + 2.0 ** -22 * (abs(z) + Q * s + np.abs(v.astype(np.float64)))
        assert np.all(err <= bound), (err.max(), s)
        # the dequantized value is exactly the grid point rounded once to binary32
        exact = (z + gq.codes.astype(np.float64) * s).astype(np.float32)
        assert np.array_equal(exact.view(np.uint32), gq.vhat.view(np.uint32))


def test_eight_bits_beats_four_bits():
    rng = np.random.default_rng(40)
    e4 = e8 = 0.0
    for _ in range(200):
        v = rng.standard_normal(128).astype(np.float32)
        e4 += float(np.sum((O.quantize_group(v, 4).vhat - v) ** 2))
        e8 += float(np.sum((O.quantize_group(v, 8).vhat - v) ** 2))
    # 17x finer step => error power ~ 289x smaller
    assert e8 * 100 < e4


@pytest.mark.parametrize("bits", [4, 8])
def test_constant_group_is_exact(bits):
    for c in [0.0, -0.0, 1.0, -2.5, 0.375, 1000.0, -65504.0, 6.1035156e-05]:
        v = np.full(37, c, np.float32)
        gq = O.quantize_group(v, bits)
        assert gq.s_bits == 0
        assert np.all(gq.codes == 0)
        assert np.all(gq.vhat == np.float32(c))


@pytest.mark.parametrize("bits", [4, 8])
def test_negative_zero_extremes_are_canonical(bits):
    """A group whose minimum (or maximum) is -0 quantizes exactly as with +0:
    the +0 added to min and max makes the parameters independent of how a
    min/max reduction orders signed zeros."""
    for v in ([-0.0, 1.0, 2.0, 0.5], [-0.0, -1.5, -0.25], [-0.0, -0.0], [-0.0, 0.0, 3.0]):
        a = O.quantize_group(np.array(v, np.float32), bits)
        b = O.quantize_group(np.array([0.0 if x == 0 else x for x in v], np.float32), bits)
        assert (a.s_bits, a.z_bits) == (b.s_bits, b.z_bits)
        assert a.z_bits != 0x8000 and a.s_bits != 0x8000
        assert np.array_equal(a.codes, b.codes)


def test_range_flag():
    assert O.quantize_group(np.array([1.0, 70000.0], np.float32), 4).flag == O.FLAG_RANGE
    assert O.quantize_group(np.array([1.0, np.nan], np.float32), 4).flag == O.FLAG_RANGE
    assert O.quantize_group(np.array([-65504.0, 65504.0], np.float32), 4).flag == 0


def test_packing_layout_golden():
    """Reading of the payload: element 2i -> low nibble, 2i+1 -> high nibble."""
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "packing.json")) as f:
        g = json.load(f)
    for case in g["cases"]:
        codes = np.array(case["codes"], np.uint8)
        packed = O.pack_codes(codes, case["group"], case["bits"])
        assert packed.tolist() == case["packed"]
        assert O.unpack_codes(packed, case["group"], case["bits"]).tolist() == case["codes"]


@pytest.mark.parametrize("P,G", [(1, 1), (2, 1), (3, 7), (4, 4), (8, 5), (8, 1000), (16, 33), (64, 63)])
def test_segments_partition_groups(P, G):
    begins = [O.segment_begin(s, G, P) for s in range(P + 1)]
    assert begins[0] == 0 and begins[-1] == G
    sizes = np.diff(begins)
    assert np.all(sizes >= 0) and sizes.max() - sizes.min() <= 1
    for j in range(0, G, max(1, G // 50)):
        o = O.owner(j, G, P)
        assert begins[o] <= j < begins[o + 1]
