"""Pins for one oracle all-reduce call.

Facts checked (none of them re-derives the oracle's arithmetic):
  * at most two quantizer passes per value, for any P: a non-owner's
    contribution passes twice, the owner's once, a lone rank's never
    (Echo abstract; explainer section "Echoの仕組み①");
  * the ranks' residuals sum to minus the injected error,
    sum_r rho_r = sum_r x'_r - y, to binary32 round-off
    (explainer section "Echoの仕組み②");
  * stage-1 and stage-2 errors stay within half a quantization step;
  * every rank receives the same result;
  * P = 1 with fresh state returns its input exactly; constant groups whose
    values and sums are representable come back exactly with zero residual;
  * the EMA recursion matches its closed form (a geometric sum) and the
    compensation reduces to its special cases;
  * payload size: 4-bit codes + two fp16 per group of 128 = 4.25 bits per
    element, i.e. the 3.8x ceiling of the explainer's FAQ.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W


def _rand_bf16(rng, shape, scale=1.0):
    v = torch.from_numpy((rng.standard_normal(shape) * scale).astype(np.float32))
    return W.bf16_bits(v.to(torch.bfloat16))


def _f32(bits_u16):
    return (bits_u16.astype(np.uint32) << 16).view(np.float32)


def _h(a):
    return np.asarray(a, np.uint16).view(np.float16).astype(np.float64)


CASES = [
    # P, n, group, bits
    (1, 1000, 128, 4),
    (2, 4096, 128, 4),
    (3, 1000, 32, 4),
    (4, 777, 64, 8),
    (8, 8192, 128, 4),
    (8, 1000, 128, 4),      # G = 8 = P, partial last group
    (16, 3000, 128, 4),     # G < P: empty segments
    (5, 2048, 256, 8),
]


@pytest.mark.parametrize("P,n,group,bits", CASES)
def test_pass_count_at_most_two(P, n, group, bits):
    rng = np.random.default_rng(P * 1000 + n)
    G = -(-n // group)
    jc = G
    x = np.zeros((P, jc * group), np.uint16)
    x[:, :n] = _rand_bf16(rng, (P, n))
    res = O.echo_allreduce(x, n_total=n, group=group, bits=bits, debug=True)
    assert res.passes.max() <= 2
    for j in range(G):
        o = O.owner(j, G, P)
        lo, hi = j * group, min(n, (j + 1) * group)
        for r in range(P):
            want = 0 if P == 1 else (1 if r == o else 2)
            assert np.all(res.passes[r, lo:hi] == want), (j, r)


@pytest.mark.parametrize("P,n,group,bits", CASES)
@pytest.mark.parametrize("feedback", [False, True])
def test_residuals_sum_to_minus_injected_error(P, n, group, bits, feedback):
    rng = np.random.default_rng(7 * P + n + feedback)
    G = -(-n // group)
    ld = G * group
    x = np.zeros((P, ld), np.uint16)
    x[:, :n] = _rand_bf16(rng, (P, n), 2.0)
    el = es = None
    if feedback:
        el = (rng.standard_normal((P, ld)) * 0.05).astype(np.float32)
        es = (rng.standard_normal((P, ld)) * 0.05).astype(np.float32)
    res = O.echo_allreduce(x, n_total=n, group=group, bits=bits, e_long=el, e_short=es,
                           eta=1.0, alpha_long=0.05, alpha_short=0.5, w=0.3, debug=True)
    assert res.flags == 0
    y = _f32(res.y[:, :n]).astype(np.float64)
    for r in range(1, P):
        assert np.array_equal(res.y[r, :n], res.y[0, :n])          # same result everywhere
    xp = res.xprime[:, :n].astype(np.float64)
    rho = res.rho[:, :n].astype(np.float64)
    injected = y[0] - xp.sum(axis=0)
    lhs = rho.sum(axis=0)
    bound = (P + 2) * 2.0 ** -23 * (np.abs(xp).sum(axis=0) + np.abs(y[0]) + np.abs(rho).sum(axis=0))
    assert np.all(np.abs(lhs + injected) <= bound + 1e-30)
    if P >= 2:
        assert np.abs(injected).max() > 0        # 4-bit rounding does inject an error


@pytest.mark.parametrize("P,n,group,bits", CASES)
def test_errors_within_half_step_at_both_stages(P, n, group, bits):
    Q = (1 << bits) - 1
    rng = np.random.default_rng(11 * P + n)
    G = -(-n // group)
    ld = G * group
    x = np.zeros((P, ld), np.uint16)
    x[:, :n] = _rand_bf16(rng, (P, n), 3.0)
    res = O.echo_allreduce(x, n_total=n, group=group, bits=bits, debug=True)
    if P == 1:
        return
    cb = group * bits // 8
    for j in range(G):
        o = O.owner(j, G, P)
        lo, hi = j * group, min(n, (j + 1) * group)
        m = hi - lo
        for r in range(P):
            if r == o:
                continue
            s, z = _h(res.a2a_params[r, j])
            codes = O.unpack_codes(res.a2a_codes[r, j], group, bits)[:m].astype(np.float64)
            v = res.xprime[r, lo:hi].astype(np.float64)
            err = np.abs(v - (z + codes * s))
            assert np.all(err <= s / 2 + 2.0 ** -22 * (abs(z) + Q * s + np.abs(v)))
            assert np.all(O.unpack_codes(res.a2a_codes[r, j], group, bits)[m:] == 0)  # padding
            assert cb == res.a2a_codes.shape[2]
        # stage 2: the owner's sum against what every rank receives
        s, z = _h(res.gather_params[j])
        codes = O.unpack_codes(res.gather_codes[j], group, bits)[:m].astype(np.float64)
        acc = res.rho[o, lo:hi].astype(np.float64) + _f32(res.y[o, lo:hi]).astype(np.float64)
        err = np.abs(acc - (z + codes * s))
        assert np.all(err <= s / 2 + 2.0 ** -21 * (abs(z) + Q * s + np.abs(acc)))


def test_single_rank_fresh_state_is_identity():
    rng = np.random.default_rng(3)
    n = 1000
    G = -(-n // 128)
    x = np.zeros((1, G * 128), np.uint16)
    x[:, :n] = _rand_bf16(rng, (1, n))
    el = np.zeros_like(x, dtype=np.float32)
    es = np.zeros_like(el)
    res = O.echo_allreduce(x, n_total=n, group=128, bits=4, e_long=el, e_short=es, debug=True)
    assert np.array_equal(res.y[:, :n], x[:, :n])
    assert np.all(res.rho == 0) and np.all(el == 0) and np.all(es == 0)
    assert np.all(res.passes == 0)


@pytest.mark.parametrize("P", [2, 3, 8])
@pytest.mark.parametrize("bits", [4, 8])
def test_constant_representable_groups_are_exact(P, bits):
    group, G = 64, 9
    n = G * group
    rng = np.random.default_rng(P + bits)
    k = rng.integers(-63, 64, size=(P, G))                       # value k/4 per (rank, group)
    vals = np.repeat(k / 4.0, group, axis=1).astype(np.float32)
    x = W.bf16_bits(torch.from_numpy(vals).to(torch.bfloat16))
    el = np.zeros((P, n), np.float32)
    es = np.zeros_like(el)
    res = O.echo_allreduce(x, n_total=n, group=group, bits=bits, e_long=el, e_short=es, debug=True)
    want = vals.astype(np.float64).sum(axis=0)
    for r in range(P):
        assert np.array_equal(_f32(res.y[r]).astype(np.float64), want)
    assert np.all(res.rho == 0) and np.all(el == 0) and np.all(es == 0)


def test_two_rank_exact_grid_worked_example():
    """P = 2, group 32, two groups. Rank 1 sends group 0 to rank 0 and rank 0
    sends group 1 to rank 1. Rank 1's group 0 holds (i mod 16)/4, which sits on
    the grid z = 0, s = 1/4 exactly (codes i mod 16); rank 0's own group 0 is
    all ones, so the owner's sum is 1 + (i mod 16)/4, on the grid z = 1,
    s = 1/4. Everything is exact: no residual anywhere."""
    group, n = 32, 64
    i = np.arange(32)
    r0 = np.concatenate([np.ones(32), (i % 8) * 0.5])            # group 1: 0..3.5 step 1/2
    r1 = np.concatenate([(i % 16) / 4.0, np.full(32, -1.0)])
    x = W.bf16_bits(torch.tensor(np.stack([r0, r1]), dtype=torch.float32).to(torch.bfloat16))
    el = np.zeros((2, n), np.float32)
    es = np.zeros_like(el)
    res = O.echo_allreduce(x, n_total=n, group=group, bits=4, e_long=el, e_short=es, debug=True)
    assert O.owner(0, 2, 2) == 0 and O.owner(1, 2, 2) == 1
    # stage 1, rank 1 -> owner 0, group 0: z = 0, s = 0.25, codes = i mod 16
    assert res.a2a_params[1, 0].tolist() == [0x3400, 0x0000]
    assert O.unpack_codes(res.a2a_codes[1, 0], 32, 4).tolist() == (i % 16).tolist()
    assert res.a2a_codes[1, 0].tolist() == [0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE] * 2
    # stage 1, rank 0 -> owner 1, group 1: 0..3.5 step 0.5 -> z = 0, s = RU(3.5/15)
    s1 = _h(res.a2a_params[0, 1])[0]
    assert s1 >= 3.5 / 15 and res.a2a_params[0, 1][1] == 0
    # stage 2, owner 0, group 0: sum 1 + (i mod 16)/4 -> z = 1, s = 0.25
    assert res.gather_params[0].tolist() == [0x3400, 0x3C00]
    assert O.unpack_codes(res.gather_codes[0], 32, 4).tolist() == (i % 16).tolist()
    assert np.array_equal(_f32(res.y[0, :32]), (1 + (i % 16) / 4.0).astype(np.float32))
    assert np.all(res.rho[:, :32] == 0)


def test_ema_closed_form():
    rng = np.random.default_rng(8)
    for alpha in [0.0, 0.05, 0.5, 1.0, 0.3]:
        T, m = 60, 64
        rho = rng.standard_normal((T, m)).astype(np.float32)
        e = np.zeros(m, np.float32)
        for t in range(T):
            O.ema_update(e, rho[t], alpha)
        # e_T = sum_t alpha (1-alpha)^(T-1-t) rho_t
        wts = alpha * (1 - alpha) ** np.arange(T - 1, -1, -1, dtype=np.float64)
        ref = (wts[:, None] * rho.astype(np.float64)).sum(axis=0)
        assert np.allclose(e, ref, rtol=0, atol=T * 2.0 ** -22 * (np.abs(rho).max() + 1))
        if alpha == 1.0:
            assert np.array_equal(e, rho[-1])
        if alpha == 0.0:
            assert np.all(e == 0)


def test_compensation_special_cases():
    rng = np.random.default_rng(9)
    for _ in range(200):
        el, es = (float(np.float32(v)) for v in rng.standard_normal(2))
        eta = float(np.float32(rng.uniform(0, 2)))
        assert O.compensation(el, es, eta, 1.0) == np.float32(eta) * np.float32(es)
        assert O.compensation(el, es, eta, 0.0) == np.float32(eta) * np.float32(el)
        assert O.compensation(el, es, 0.0, 0.5) == 0.0
        assert O.compensation(el, el, 1.0, 0.5) == np.float32(el)
        assert O.compensation(el, es, 1.0, 0.5) == np.float32(np.float64(el) / 2 + np.float64(es) / 2)


def test_payload_size_matches_four_bit_ceiling():
    with open(os.path.join(os.path.dirname(__file__), "golden", "page_numbers.json")) as f:
        pages = {e["name"]: e["value"] for e in json.load(f)["entries"]}
    P, group, n = 8, 128, 1 << 16
    G = n // group
    x = np.zeros((P, n), np.uint16)
    res = O.echo_allreduce(x, n_total=n, group=group, bits=4)
    bytes_per_group = res.a2a_codes.shape[2] + res.a2a_params.shape[2] * res.a2a_params.itemsize
    bits_per_element = 8 * bytes_per_group / group
    assert bits_per_element == 4.25
    assert round(16 / bits_per_element, 1) == pages["four_bit_ceiling"]
    assert res.gather_codes.shape == (G, 64)
    assert round(pages["sites_qwen3_0p6b"] / pages["bound_constant_eta1"]) == pages["ratio_at_56"]


def test_range_flag_is_raised_and_sticky():
    P, n = 2, 256
    x = np.zeros((P, n), np.uint16)
    x[0, 5] = W.bf16_bits(torch.tensor([1e6], dtype=torch.bfloat16))[0]
    res = O.echo_allreduce(x, n_total=n, group=128, bits=4)
    assert res.flags & O.FLAG_RANGE
    x[0, 5] = 0
    res = O.echo_allreduce(x, n_total=n, group=128, bits=4)
    assert res.flags == 0


def test_column_subset_equals_full_call():
    """Group columns are independent: a call on a column range reproduces the
    corresponding slice of the full call (used for sampled checks)."""
    rng = np.random.default_rng(12)
    P, group = 8, 128
    n = 50 * group - 17
    G = -(-n // group)
    x = np.zeros((P, G * group), np.uint16)
    x[:, :n] = _rand_bf16(rng, (P, n))
    el = (rng.standard_normal((P, G * group)) * 0.01).astype(np.float32)
    es = (rng.standard_normal((P, G * group)) * 0.01).astype(np.float32)
    el2, es2 = el.copy(), es.copy()
    full = O.echo_allreduce(x, n_total=n, group=group, bits=4, e_long=el, e_short=es)
    for j0, jc in [(0, 3), (5, 7), (G - 4, 4), (24, 2)]:
        sl = slice(j0 * group, (j0 + jc) * group)
        a, b = np.ascontiguousarray(el2[:, sl]), np.ascontiguousarray(es2[:, sl])
        part = O.echo_allreduce(np.ascontiguousarray(x[:, sl]), n_total=n, group=group, bits=4,
                                e_long=a, e_short=b, j0=j0, jc=jc)
        valid = np.arange(j0 * group, (j0 + jc) * group) < n
        assert np.array_equal(part.y[:, valid], full.y[:, sl][:, valid])
        assert np.array_equal(a[:, valid], el[:, sl][:, valid])
        assert np.array_equal(part.gather_codes, full.gather_codes[j0:j0 + jc])
        assert np.array_equal(part.a2a_params, full.a2a_params[:, j0:j0 + jc])
