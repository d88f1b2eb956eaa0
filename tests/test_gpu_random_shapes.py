"""Seeded random shapes and parameters against the oracle, through the C ABI.

Each case draws P (1-64), n (1 to ~200 k elements per rank, so ragged tails
and G < P occur), the group size, the bit width, the quantizer form, whether
there is feedback state, and eta / alpha_long / alpha_short / w; inputs are
scaled normal values. The simulation runs two calls with carried state and
must match the oracle bit for bit (check_full_call); the rank mode (P up to
16, exchanges in-process) likewise.
"""
import numpy as np
import pytest
import torch

import oracle as O
import bit_error_compensated_group_b200 as E
from parity import Params, check_full_call, padded, random_inputs, seeded_state, u16

pytestmark = pytest.mark.gpu


def _draw(seed, max_p):
    rng = np.random.default_rng(seed)
    P = int(rng.choice([1, 2, 3, 4, 5, 7, 8, 12, 16, 31, 64][: 9 if max_p <= 16 else 11]))
    n = int(rng.integers(1, 200_000))
    group = int(rng.choice([32, 64, 128, 256]))
    bits = int(rng.choice([4, 8]))
    quantizer = int(rng.choice([O.Q_DIRECTED, O.Q_NEAREST, O.Q_INT_ZERO]))
    feedback = bool(rng.integers(0, 2))
    eta = float(rng.choice([0.0, 0.5, 1.0, 1.5]))
    aL, aS, w = (float(v) for v in rng.uniform(0.0, 1.0, 3))
    scale = float(rng.choice([0.01, 1.0, 30.0]))
    return P, n, group, bits, quantizer, feedback, eta, aL, aS, w, scale


@pytest.mark.parametrize("seed", range(24))
def test_simulation_random(seed):
    P, n, group, bits, quantizer, feedback, eta, aL, aS, w, scale = _draw(1000 + seed, 64)
    p = Params(bits=bits, group=group, eta=eta, alpha_long=aL, alpha_short=aS, w=w, quantizer=quantizer)
    x = random_inputs(P, n, 7 * seed + 1, scale)
    el0, es0 = seeded_state(P, n, seed + 99, 0.05 * scale) if feedback else (None, None)
    check_full_call(P, n, p, x, el0, es0, feedback, calls=2)


@pytest.mark.parametrize("seed", range(12))
def test_ranks_random(seed):
    P, n, group, bits, quantizer, feedback, eta, aL, aS, w, scale = _draw(2000 + seed, 16)
    fb = (eta, aL, aS, w)
    G = -(-n // group)
    ld = G * group
    ranks = [E.EchoRank(n, P, r, group, max(bits, 4), feedback, quantizer=quantizer) for r in range(P)]
    try:
        x = random_inputs(P, n, 11 * seed + 3, scale)
        xs = [x[r].cuda() for r in range(P)]
        outs = [torch.empty_like(t) for t in xs]
        el = es = None
        if feedback:
            el0, es0 = seeded_state(P, n, seed + 7, 0.05 * scale)
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
            E.exchange_in_process(plans, "all_to_all")
            for r in range(P):
                ranks[r].reduce(xs[r], outs[r], bits, *fb)
            E.exchange_in_process(plans, "all_gather")
            for r in range(P):
                ranks[r].decode(outs[r], bits)
            orc = O.echo_allreduce(xb, n_total=n, group=group, bits=bits, e_long=el, e_short=es, eta=eta,
                                   alpha_long=aL, alpha_short=aS, w=w, quantizer=quantizer)
            flags = 0
            for rk in ranks:
                flags |= rk.status()[1]
            assert flags == orc.flags
            for r in range(P):
                assert np.array_equal(u16(outs[r]), orc.y[r, :n]), f"call {call}: output of rank {r}"
                if feedback:
                    L, S = ranks[r].ema_views()
                    assert np.array_equal(L.cpu().numpy(), el[r, :n]) and np.array_equal(S.cpu().numpy(), es[r, :n])
            xs = [o.clone() for o in outs]
            xb = padded(orc.y[:, :n].copy(), ld)
    finally:
        for rk in ranks:
            rk.close()
