"""Pins for chains of oracle calls (error feedback carried across sites).

Echo explainer, sections "Echoの仕組み②" (dual time-constant feedback) and
"理論保証" (theory): without compensation the per-site errors add up over the
N sites of a network; with the feedback (gain 1) the accumulated error stays
bounded independently of depth.

With R_j = sum_r rho_{j,r} the residual sum at site j and the feedback
c = eta * (w * e_short + (1 - w) * e_long), each EMA e <- (1-a) e + a rho, the
accumulated error after T sites, S_T = sum_t (y_t - sum_r x_{t,r}), has the
closed form (derived from the two recursions alone)

    S_T = sum_{j<T} R_j * [eta * (1 - w*(1-aS)^(T-1-j) - (1-w)*(1-aL)^(T-1-j)) - 1]

so with eta = 1 only the most recent residuals survive, and without state
S_T = -sum_j R_j grows like sqrt(T) * q for independent errors (T * q worst
case). These tests run the oracle on short synthetic chains and check the
closed form to round-off, the growth laws and the worst-case bound.
"""
import numpy as np
import pytest

import oracle as O
import workloads as W


def _f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def run_chain(w: W.Workload, feedback: bool, eta=1.0, wt=None, aL=None, aS=None):
    wt = w.w if wt is None else wt
    aL = w.alpha_long if aL is None else aL
    aS = w.alpha_short if aS is None else aS
    P, n = w.P, w.n
    el = np.zeros((P, n), np.float32) if feedback else None
    es = np.zeros((P, n), np.float32) if feedback else None
    x = W.inputs(w, 0)
    S = np.zeros(n)
    S_hist, R_hist = [], []
    for t in range(w.sites):
        xb = W.bf16_bits(x)
        res = O.echo_allreduce(xb, n_total=n, group=w.group, bits=w.bits_at(t), e_long=el,
                               e_short=es, eta=eta, alpha_long=aL, alpha_short=aS, w=wt,
                               debug=True)
        assert res.flags == 0
        S += _f64(res.y[0]) - _f64(xb).sum(axis=0)
        S_hist.append(S.copy())
        R_hist.append(res.rho.astype(np.float64).sum(axis=0))
        x = W.chain_next_input(W.from_bf16_bits(res.y[0]), W.chain_noise(w, t + 1), P, w.decay)
    return np.array(S_hist), np.array(R_hist)


def closed_form(R, eta, wt, aL, aS):
    T = R.shape[0]
    k = (T - 1) - np.arange(T)
    coef = eta * (1 - wt * (1 - aS) ** k - (1 - wt) * (1 - aL) ** k) - 1
    return (coef[:, None] * R).sum(axis=0)


SMALL56 = W.Workload("chain_small56", 60, P=4, tokens=16, hidden=1024, sites=56)


@pytest.mark.parametrize("wt,aL,aS", [(0.5, 0.05, 0.5), (0.3, 0.1, 0.7), (1.0, 0.05, 0.5)])
def test_accumulated_error_closed_form(wt, aL, aS):
    S, R = run_chain(SMALL56, True, 1.0, wt, aL, aS)
    Sc = closed_form(R, 1.0, wt, aL, aS)
    assert np.abs(S[-1] - Sc).max() <= 1e-4 * (1 + np.abs(S[-1]).max())
    # same identity after every prefix of the chain
    for T in (1, 7, 30):
        assert np.abs(S[T - 1] - closed_form(R[:T], 1.0, wt, aL, aS)).max() <= 1e-4 * (1 + np.abs(S[T - 1]).max())


def test_without_feedback_errors_add_up():
    S, R = run_chain(SMALL56, False)
    assert np.abs(S[-1] + R.sum(axis=0)).max() <= 1e-5 * (1 + np.abs(S[-1]).max())
    q = np.sqrt(np.mean(R ** 2))
    for T in (14, 56):
        ratio = np.sqrt(np.mean(S[T - 1] ** 2)) / q
        assert 0.7 * np.sqrt(T) <= ratio <= 1.3 * np.sqrt(T), (T, ratio)
    assert np.abs(S[-1]).max() <= 56 * np.abs(R).max()          # N*q worst case


def test_with_feedback_error_is_depth_independent():
    wl = SMALL56
    S, R = run_chain(wl, True)
    q = np.sqrt(np.mean(R ** 2))
    a, b, wt = 1 - wl.alpha_short, 1 - wl.alpha_long, wl.w
    k = np.arange(200)
    predicted = np.sqrt(np.sum((wt * a ** k + (1 - wt) * b ** k) ** 2))   # ~1.96 at these rates
    ratios = [np.sqrt(np.mean(S[T - 1] ** 2)) / q for T in (14, 28, 56)]
    for r in ratios:
        assert 0.7 * predicted <= r <= 1.3 * predicted, (ratios, predicted)
    assert max(ratios) / min(ratios) < 1.3
    # worst case: |S_T| <= (w / aS + (1 - w) / aL) * max|R|  (11 q_max here)
    bound = (wt / wl.alpha_short + (1 - wt) / wl.alpha_long) * np.abs(R).max()
    assert np.abs(S).max() <= bound
    # and it is much smaller than the uncompensated chain at the same depth
    S0, R0 = run_chain(wl, False)
    assert np.sqrt(np.mean(S0[-1] ** 2)) > 2.5 * np.sqrt(np.mean(S[-1] ** 2))


def test_mixed_precision_chain_carries_state():
    wl = W.Workload("chain_small_mixed", 61, P=4, tokens=8, hidden=1280, sites=24, int8_sites=6)
    S, R = run_chain(wl, True)
    q8 = np.sqrt(np.mean(R[:6] ** 2))
    q4 = np.sqrt(np.mean(R[6:] ** 2))
    assert q8 * 8 < q4                                   # 8-bit sites inject far less error
    Sc = closed_form(R, 1.0, wl.w, wl.alpha_long, wl.alpha_short)
    assert np.abs(S[-1] - Sc).max() <= 1e-4 * (1 + np.abs(S[-1]).max())
