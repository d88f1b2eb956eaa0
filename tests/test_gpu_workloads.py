"""GPU <-> oracle parity on the full-size workloads.

Group columns (all ranks' group j plus their state) are independent, so the
oracle is run on sampled column ranges -- the first and last columns, every
owner boundary and the middle -- while the GPU runs the full message. Chains
carry the EMA state from site to site on both sides; each side builds its next
input from its own output with the same noise.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
import bit_error_compensated_group_b200 as E
from parity import assert_state_close, column_ranges, u16

pytestmark = pytest.mark.gpu


class Sampled:
    """Oracle state for a set of sampled column ranges."""

    def __init__(self, w: W.Workload, width: int, feedback: bool = True):
        self.w = w
        self.G = -(-w.n // w.group)
        self.ranges = column_ranges(self.G, w.P, width)
        self.el, self.es = {}, {}
        for (j0, jc) in self.ranges:
            ld = jc * w.group
            self.el[j0] = np.zeros((w.P, ld), np.float32) if feedback else None
            self.es[j0] = np.zeros((w.P, ld), np.float32) if feedback else None

    def cols(self, j0, jc):
        g = self.w.group
        return slice(j0 * g, min(self.w.n, (j0 + jc) * g))

    def padded_slice(self, xfull_u16, j0, jc):
        """[P][jc*group] uint16 slice of a [P][n] uint16 array (zero past n)."""
        c = self.cols(j0, jc)
        out = np.zeros((self.w.P, jc * self.w.group), np.uint16)
        out[:, :c.stop - c.start] = xfull_u16[:, c]
        return out


def _gpu_inputs_u16(inputs, c):
    return np.stack([u16(t[c]) for t in inputs])


def _compare_sampled(ar, outputs, S: Sampled, orcs, bits, site):
    a2a_c, a2a_p, g_c, g_p = ar.payload_views(bits)
    el_v, es_v = ar.ema_views() if ar.state is not None else (None, None)
    w = S.w
    for (j0, jc), orc in zip(S.ranges, orcs):
        c = S.cols(j0, jc)
        m = c.stop - c.start
        got_y = np.stack([u16(o[c]) for o in outputs])
        assert np.array_equal(got_y, orc.y[:, :m]), f"site {site}: outputs differ in columns {j0}+{jc}"
        gc = g_c[j0:j0 + jc].cpu().numpy()
        gp = g_p[j0:j0 + jc].cpu().numpy().view(np.uint16).reshape(jc, 2)
        assert np.array_equal(gc, orc.gather_codes) and np.array_equal(gp, orc.gather_params), f"site {site}"
        ac = a2a_c[:, j0:j0 + jc].cpu().numpy()
        ap = a2a_p[:, j0:j0 + jc].cpu().numpy().view(np.uint16).reshape(w.P, jc, 2)
        for jl in range(jc):
            o = O.owner(j0 + jl, S.G, w.P)
            for r in range(w.P):
                if r != o:
                    assert np.array_equal(ac[r, jl], orc.a2a_codes[r, jl]), f"site {site} a2a r={r} j={j0 + jl}"
                    assert np.array_equal(ap[r, jl], orc.a2a_params[r, jl]), f"site {site} a2a r={r} j={j0 + jl}"
        if S.el[j0] is not None:
            assert_state_close(el_v[:, c].cpu().numpy(), S.el[j0][:, :m], f"site {site} e_long")
            assert_state_close(es_v[:, c].cpu().numpy(), S.es[j0][:, :m], f"site {site} e_short")


def _oracle_step(S: Sampled, x_by_range, bits, quantizer=O.Q_DIRECTED):
    w = S.w
    out = []
    for (j0, jc) in S.ranges:
        out.append(O.echo_allreduce(x_by_range[j0], n_total=w.n, group=w.group, bits=bits,
                                    e_long=S.el[j0], e_short=S.es[j0], eta=w.eta, alpha_long=w.alpha_long,
                                    alpha_short=w.alpha_short, w=w.w, j0=j0, jc=jc, quantizer=quantizer))
    return out


def run_chain(w: W.Workload, feedback: bool, width: int = 32, quantizer: int = O.Q_DIRECTED):
    """Full chain on the GPU, sampled chain on the oracle, compared per site.
    Returns the GPU's accumulated error S_T = sum_t (y_t - sum_r x_t,r)."""
    P, n = w.P, w.n
    ar = E.EchoAllReduce(n, P, w.group, 8 if w.int8_sites else 4, feedback, quantizer=quantizer)
    S = Sampled(w, width, feedback)
    x_cpu = W.inputs(w, 0)
    inputs = [x_cpu[r].cuda() for r in range(P)]
    outputs = [torch.empty_like(t) for t in inputs]
    x_orc = {j0: S.padded_slice(u16(x_cpu), j0, jc) for (j0, jc) in S.ranges}
    acc_err = torch.zeros(n, dtype=torch.float64, device="cuda")
    try:
        for t in range(w.sites):
            bits = w.bits_at(t)
            ar(inputs, outputs, bits, w.eta, w.alpha_long, w.alpha_short, w.w)
            orcs = _oracle_step(S, x_orc, bits, quantizer)
            rc, flags = ar.status()
            assert rc == E.ECHO_OK and all(o.flags == 0 for o in orcs)
            _compare_sampled(ar, outputs, S, orcs, bits, t)
            xs = torch.stack([i.double() for i in inputs]).sum(0)
            acc_err += outputs[0].double() - xs
            # next site: each side from its own output, same noise
            noise = W.chain_noise(w, t + 1)
            x_next = W.chain_next_input(outputs[0], noise, P, w.decay)
            for r in range(P):
                inputs[r].copy_(x_next[r])
            for (j0, jc), orc in zip(S.ranges, orcs):
                c = S.cols(j0, jc)
                m = c.stop - c.start
                y_o = W.from_bf16_bits(orc.y[0, :m])
                xn = W.chain_next_input(y_o, noise[:, c], P, w.decay)
                x_orc[j0] = np.zeros((P, jc * w.group), np.uint16)
                x_orc[j0][:, :m] = u16(xn)
        return acc_err.cpu().numpy()
    finally:
        ar.close()


def test_chain_56_sites_p8():
    w = W.CHAIN56
    with_fb = run_chain(w, True)
    without = run_chain(w, False)
    rms_fb = float(np.sqrt(np.mean(with_fb ** 2)))
    rms_no = float(np.sqrt(np.mean(without ** 2)))
    # the explainer's theory section: bounded with feedback, growing without
    assert rms_no > 2.5 * rms_fb, (rms_no, rms_fb)


def test_chain_ablation_quantizer_forms():
    """The ablation of the quantizer form on the 56-site chain (P = 8): each
    form, with and without feedback, run in full on the GPU and checked site
    by site against the oracle on sampled columns. Reported: RMS of the
    accumulated error S_T over the last site, in units of q, the RMS per-site
    error of the default form without feedback. Feedback keeps S_T bounded
    for every form (the explainer's theory section)."""
    w = W.CHAIN56
    res = {}
    for q in (O.Q_DIRECTED, O.Q_NEAREST, O.Q_INT_ZERO):
        for fb in (True, False):
            res[(q, fb)] = float(np.sqrt(np.mean(run_chain(w, fb, width=16, quantizer=q) ** 2)))
    names = {O.Q_DIRECTED: "directed", O.Q_NEAREST: "nearest", O.Q_INT_ZERO: "int_zero"}
    print("\nablation RMS(S_56):", {f"{names[q]}/{'fb' if fb else 'nofb'}": round(v, 5) for (q, fb), v in res.items()})
    for q in names:
        assert res[(q, False)] > 2.5 * res[(q, True)], (names[q], res[(q, False)], res[(q, True)])


def test_chain_48_sites_p4_early_int8():
    w = W.CHAIN48_MIXED
    run_chain(w, True)


@pytest.mark.parametrize("feedback,bits", [(True, 4), (False, 4), (True, 8)])
def test_headline_1gb_sampled_columns(feedback, bits):
    """P = 8, 1 GB per rank, two calls (state carried when there is one), in
    the launch sequences the benchmark times: first one echo_allreduce_sim
    call (its headline steps: the owners' pass a programmatic dependent of
    the quantize pass), then the two phase entry points (its per-kernel
    pass). The early-site 8-bit mode on the same message too."""
    w = W.HEADLINE
    P, n = w.P, w.n
    free, _ = torch.cuda.mem_get_info()
    if free < 65e9:
        pytest.skip("needs ~60 GB of free device memory")
    ar = E.EchoAllReduce(n, P, w.group, bits, feedback)
    S = Sampled(w, 256, feedback)
    try:
        inputs = [W.rank_input(w, r, 0, "cuda") for r in range(P)]
        outputs = [torch.empty_like(t) for t in inputs]
        x_orc = {}
        for (j0, jc) in S.ranges:
            c = S.cols(j0, jc)
            x_orc[j0] = np.zeros((P, jc * w.group), np.uint16)
            x_orc[j0][:, :c.stop - c.start] = _gpu_inputs_u16(inputs, c)
        fb = (w.eta, w.alpha_long, w.alpha_short, w.w)
        for call in range(2):
            if call == 0:
                E.echo_allreduce_sim(inputs, outputs, ar.handle, n, P, bits, w.group, *fb)
            else:
                E.echo_phase_quantize(inputs, ar.handle, bits, *fb)
                E.echo_phase_reduce(inputs, outputs, ar.handle, bits, *fb)
            orcs = _oracle_step(S, x_orc, bits)
            rc, flags = ar.status()
            assert rc == E.ECHO_OK
            _compare_sampled(ar, outputs, S, orcs, bits, call)
        # properties over the whole message: every rank holds the same result
        for r in range(1, P):
            assert torch.equal(outputs[r].view(torch.int16), outputs[0].view(torch.int16))
    finally:
        ar.close()
        torch.cuda.empty_cache()
