"""GPU <-> oracle parity of the CUDA path, called through the C ABI.

Bar: packed codes, fp16 parameters and bf16 outputs bit-identical; EMA state
within 1e-6 relative (1e-7 absolute near zero). Sizes span many kernel tiles
and ragged tails; the 1 GB workload is checked on sampled group columns
(columns are independent), in the launch configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
import bit_error_compensated_group_b200 as E
from parity import (GpuEcho, Params, assert_payload_equal, assert_state_close, column_ranges, padded, u16,
                    check_full_call as _check_full_call, random_inputs as _random_inputs,
                    seeded_state as _seeded_state)

pytestmark = pytest.mark.gpu


def test_tiny_workload():
    w = W.TINY
    _check_full_call(w.P, w.n, Params(), W.inputs(w))


CASES = [
    # P, n, group, bits
    (1, 1000, 128, 4),
    (2, 4096, 128, 4),
    (3, 1000, 32, 4),
    (4, 777, 64, 8),
    (8, 8192, 128, 4),
    (8, 1000, 128, 4),          # G == P, partial last group
    (16, 3000, 128, 4),         # G < P: empty segments
    (5, 3 * 2048 + 5, 256, 8),
    (64, 3 * 64 * 128 + 17, 128, 4),   # largest P
    (3, 148 * 8 * 256 * 3 + 37, 128, 4),  # several passes of the persistent grid
    (2, 1, 32, 4),              # a single element
    (7, 333333, 64, 8),
]


@pytest.mark.parametrize("P,n,group,bits", CASES)
@pytest.mark.parametrize("feedback", [True, False])
def test_parity_odd_shapes(P, n, group, bits, feedback):
    x = _random_inputs(P, n, P * 7919 + n, 2.0)
    el0, es0 = _seeded_state(P, n, n + P) if feedback else (None, None)
    _check_full_call(P, n, Params(bits=bits, group=group, w=0.3, alpha_long=0.1, alpha_short=0.6), x,
                     el0, es0, feedback, calls=2)


def test_tp_shape_with_outliers_two_calls():
    w = W.TP8B
    _check_full_call(w.P, w.n, Params(), W.inputs(w), calls=2)


def test_phase_entry_points_compose():
    """echo_phase_quantize alone produces the all-to-all payload and the
    non-owned EMAs; the three phases in order equal echo_allreduce_sim."""
    P, n, p = 4, 10000, Params()
    G = -(-n // 128)
    x = _random_inputs(P, n, 5)
    el0, es0 = _seeded_state(P, n, 6)
    gpu = GpuEcho(P, n)
    try:
        gpu.set_inputs(x)
        gpu.set_state(el0, es0)
        h = gpu.ar.handle
        E.echo_phase_quantize(gpu.inputs, h, 4, p.eta, p.alpha_long, p.alpha_short, p.w)
        el, es = padded(el0, G * 128), padded(es0, G * 128)
        orc = O.echo_allreduce(padded(u16(x), G * 128), n_total=n, group=128, bits=4, e_long=el, e_short=es)
        a2a_c, a2a_p, _, _ = gpu.payload(4)
        gl, gs = gpu.state()
        for j in range(G):
            o = O.owner(j, G, P)
            cols = slice(j * 128, min(n, (j + 1) * 128))
            for r in range(P):
                if r == o:
                    assert np.array_equal(gl[r, cols], el0[r, cols])      # owner state untouched
                    continue
                assert np.array_equal(a2a_c[r, j], orc.a2a_codes[r, j])
                assert np.array_equal(a2a_p[r, j], orc.a2a_params[r, j])
                assert np.array_equal(gl[r, cols], el[r, cols]) and np.array_equal(gs[r, cols], es[r, cols])
        E.echo_phase_reduce(gpu.inputs, None, h, 4, p.eta, p.alpha_long, p.alpha_short, p.w)
        E.echo_phase_gather(gpu.outputs, h, 4)
        assert np.array_equal(gpu.outputs_u16(), orc.y[:, :n])
        gl, gs = gpu.state()
        assert np.array_equal(gl, el[:, :n]) and np.array_equal(gs, es[:, :n])
    finally:
        gpu.close()


@pytest.mark.parametrize("P,n,group,bits", [(4, 10000, 128, 4), (3, 5000 + 11, 32, 8), (8, 1 << 18, 128, 4)])
def test_reduce_with_outputs_equals_reduce_then_gather(P, n, group, bits):
    """Phase 4 in the owner's pass (echo_phase_reduce given outputs) writes
    exactly what decoding the all-gather payload afterwards writes."""
    x = _random_inputs(P, n, 40 + P)
    el0, es0 = _seeded_state(P, n, 41 + P)
    fb = (1.0, 0.05, 0.5, 0.5)
    outs = []
    for fused in (False, True):
        gpu = GpuEcho(P, n, group, bits)
        try:
            gpu.set_inputs(x)
            gpu.set_state(el0, es0)
            h = gpu.ar.handle
            E.echo_phase_quantize(gpu.inputs, h, bits, *fb)
            if fused:
                E.echo_phase_reduce(gpu.inputs, gpu.outputs, h, bits, *fb)
            else:
                E.echo_phase_reduce(gpu.inputs, None, h, bits, *fb)
                E.echo_phase_gather(gpu.outputs, h, bits)
            outs.append((gpu.outputs_u16(), *gpu.state(), *gpu.payload(bits)[2:]))
        finally:
            gpu.close()
    for a, b in zip(*outs):
        assert np.array_equal(a, b)


def test_in_place_outputs():
    P, n = 4, 50000
    x = _random_inputs(P, n, 9)
    G = -(-n // 128)
    gpu = GpuEcho(P, n)
    try:
        gpu.set_inputs(x)
        E.echo_allreduce_sim(gpu.inputs, gpu.inputs, gpu.ar.handle, n, P, 4, 128, 1.0, 0.05, 0.5, 0.5)
        orc = O.echo_allreduce(padded(u16(x), G * 128), n_total=n, group=128, bits=4,
                               e_long=np.zeros((P, G * 128), np.float32), e_short=np.zeros((P, G * 128), np.float32))
        assert np.array_equal(np.stack([u16(t) for t in gpu.inputs]), orc.y[:, :n])
    finally:
        gpu.close()


@pytest.mark.parametrize("feedback", [True, False])
@pytest.mark.parametrize("bad", [1e6, -1e6, float("nan"), float("-inf")])
@pytest.mark.parametrize("rank", [0, 1])
def test_range_flag_and_recovery(feedback, bad, rank):
    """A value outside the fp16 parameter range (or a NaN) raises the sticky
    flag, from a non-owned group (rank 1: the quantize pass) or an owned one
    (rank 0: the owner's sum); echo_get_status reports and clears it. The EMAs
    of a flagged group are unspecified, so the recovery call starts from fresh
    state."""
    P, n = 2, 4096
    x = _random_inputs(P, n, 10)
    x[rank, 1234] = bad
    gpu = GpuEcho(P, n, feedback=feedback)
    try:
        gpu.set_inputs(x)
        gpu.call(Params())
        rc, flags = gpu.status()
        assert rc == E.ECHO_ERANGE and flags & E.ECHO_FLAG_RANGE
        rc, flags = gpu.status()                     # cleared by the read
        assert rc == E.ECHO_OK and flags == 0
        x[rank, 1234] = 0.5
        gpu.set_inputs(x)
        if feedback:
            gpu.set_state(np.zeros((P, n), np.float32), np.zeros((P, n), np.float32))
        gpu.call(Params())
        rc, flags = gpu.status()
        assert rc == E.ECHO_OK and flags == 0
    finally:
        gpu.close()


def test_bad_arguments_on_device():
    P, n = 2, 4096
    gpu = GpuEcho(P, n)
    try:
        h = gpu.ar.handle
        with pytest.raises(E.EchoError) as ei:     # bits above the handle's max_bits
            E.echo_allreduce_sim(gpu.inputs, gpu.outputs, h, n, P, 8, 128, 1.0, 0.05, 0.5, 0.5)
        assert ei.value.status == E.ECHO_EINVAL
        with pytest.raises(E.EchoError):            # n differs from the handle
            E.echo_allreduce_sim(gpu.inputs, gpu.outputs, h, n + 1, P, 4, 128, 1.0, 0.05, 0.5, 0.5)
        with pytest.raises(E.EchoError):            # misaligned input pointer
            bad = [gpu.inputs[0].data_ptr() + 2, gpu.inputs[1].data_ptr()]
            E.echo_allreduce_sim(bad, gpu.outputs, h, n, P, 4, 128, 1.0, 0.05, 0.5, 0.5)
        with pytest.raises(E.EchoError):            # alpha outside [0, 1]
            E.echo_allreduce_sim(gpu.inputs, gpu.outputs, h, n, P, 4, 128, 1.0, 1.5, 0.5, 0.5)
    finally:
        gpu.close()


def test_deterministic():
    P, n = 8, 1 << 20
    x = _random_inputs(P, n, 11)
    outs = []
    for _ in range(2):
        gpu = GpuEcho(P, n)
        try:
            gpu.set_inputs(x)
            gpu.call(Params())
            gpu.call(Params())
            outs.append((gpu.outputs_u16(), *gpu.state()))
        finally:
            gpu.close()
    for a, b in zip(*outs):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("P,n,group,bits", [(6, 5000, 32, 8), (2, 4096, 128, 8), (9, 70001, 128, 8), (3, 2 * 2048 * 5 + 300, 256, 4)])
def test_parity_more_shapes(P, n, group, bits):
    x = _random_inputs(P, n, 31 * P + n, 1.0)
    el0, es0 = _seeded_state(P, n, n + 3 * P)
    _check_full_call(P, n, Params(bits=bits, group=group), x, el0, es0, True, calls=2)


@pytest.mark.parametrize("eta,w,aL,aS", [(0.0, 0.5, 0.05, 0.5), (1.5, 0.0, 1.0, 0.0), (0.5, 1.0, 0.0, 1.0), (1.0, 0.25, 0.3, 0.9)])
def test_parity_feedback_parameters(eta, w, aL, aS):
    P, n = 4, 3 * 4096 + 77
    x = _random_inputs(P, n, 17, 1.5)
    el0, es0 = _seeded_state(P, n, 18, scale=0.2)
    _check_full_call(P, n, Params(eta=eta, w=w, alpha_long=aL, alpha_short=aS), x, el0, es0, True, calls=3)


def test_parity_special_values():
    """Groups that are constant (s = 0: every code 0), all zero, holding -0,
    bf16 subnormals, or values close to the fp16 edge after the sum."""
    P, n, group = 4, 64 * 128, 128
    g = torch.Generator().manual_seed(21)
    x = torch.randn(P, n, generator=g)
    x[:, 0:128] = 0.0                                   # all-zero group on every rank
    x[:, 128:256] = -0.0                                # negative zeros
    x[0, 256:384] = 3.25                                # constant on one rank
    x[:, 384:512] = 1.5                                 # constant on every rank (sum exact)
    x[1, 512:640] = torch.randn(128, generator=g) * 1e-39   # bf16 subnormals
    x[:, 640:768] = 16000.0 + torch.randn(P, 128, generator=g)  # sum near 64000 < 65504
    x[2, 768:896] = -3.0e4                              # large negative on one rank
    x[:, 896:900] = torch.tensor([1e-30, -1e-30, 2e-38, -2e-38])
    xb = x.to(torch.bfloat16)
    for feedback in (True, False):
        el0, es0 = (np.zeros((P, n), np.float32), np.zeros((P, n), np.float32)) if feedback else (None, None)
        _check_full_call(P, n, Params(), xb, el0, es0, feedback, calls=2)
