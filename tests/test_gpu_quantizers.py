"""GPU <-> oracle parity for the quantizer forms of the ablations.

The Echo explainer's mechanism-1 section names an asymmetric zero-point
quantizer with half-precision parameters; the library offers, besides the
default form (fp16 zero rounded down, step rounded up), the zero and step
rounded to nearest, and an integer zero point (echo_set_quantizer). Each form
is compared bit for bit with the oracle: codes, parameter words, outputs, and
EMA state, over two calls with the state carried.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
import bit_error_compensated_group_b200 as E
from parity import GpuEcho, Params, check_full_call, random_inputs, seeded_state

pytestmark = pytest.mark.gpu

FORMS = [E.ECHO_QUANT_NEAREST, E.ECHO_QUANT_INT_ZERO]

CASES = [
    # P, n, group, bits
    (2, 4096, 128, 4),
    (3, 1000, 32, 4),
    (4, 777, 64, 8),
    (8, 8192, 128, 4),
    (8, 1000, 128, 4),          # G == P, partial last group
    (16, 3000, 128, 4),         # G < P: empty segments
    (5, 3 * 2048 + 5, 256, 8),
    (9, 70001, 128, 8),         # more ranks than one payload batch at 8 bits
    (3, 148 * 8 * 256 * 3 + 37, 128, 4),  # several passes of the persistent grid
    (2, 1, 32, 4),              # a single element
    (1, 5000, 128, 4),          # nothing is quantized
]


def test_library_and_oracle_number_the_forms_alike():
    assert (E.ECHO_QUANT_DIRECTED, E.ECHO_QUANT_NEAREST, E.ECHO_QUANT_INT_ZERO) == \
        (O.Q_DIRECTED, O.Q_NEAREST, O.Q_INT_ZERO)


@pytest.mark.parametrize("quantizer", FORMS)
@pytest.mark.parametrize("P,n,group,bits", CASES)
@pytest.mark.parametrize("feedback", [True, False])
def test_parity_shapes(quantizer, P, n, group, bits, feedback):
    x = random_inputs(P, n, P * 131 + n + quantizer, 2.0)
    el0, es0 = seeded_state(P, n, n + 3 * P + quantizer) if feedback else (None, None)
    check_full_call(P, n, Params(bits=bits, group=group, w=0.3, alpha_long=0.1, alpha_short=0.6,
                                 quantizer=quantizer), x, el0, es0, feedback, calls=2)


@pytest.mark.parametrize("quantizer", FORMS)
def test_parity_tp_shape_with_outliers(quantizer):
    w = W.TP8B
    check_full_call(w.P, w.n, Params(quantizer=quantizer), W.inputs(w), calls=2)


@pytest.mark.parametrize("quantizer", FORMS)
@pytest.mark.parametrize("bits", [4, 8])
def test_parity_special_values(quantizer, bits):
    """Groups that are constant, all zero, hold -0 or bf16 subnormals, lie all
    above or all below zero, ramp through zero, or sum where the binary16
    spacing is coarse (the owner's binary32 sums there make the nearest form's
    zero round above the minimum, which its clamp handles) or near the fp16
    edge."""
    P, n = 4, 64 * 128
    g = torch.Generator().manual_seed(31 + bits)
    x = torch.randn(P, n, generator=g)
    x[:, 0:128] = 0.0
    x[:, 128:256] = -0.0
    x[0, 256:384] = 3.25
    x[:, 384:512] = 1.5
    x[1, 512:640] = torch.randn(128, generator=g) * 1e-39
    x[:, 640:768] = 16000.0 + torch.randn(P, 128, generator=g)
    x[2, 768:896] = -3.0e4
    x[:, 896:900] = torch.tensor([1e-30, -1e-30, 2e-38, -2e-38])
    x[:, 1024:1152] = 5.0 + torch.rand(P, 128, generator=g)             # all positive
    x[:, 1152:1280] = -5.0 - torch.rand(P, 128, generator=g)            # all negative
    x[0, 1280:1408] = 30000.0 + 1000.0 * torch.rand(128, generator=g)    # sums where fp16 spacing is 16
    x[3, 1408:1536] = 4.0 * torch.arange(128) / 127.0 - 1.0              # a ramp through 0
    xb = x.to(torch.bfloat16)
    for feedback in (True, False):
        el0, es0 = (np.zeros((P, n), np.float32), np.zeros((P, n), np.float32)) if feedback else (None, None)
        check_full_call(P, n, Params(bits=bits, quantizer=quantizer), xb, el0, es0, feedback, calls=2)


def test_set_quantizer_switches_between_calls():
    """One handle, the form changed between calls: each call matches the
    oracle run with the form in force at that call."""
    P, n = 4, 5000
    x = random_inputs(P, n, 77, 1.0)
    gpu = GpuEcho(P, n)
    try:
        gpu.set_inputs(x)
        from parity import u16
        xb = u16(x)
        for q in (E.ECHO_QUANT_INT_ZERO, E.ECHO_QUANT_DIRECTED, E.ECHO_QUANT_NEAREST):
            E.echo_set_quantizer(gpu.ar.handle, q)
            gpu.set_state(np.zeros((P, n), np.float32), np.zeros((P, n), np.float32))
            gpu.call(Params())
            G = -(-n // 128)
            xp = np.zeros((P, G * 128), np.uint16)
            xp[:, :n] = xb
            orc = O.echo_allreduce(xp, n_total=n, group=128, bits=4, e_long=np.zeros((P, G * 128), np.float32),
                                   e_short=np.zeros((P, G * 128), np.float32), quantizer=q)
            assert np.array_equal(gpu.outputs_u16(), orc.y[:, :n]), q
    finally:
        gpu.close()


def test_set_quantizer_rejects_unknown_forms():
    gpu = GpuEcho(2, 256)
    try:
        with pytest.raises(E.EchoError):
            E.echo_set_quantizer(gpu.ar.handle, 3)
        with pytest.raises(E.EchoError):
            E.echo_set_quantizer(gpu.ar.handle, -1)
    finally:
        gpu.close()
