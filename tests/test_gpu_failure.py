"""Failure detection on the GPU without a GPU fault.

The bulk-copy pipelines bound every device-side wait. This test makes such a
wait run out -- one thread waits on a barrier that nothing ever completes --
and checks that the expiry reaches the host as ECHO_ETIMEOUT, that reading the
status clears it, and that the context is still usable: a normal call right
after matches the oracle.
"""
import time

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
import bit_error_compensated_group_b200 as E
from parity import GpuEcho, Params, padded, u16

pytestmark = pytest.mark.gpu


def test_expired_wait_reports_timeout_and_context_survives():
    w = W.TINY
    gpu = GpuEcho(w.P, w.n)
    try:
        t0 = time.perf_counter()
        E.echo_check_watchdog(gpu.ar.handle, 200_000)          # 0.2 s
        rc, flags = gpu.status()
        waited = time.perf_counter() - t0
        assert rc == E.ECHO_ETIMEOUT and flags & E.ECHO_FLAG_TIMEOUT
        assert 0.15 < waited < 5.0
        rc, flags = gpu.status()
        assert rc == E.ECHO_OK and flags == 0
        # the context still works: one ordinary call, checked against the oracle
        x = W.inputs(w)
        gpu.set_inputs(x)
        gpu.call(Params())
        rc, flags = gpu.status()
        assert rc == E.ECHO_OK
        G = -(-w.n // 128)
        ref = O.echo_allreduce(padded(u16(x), G * 128), n_total=w.n, group=128, bits=4,
                               e_long=np.zeros((w.P, G * 128), np.float32),
                               e_short=np.zeros((w.P, G * 128), np.float32))
        assert np.array_equal(gpu.outputs_u16(), ref.y[:, :w.n])
    finally:
        gpu.close()


def test_watchdog_argument_checks():
    w = W.TINY
    gpu = GpuEcho(w.P, w.n)
    try:
        for bad in (0, 10_000_001):
            with pytest.raises(E.EchoError) as ei:
                E.echo_check_watchdog(gpu.ar.handle, bad)
            assert ei.value.status == E.ECHO_EINVAL
    finally:
        gpu.close()
