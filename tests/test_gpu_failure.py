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
        with pytest.raises(E.EchoError) as ei:
            E.echo_check_watchdog(gpu.ar.handle, 10_000_001)
        assert ei.value.status == E.ECHO_EINVAL
        h = gpu.ar.handle
        assert E.echo_get_wait_limit(h) == 1_000_000          # default: 1 s
        for bad in (0, 999, 60_000_001):
            with pytest.raises(E.EchoError) as ei:
                E.echo_set_wait_limit(h, bad)
            assert ei.value.status == E.ECHO_EINVAL
        assert E.echo_get_wait_limit(h) == 1_000_000          # unchanged by a refused setting
    finally:
        gpu.close()


def test_handle_wait_limit_reaches_the_kernels():
    """The handle's wait limit is what a kernel's bounded wait uses: the
    watchdog with limit 0 waits for the handle's setting (0.2 s here, then
    0.6 s), and ordinary calls under a short limit still run correctly."""
    w = W.TINY
    gpu = GpuEcho(w.P, w.n)
    try:
        h = gpu.ar.handle
        for limit_us, lo, hi in ((200_000, 0.15, 0.55), (600_000, 0.55, 5.0)):
            E.echo_set_wait_limit(h, limit_us)
            assert E.echo_get_wait_limit(h) == limit_us
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            E.echo_check_watchdog(h, 0)
            rc, flags = gpu.status()
            waited = time.perf_counter() - t0
            assert rc == E.ECHO_ETIMEOUT and flags & E.ECHO_FLAG_TIMEOUT
            assert lo < waited < hi, (limit_us, waited)
        # a 50 ms limit is far above any wait of this small call
        E.echo_set_wait_limit(h, 50_000)
        x = W.inputs(w)
        gpu.set_inputs(x)
        G = -(-w.n // 128)
        el = np.zeros((w.P, G * 128), np.float32)
        es = np.zeros((w.P, G * 128), np.float32)
        for _ in range(2):
            gpu.call(Params())
            ref = O.echo_allreduce(padded(u16(x), G * 128), n_total=w.n, group=128, bits=4, e_long=el, e_short=es)
            assert gpu.status() == (E.ECHO_OK, 0)
            assert np.array_equal(gpu.outputs_u16(), ref.y[:, :w.n])
    finally:
        gpu.close()


def test_injected_launch_failures_reach_the_caller():
    """With the host hook on, every entry point that launches a kernel returns
    ECHO_ECUDA (raised as EchoError); nothing fails on the GPU, and with the
    hook off the next call is correct."""
    import numpy as np
    import oracle as O
    from parity import padded, random_inputs, u16
    P, n = 4, 10000
    G = -(-n // 128)
    x = random_inputs(P, n, 21)
    ar = E.EchoAllReduce(n, P)
    rk = E.EchoRank(n, 1, 0)
    rk2 = E.EchoRank(n, 2, 0)
    ins = [x[r].cuda() for r in range(P)]
    outs = [torch.empty_like(t) for t in ins]
    host_in = [x[r].clone() for r in range(P)]
    host_out = torch.empty(n, dtype=torch.bfloat16)
    state_na = torch.zeros(E.echo_state_bytes(n, P, 128) // 4, dtype=torch.float32, device="cuda")
    fb = (1.0, 0.05, 0.5, 0.5)
    try:
        assert E.echo_inject_launch_failure(True) is False
        try:
            for fn in (lambda: ar(ins, outs, 4),
                       lambda: E.echo_phase_quantize(ins, ar.handle, 4, *fb),
                       lambda: E.echo_phase_reduce(ins, outs, ar.handle, 4, *fb),
                       lambda: E.echo_phase_gather(outs, ar.handle, 4),
                       lambda: E.echo_allreduce_sim_range(ins, outs, ar.handle, n, P, 4, 128, *fb, 0, G),
                       lambda: E.echo_allreduce_sim_host(host_in, host_out, ins, outs, ar.handle, n, P, 4, 128, *fb),
                       lambda: E.echo_allreduce_sim_noalloc(ins, outs, state_na, n, P, 4, 128, *fb),
                       lambda: rk.reduce(ins[0], outs[0], 4),
                       lambda: rk2.quantize(ins[0], 4),
                       lambda: rk2.reduce(ins[0], outs[0], 4),
                       lambda: rk2.decode(outs[0], 4)):
                with pytest.raises(E.EchoError) as ei:
                    fn()
                assert ei.value.status == E.ECHO_ECUDA
        finally:
            assert E.echo_inject_launch_failure(False) is True
        torch.cuda.synchronize()
        ar(ins, outs, 4)
        el = np.zeros((P, G * 128), np.float32)
        es = np.zeros((P, G * 128), np.float32)
        orc = O.echo_allreduce(padded(u16(x), G * 128), n_total=n, group=128, bits=4, e_long=el, e_short=es)
        assert ar.status() == (E.ECHO_OK, 0)
        assert np.array_equal(np.stack([u16(o) for o in outs]), orc.y[:, :n])
        # the no-allocation call's flag clear stayed enqueued under the hook;
        # its next call is correct (fresh state, so the same first-call result)
        outs_na = [torch.empty_like(t) for t in ins]
        assert E.echo_allreduce_sim_noalloc(ins, outs_na, state_na, n, P, 4, 128, *fb) == 0
        assert np.array_equal(np.stack([u16(o) for o in outs_na]), orc.y[:, :n])
    finally:
        E.echo_inject_launch_failure(False)
        ar.close()
        rk.close()
        rk2.close()
