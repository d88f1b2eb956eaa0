"""echo_allreduce_sim_noalloc: the all-reduce for callers that cannot
allocate device memory.

Some callers may not allocate device memory where they run the all-reduce:
a serving engine that reserved the device for its own pools at start-up, or
a latency-critical path that cannot pay the device-wide synchronization of
cudaMalloc/cudaFree. The no-allocation entry point keeps the payloads in a
fixed scratch array inside the library, so such a caller passes only its
inputs, outputs and EMA state. These tests call it through the C ABI and
check that two calls in a row give exactly what the ordinary, workspace-based
echo_allreduce_sim gives and what the oracle gives (outputs bit-identical,
EMA state within the usual 1e-6 relative bar -- in fact identical), that a
value outside the fp16 parameter range is reported through the call's return
code, and that a message too large for the scratch is refused.

This file is collected last on purpose: it runs alone or after everything
else, and the shared scratch must not depend on what ran before.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
import bit_error_compensated_group_b200 as E
from bit_error_compensated_group_b200 import echo as EE
from parity import assert_state_close, padded, u16

pytestmark = pytest.mark.gpu


def _inputs(P, n, seed):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(P, n, generator=g) * 1.5).to(torch.bfloat16)
    return [x[r].cuda() for r in range(P)]


@pytest.mark.parametrize("P,n,group,bits,feedback", [
    (8, 2 * 1024 * 1024 - 37, 128, 4, True),    # partial last group, feedback on
    (3, 300_001, 64, 8, False),                  # 8-bit mode, no feedback
    (1, 5000, 128, 4, True),                     # single rank
])
def test_noalloc_matches_workspace_entry_point(P, n, group, bits, feedback):
    assert EE.echo_query_layout(n, P, group, bits, bits).workspace_bytes <= E.echo.ECHO_NOALLOC_SCRATCH_BYTES
    ins = _inputs(P, n, 1000 + P)
    out_ref = [torch.empty_like(t) for t in ins]
    out_na = [torch.full_like(t, 7.0) for t in ins]
    ref = E.EchoAllReduce(n, P, group, bits, feedback)
    state_na = None
    if feedback:
        state_na = torch.zeros(E.echo_state_bytes(n, P, group) // 4, dtype=torch.float32, device="cuda")
    kw = dict(eta=1.0, alpha_long=0.05, alpha_short=0.5, w=0.5)
    G = -(-n // group)
    x_host = padded(np.stack([u16(t) for t in ins]), G * group)
    el = np.zeros((P, G * group), np.float32) if feedback else None
    es = np.zeros((P, G * group), np.float32) if feedback else None
    try:
        for call in range(2):
            ref(ins, out_ref, bits, **kw)
            flags = EE.echo_allreduce_sim_noalloc(ins, out_na, state_na, n, P, bits, group, kw["eta"],
                                                  kw["alpha_long"], kw["alpha_short"], kw["w"])
            rc, ref_flags = ref.status()
            assert flags == 0 and ref_flags == 0 and rc == E.ECHO_OK
            orc = O.echo_allreduce(x_host, n_total=n, group=group, bits=bits, e_long=el, e_short=es, **kw)
            for r in range(P):
                assert np.array_equal(u16(out_na[r]), u16(out_ref[r])), f"call {call} rank {r}"
                assert np.array_equal(u16(out_na[r]), orc.y[r, :n]), f"call {call} rank {r} vs oracle"
            if feedback:
                got = state_na.cpu().numpy()
                want = ref.state.cpu().numpy()
                S = int(ref.layout.state_stride)
                g3, w3 = got.reshape(P, 2, S)[:, :, :n], want.reshape(P, 2, S)[:, :, :n]
                assert_state_close(g3, w3, f"EMA state call {call}")
                assert np.array_equal(g3, w3)
                o3 = np.stack([el[:, :n], es[:, :n]], axis=1)
                assert_state_close(g3, o3, f"EMA state call {call} vs oracle")
    finally:
        ref.close()


def test_noalloc_reports_range_violations_in_its_return_code():
    """A value beyond the fp16 range (here 2^17 in rank 1's input) cannot get
    fp16 parameters: the kernels raise the range flag, and with a flag word
    requested the call returns ECHO_ERANGE (there is no handle to ask later).
    The next call on ordinary inputs is clean again: each call clears the
    flag word first."""
    P, n, group, bits = 2, 4096, 128, 4
    ins = _inputs(P, n, 77)
    ins[1][300] = 2.0 ** 17
    outs = [torch.empty_like(t) for t in ins]
    with pytest.raises(E.EchoError) as ei:
        EE.echo_allreduce_sim_noalloc(ins, outs, None, n, P, bits, group, 1.0, 0.05, 0.5, 0.5)
    assert ei.value.status == EE.ECHO_ERANGE
    ins[1][300] = 1.0
    assert EE.echo_allreduce_sim_noalloc(ins, outs, None, n, P, bits, group, 1.0, 0.05, 0.5, 0.5) == 0
    # without a flag word nothing reads the flags: the call itself succeeds
    ins[1][300] = 2.0 ** 17
    assert EE.echo_allreduce_sim_noalloc(ins, outs, None, n, P, bits, group, 1.0, 0.05, 0.5, 0.5,
                                         read_flags=False) is None
    torch.cuda.synchronize()


def test_noalloc_refuses_messages_beyond_the_scratch():
    P, group, bits = 8, 128, 4
    n = 8 * 1024 * 1024          # needs ~39 MB of payload scratch
    assert EE.echo_query_layout(n, P, group, bits, bits).workspace_bytes > E.echo.ECHO_NOALLOC_SCRATCH_BYTES
    ins = [torch.zeros(n, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    outs = [torch.empty_like(t) for t in ins]
    with pytest.raises(E.EchoError) as ei:
        EE.echo_allreduce_sim_noalloc(ins, outs, None, n, P, bits, group, 1.0, 0.05, 0.5, 0.5)
    assert ei.value.status == EE.ECHO_ENOSPACE
    assert "scratch" in E.echo_status_string(EE.ECHO_ENOSPACE)
