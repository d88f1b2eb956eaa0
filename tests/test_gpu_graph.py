"""echo_allreduce_sim inside a CUDA graph.

Small tensor-parallel messages are launch-bound, so a caller may capture the
call (two kernel launches) into a CUDA graph and replay it. The library's
one-time per-kernel set-up (shared-memory opt-in, occupancy query) happens on
the first eager call; after that a captured call enqueues only the launches.
The test replays a captured call several times, carrying the EMA state, and
checks each replay against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle as O
import bit_error_compensated_group_b200 as E
from parity import GpuEcho, Params, padded, u16

pytestmark = pytest.mark.gpu


def test_captured_call_replays_bit_exact():
    P, n = 8, 8 * 4096 + 64          # a decode-sized message, partial last group
    G = -(-n // 128)
    g = torch.Generator().manual_seed(77)
    x = torch.randn(P, n, generator=g).to(torch.bfloat16)
    gpu = GpuEcho(P, n)
    try:
        gpu.set_inputs(x)
        el = np.zeros((P, G * 128), np.float32)
        es = np.zeros_like(el)
        xb = padded(u16(x), G * 128)
        stream = torch.cuda.Stream()
        p = Params()
        with torch.cuda.stream(stream):
            gpu.call(p)                                   # eager first call: set-up happens here
        stream.synchronize()
        O.echo_allreduce(xb, n_total=n, group=128, bits=4, e_long=el, e_short=es)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            E.echo_allreduce_sim(gpu.inputs, gpu.outputs, gpu.ar.handle, n, P, 4, 128,
                                 p.eta, p.alpha_long, p.alpha_short, p.w, stream=stream)
        for replay in range(3):
            graph.replay()
            torch.cuda.synchronize()
            ref = O.echo_allreduce(xb, n_total=n, group=128, bits=4, e_long=el, e_short=es)
            assert np.array_equal(gpu.outputs_u16(), ref.y[:, :n]), f"replay {replay}"
            gl, gs = gpu.state()
            assert np.array_equal(gl, el[:, :n]) and np.array_equal(gs, es[:, :n]), f"replay {replay}"
        rc, flags = gpu.status()
        assert rc == E.ECHO_OK
        del graph
    finally:
        gpu.close()
