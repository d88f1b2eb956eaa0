"""Chunked calls through the C ABI against the oracle.

* echo_allreduce_sim_range: windows of group columns that tile [0, G), taken
  in any order, give the oracle's whole-call result bit for bit (outputs,
  both payloads, flags; EMA state within 1e-6 relative and, as expected,
  bit-identical), and a window touches nothing outside its columns;
* echo_allreduce_sim_host: pinned host inputs in, host result out, copies on
  their own streams overlapping the kernels -- the same bits as the oracle's
  call, over consecutive calls whose state carries over.
"""
import numpy as np
import pytest
import torch

import oracle as O
import bit_error_compensated_group_b200 as E
from parity import (GpuEcho, Params, assert_payload_equal, assert_state_close, padded, random_inputs, seeded_state,
                    u16)

pytestmark = pytest.mark.gpu

P_DEF = Params(w=0.3, alpha_long=0.1, alpha_short=0.6)


def windows(G, sizes, order, seed=0):
    out, b, i = [], 0, 0
    while b < G:
        e = min(G, b + sizes[i % len(sizes)])
        out.append((b, e))
        b, i = e, i + 1
    if order == "reversed":
        out = out[::-1]
    elif order == "shuffled":
        perm = np.random.default_rng(seed).permutation(len(out))
        out = [out[k] for k in perm]
    return out


def run_windows(gpu, p, wins):
    for b, e in wins:
        E.echo_allreduce_sim_range(gpu.inputs, gpu.outputs, gpu.ar.handle, gpu.n, gpu.P, p.bits, p.group, p.eta,
                                   p.alpha_long, p.alpha_short, p.w, b, e)


def compare(gpu, orc, el, es, n, G, P, p, feedback, what):
    rc, flags = gpu.status()
    assert flags == orc.flags, what
    assert np.array_equal(gpu.outputs_u16(), orc.y[:, :n]), f"{what}: outputs differ"
    assert_payload_equal(gpu.payload(p.bits), orc, G, P, what=what)
    if feedback:
        gl, gs = gpu.state()
        assert_state_close(gl, el[:, :n], f"{what} e_long")
        assert_state_close(gs, es[:, :n], f"{what} e_short")
        assert np.array_equal(gl, el[:, :n]) and np.array_equal(gs, es[:, :n])


CASES = [
    # P, n, group, bits, window widths (cycled)
    (8, 8192 * 3 + 77, 128, 4, [5, 17, 1, 30]),      # partial last group, owner boundaries inside windows
    (3, 1000, 32, 8, [7]),
    (1, 5000, 64, 4, [3, 11]),                        # P = 1: nothing quantized
    (16, 3000, 128, 4, [2]),                          # G < P: empty segments
    (5, 148 * 8 * 256 + 37, 256, 8, [1000, 33]),
]


@pytest.mark.parametrize("P,n,group,bits,sizes", CASES)
@pytest.mark.parametrize("feedback", [True, False])
@pytest.mark.parametrize("order", ["forward", "reversed", "shuffled"])
def test_windows_tile_the_call(P, n, group, bits, sizes, feedback, order):
    p = Params(bits=bits, group=group, w=P_DEF.w, alpha_long=P_DEF.alpha_long, alpha_short=P_DEF.alpha_short)
    G = -(-n // group)
    ld = G * group
    x = random_inputs(P, n, 31 * P + n, 2.0)
    gpu = GpuEcho(P, n, group, max(bits, 4), feedback)
    try:
        gpu.set_inputs(x)
        xb = padded(u16(x), ld)
        el = es = None
        if feedback:
            el0, es0 = seeded_state(P, n, n + 3 * P)
            gpu.set_state(el0, es0)
            el, es = padded(el0, ld), padded(es0, ld)
        for c in range(2):
            run_windows(gpu, p, windows(G, sizes, order, seed=c))
            orc = O.echo_allreduce(xb, n_total=n, group=group, bits=bits, e_long=el, e_short=es, eta=p.eta,
                                   alpha_long=p.alpha_long, alpha_short=p.alpha_short, w=p.w)
            compare(gpu, orc, el, es, n, G, P, p, feedback, f"call {c} {order}")
    finally:
        gpu.close()


def test_window_touches_only_its_columns():
    P, n, group = 4, 20000, 128
    p = Params()
    G = -(-n // group)
    b, e = 37, 101                                    # straddles the owner boundary at G/4
    x = random_inputs(P, n, 77)
    el0, es0 = seeded_state(P, n, 78)
    gpu = GpuEcho(P, n)
    try:
        gpu.set_inputs(x)
        gpu.set_state(el0, es0)
        sentinel = torch.tensor(0x7E55, dtype=torch.int16).view(torch.bfloat16)
        for o in gpu.outputs:
            o.fill_(sentinel)
        run_windows(gpu, p, [(b, e)])
        el, es = el0[:, b * group:e * group].copy(), es0[:, b * group:e * group].copy()
        orc = O.echo_allreduce(np.ascontiguousarray(u16(x)[:, b * group:e * group]), n_total=n, group=group, bits=4,
                               e_long=el, e_short=es, j0=b, jc=e - b)
        out = gpu.outputs_u16()
        inside = slice(b * group, e * group)
        assert np.array_equal(out[:, inside], orc.y)
        mask = np.ones(n, bool)
        mask[inside] = False
        assert (out[:, mask] == 0x7E55).all()
        gl, gs = gpu.state()
        assert np.array_equal(gl[:, inside], el) and np.array_equal(gs[:, inside], es)
        assert np.array_equal(gl[:, mask], el0[:, mask]) and np.array_equal(gs[:, mask], es0[:, mask])
        assert_payload_equal(gpu.payload(4), orc, G, P, j0=b, jc=e - b)
        # an empty window enqueues nothing; a window past G is refused
        run_windows(gpu, p, [(5, 5)])
        with pytest.raises(E.EchoError) as ei:
            run_windows(gpu, p, [(0, G + 1)])
        assert ei.value.status == E.ECHO_EINVAL
        with pytest.raises(E.EchoError):
            run_windows(gpu, p, [(9, 8)])
    finally:
        gpu.close()


@pytest.mark.parametrize("P,n,group,bits,chunk", [
    (8, 100003, 128, 4, 0),       # default chunking, partial last group
    (4, 5000, 64, 8, 7),
    (2, 1, 32, 4, 1),             # a single element
    (1, 4096, 128, 4, 5),
    (8, 1 << 20, 128, 4, 1000),
])
def test_host_call(P, n, group, bits, chunk):
    p = Params(bits=bits, group=group)
    G = -(-n // group)
    ld = G * group
    gpu = GpuEcho(P, n, group, max(bits, 4), True)
    cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
    s = torch.cuda.current_stream()
    host_in = [torch.empty(n, dtype=torch.bfloat16, pin_memory=True) for _ in range(P)]
    host_out = torch.empty(n, dtype=torch.bfloat16, pin_memory=True)
    el = np.zeros((P, ld), np.float32)
    es = np.zeros((P, ld), np.float32)
    try:
        for c in range(3):
            x = random_inputs(P, n, 1000 * c + P + n)
            for r in range(P):
                host_in[r].copy_(x[r])
            E.echo_allreduce_sim_host(host_in, host_out, gpu.inputs, gpu.outputs, gpu.ar.handle, n, P, bits, group,
                                      p.eta, p.alpha_long, p.alpha_short, p.w, chunk, stream=s, copy_in=cin,
                                      copy_out=cout)
            s.synchronize()
            orc = O.echo_allreduce(padded(u16(x), ld), n_total=n, group=group, bits=bits, e_long=el, e_short=es)
            assert np.array_equal(u16(host_out), orc.y[0, :n]), f"host result, call {c}"
            assert np.array_equal(np.stack([u16(t) for t in gpu.inputs]), u16(x)), f"device inputs, call {c}"
            compare(gpu, orc, el, es, n, G, P, p, True, f"host call {c}")
    finally:
        gpu.close()


@pytest.mark.parametrize("windowed", [False, True])
def test_in_place_large(windowed):
    """Outputs that are the inputs, on a message whose quantize pass spans
    many tiles per CTA: the owners' pass (a programmatic dependent of the
    quantize pass) must not write an output before the quantize pass has read
    it. Two calls with carried state; every element checked."""
    P, n, group = 8, (1 << 22) + 77, 128
    p = Params()
    G = -(-n // group)
    ld = G * group
    x = random_inputs(P, n, 4242)
    gpu = GpuEcho(P, n, group, 4, True)
    el = np.zeros((P, ld), np.float32)
    es = np.zeros((P, ld), np.float32)
    try:
        xb = padded(u16(x), ld)
        for c in range(2):
            gpu.set_inputs(x if c == 0 else E_out)
            if windowed:
                for b, e in windows(G, [G // 3 + 1], "forward"):
                    E.echo_allreduce_sim_range(gpu.inputs, gpu.inputs, gpu.ar.handle, n, P, 4, group, p.eta,
                                               p.alpha_long, p.alpha_short, p.w, b, e)
            else:
                E.echo_allreduce_sim(gpu.inputs, gpu.inputs, gpu.ar.handle, n, P, 4, group, p.eta, p.alpha_long,
                                     p.alpha_short, p.w)
            orc = O.echo_allreduce(xb, n_total=n, group=group, bits=4, e_long=el, e_short=es)
            got = np.stack([u16(t) for t in gpu.inputs])
            assert np.array_equal(got, orc.y[:, :n]), f"call {c}"
            gl, gs = gpu.state()
            assert np.array_equal(gl, el[:, :n]) and np.array_equal(gs, es[:, :n]), f"state call {c}"
            # the next call reduces this call's result again (every rank holds it)
            E_out = torch.from_numpy(orc.y[:, :n].astype(np.uint16).view(np.int16)).view(torch.bfloat16)
            xb = padded(orc.y[:, :n].copy(), ld)
    finally:
        gpu.close()


@pytest.mark.parametrize("to_host,streams", [(False, "separate"), (True, "same"), (True, "pageable")])
def test_host_call_forms(to_host, streams):
    """The host-buffer call without a host result (the result stays on the
    device), with every copy on the caller's stream, and from pageable host
    memory (the copies then serialize): the same bits in every form."""
    P, n, group = 4, 70001, 64
    p = Params(group=group)
    G = -(-n // group)
    ld = G * group
    gpu = GpuEcho(P, n, group, 4, True)
    pin = streams != "pageable"
    host_in = [torch.empty(n, dtype=torch.bfloat16, pin_memory=pin) for _ in range(P)]
    host_out = torch.empty(n, dtype=torch.bfloat16, pin_memory=pin) if to_host else None
    s = torch.cuda.current_stream()
    cin, cout = (torch.cuda.Stream(), torch.cuda.Stream()) if streams == "separate" else (s, s)
    el = np.zeros((P, ld), np.float32)
    es = np.zeros((P, ld), np.float32)
    try:
        for c in range(2):
            x = random_inputs(P, n, 77 * c + 5)
            for r in range(P):
                host_in[r].copy_(x[r])
            E.echo_allreduce_sim_host(host_in, host_out, gpu.inputs, gpu.outputs, gpu.ar.handle, n, P, 4, group,
                                      p.eta, p.alpha_long, p.alpha_short, p.w, 9, stream=s, copy_in=cin,
                                      copy_out=cout)
            s.synchronize()
            orc = O.echo_allreduce(padded(u16(x), ld), n_total=n, group=group, bits=4, e_long=el, e_short=es)
            if to_host:
                assert np.array_equal(u16(host_out), orc.y[0, :n])
            compare(gpu, orc, el, es, n, G, P, p, True, f"{streams} call {c}")
    finally:
        gpu.close()


@pytest.mark.parametrize("world", [2, 3])
def test_column_split_across_gpus(world):
    """The benchmark's split of one message over N GPUs, on one GPU: N
    separate handles (each with its own EMA state and workspace, as on
    separate GPUs) run echo_allreduce_sim_range on their column windows
    (column_window); their windows of the outputs and state, put together,
    are the oracle's whole call, twice in a row."""
    P, n, group = 8, 8192 * 5 + 77, 128
    p = Params()
    G = -(-n // group)
    ld = G * group
    x = random_inputs(P, n, 4242, 1.5)
    xb = padded(u16(x), ld)
    el, es = np.zeros((P, ld), np.float32), np.zeros((P, ld), np.float32)
    gpus = [GpuEcho(P, n) for _ in range(world)]
    try:
        wins = [E.column_window(k, world, G) for k in range(world)]
        for g in gpus:
            g.set_inputs(x)
            g.set_state(el, es)
        for call in range(2):
            for g, (c0, c1) in zip(gpus, wins):
                run_windows(g, p, [(c0, c1)])
            orc = O.echo_allreduce(xb, n_total=n, group=group, bits=4, e_long=el, e_short=es)
            for g, (c0, c1) in zip(gpus, wins):
                assert g.status() == (E.ECHO_OK, 0)
                sl = slice(c0 * group, min(c1 * group, n))
                assert np.array_equal(g.outputs_u16()[:, sl], orc.y[:, sl]), (call, c0, c1)
                gl, gs = g.state()
                assert np.array_equal(gl[:, sl], el[:, sl]) and np.array_equal(gs[:, sl], es[:, sl]), (call, c0, c1)
    finally:
        for g in gpus:
            g.close()
