"""Shared helpers for the GPU parity tests: run the CUDA path through the C
ABI and the oracle on the same seeded inputs, and compare element by element.

The oracle only ever sees inputs from ``workloads`` (or seeded states made
here) and its own previous outputs -- never a value computed by the CUDA path.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

import oracle as O
import workloads as W
import bit_error_compensated_group_b200 as E


@dataclass
class Params:
    bits: int = 4
    group: int = 128
    eta: float = 1.0
    alpha_long: float = 0.05
    alpha_short: float = 0.5
    w: float = 0.5
    quantizer: int = O.Q_DIRECTED   # the oracle's and the library's form numbers agree (0, 1, 2)


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def owners(G: int, P: int) -> np.ndarray:
    return np.array([O.owner(j, G, P) for j in range(G)], np.int64) if G <= 200000 else None


class GpuEcho:
    """The CUDA path for one message shape: per-rank input/output buffers and
    the library handle (state and workspace owned by torch)."""

    def __init__(self, P: int, n: int, group: int = 128, max_bits: int = 4, feedback: bool = True,
                 quantizer: int = O.Q_DIRECTED):
        self.P, self.n, self.group = P, n, group
        self.ar = E.EchoAllReduce(n, P, group, max_bits, feedback, quantizer=quantizer)
        self.G = int(self.ar.layout.groups)
        self.inputs = [torch.empty(n, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
        self.outputs = [torch.empty(n, dtype=torch.bfloat16, device="cuda") for _ in range(P)]

    def set_inputs(self, x: torch.Tensor) -> None:
        for r in range(self.P):
            self.inputs[r].copy_(x[r].reshape(-1), non_blocking=False)

    def set_state(self, el: np.ndarray, es: np.ndarray) -> None:
        L, S = self.ar.ema_views()
        L.copy_(torch.from_numpy(np.ascontiguousarray(el[:, :self.n])))
        S.copy_(torch.from_numpy(np.ascontiguousarray(es[:, :self.n])))

    def call(self, p: Params) -> None:
        self.ar(self.inputs, self.outputs, p.bits, p.eta, p.alpha_long, p.alpha_short, p.w)

    def status(self):
        return self.ar.status()

    def state(self) -> Tuple[np.ndarray, np.ndarray]:
        L, S = self.ar.ema_views()
        return L.cpu().numpy(), S.cpu().numpy()

    def outputs_u16(self, cols: Optional[slice] = None) -> np.ndarray:
        if cols is None:
            return np.stack([u16(o) for o in self.outputs])
        return np.stack([u16(o[cols]) for o in self.outputs])

    def payload(self, bits: int):
        a2a_c, a2a_p, g_c, g_p = self.ar.payload_views(bits)
        return (a2a_c.cpu().numpy(), a2a_p.cpu().numpy().view(np.uint16).reshape(self.P, self.G, 2),
                g_c.cpu().numpy(), g_p.cpu().numpy().view(np.uint16).reshape(self.G, 2))

    def close(self):
        self.ar.close()


def padded(a: np.ndarray, ld: int) -> np.ndarray:
    out = np.zeros((a.shape[0], ld), a.dtype)
    out[:, :a.shape[1]] = a
    return out


def assert_state_close(got: np.ndarray, want: np.ndarray, what: str) -> None:
    """EMA state bar: within 1e-6 relative, 1e-7 absolute near zero."""
    got = got.astype(np.float64)
    want = want.astype(np.float64)
    err = np.abs(got - want)
    tol = np.maximum(1e-6 * np.abs(want), 1e-7)
    bad = err > tol
    assert not bad.any(), f"{what}: {bad.sum()} elements off, max err {err.max():.3g}"


def assert_payload_equal(gpu_payload, orc: O.CallResult, G: int, P: int, j0: int = 0, jc: Optional[int] = None,
                         what: str = "") -> None:
    """Non-owner all-to-all slots and the gather payload must be bit-identical
    (the owner's own all-to-all slot is unused and not compared)."""
    jc = G - j0 if jc is None else jc
    a2a_c, a2a_p, g_c, g_p = gpu_payload
    for jl in range(jc):
        j = j0 + jl
        o = O.owner(j, G, P)
        for r in range(P):
            if r == o:
                continue
            assert np.array_equal(a2a_c[r, j], orc.a2a_codes[r, jl]), f"{what} a2a codes r={r} j={j}"
            assert np.array_equal(a2a_p[r, j], orc.a2a_params[r, jl]), f"{what} a2a params r={r} j={j}"
    if P >= 2:
        assert np.array_equal(g_c[j0:j0 + jc], orc.gather_codes), f"{what} gather codes"
        assert np.array_equal(g_p[j0:j0 + jc], orc.gather_params), f"{what} gather params"


def column_ranges(G: int, P: int, width: int) -> List[Tuple[int, int]]:
    """Sampled group-column ranges: the first and last columns, and each
    segment boundary (where the owner changes)."""
    starts = {0, max(0, G - width)}
    for s in range(1, P):
        b = O.segment_begin(s, G, P)
        starts.add(min(max(0, b - width // 2), max(0, G - width)))
    starts.add(G // 2)
    out = []
    for s in sorted(starts):
        jc = min(width, G - s)
        if out and s < out[-1][0] + out[-1][1]:
            continue
        out.append((s, jc))
    return out


def seeded_state(P, n, seed, scale=0.05):
    rng = np.random.default_rng(seed)
    return ((rng.standard_normal((P, n)) * scale).astype(np.float32),
            (rng.standard_normal((P, n)) * scale).astype(np.float32))


def random_inputs(P, n, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(P, n, generator=g) * scale).to(torch.bfloat16)


def check_full_call(P, n, p: Params, x, el0=None, es0=None, feedback=True, calls=1):
    """Run `calls` consecutive calls on both sides (state carried) and compare
    everything after each call."""
    G = -(-n // p.group)
    ld = G * p.group
    gpu = GpuEcho(P, n, p.group, max(p.bits, 4), feedback, p.quantizer)
    try:
        gpu.set_inputs(x)
        xb = padded(u16(x), ld)
        if feedback:
            el = padded(el0, ld) if el0 is not None else np.zeros((P, ld), np.float32)
            es = padded(es0, ld) if es0 is not None else np.zeros((P, ld), np.float32)
            gpu.set_state(el, es)
        else:
            el = es = None
        for c in range(calls):
            gpu.call(p)
            orc = O.echo_allreduce(xb, n_total=n, group=p.group, bits=p.bits, e_long=el, e_short=es,
                                   eta=p.eta, alpha_long=p.alpha_long, alpha_short=p.alpha_short, w=p.w,
                                   quantizer=p.quantizer)
            rc, flags = gpu.status()
            assert flags == orc.flags
            assert np.array_equal(gpu.outputs_u16(), orc.y[:, :n]), f"outputs differ (call {c})"
            assert_payload_equal(gpu.payload(p.bits), orc, G, P, what=f"call {c}")
            if feedback:
                gl, gs = gpu.state()
                assert_state_close(gl, el[:, :n], f"e_long call {c}")
                assert_state_close(gs, es[:, :n], f"e_short call {c}")
                assert np.array_equal(gl, el[:, :n]) and np.array_equal(gs, es[:, :n])  # expected bit-exact
    finally:
        gpu.close()
