"""ctypes binding of ``libecho_b200.so`` (the C ABI in ``include/echo.h``).

Argument marshalling only: every step of the all-reduce runs in the library's
CUDA kernels. Functions keep the C names; tensors are passed as device
pointers and the stream defaults to torch's current stream. A missing or
unloadable library raises immediately -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

from . import _build

ECHO_OK, ECHO_EINVAL, ECHO_ECUDA, ECHO_ERANGE, ECHO_ETIMEOUT, ECHO_ENOSPACE = 0, 1, 2, 3, 4, 5
ECHO_NOALLOC_SCRATCH_BYTES = 16 << 20
ECHO_FLAG_RANGE = 1
ECHO_FLAG_TIMEOUT = 2
ECHO_MAX_RANKS = 64
ECHO_MAX_CHUNKS = 4096
ECHO_QUANT_DIRECTED, ECHO_QUANT_NEAREST, ECHO_QUANT_INT_ZERO = 0, 1, 2

LIB_PATH = _build.LIB

_lib: Optional[ctypes.CDLL] = None


class EchoError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {echo_status_string(status)} ({status})")


class EchoLayout(ctypes.Structure):
    _fields_ = [
        ("groups", ctypes.c_int64),
        ("state_stride", ctypes.c_int64),
        ("code_bytes", ctypes.c_uint64),
        ("flags_offset", ctypes.c_uint64),
        ("a2a_codes_offset", ctypes.c_uint64),
        ("a2a_params_offset", ctypes.c_uint64),
        ("gather_codes_offset", ctypes.c_uint64),
        ("gather_params_offset", ctypes.c_uint64),
        ("workspace_bytes", ctypes.c_uint64),
        ("state_bytes", ctypes.c_uint64),
    ]


class EchoRankLayout(ctypes.Structure):
    _fields_ = [
        ("groups", ctypes.c_int64),
        ("seg_begin", ctypes.c_int64),
        ("seg_groups", ctypes.c_int64),
        ("seg_max", ctypes.c_int64),
        ("code_bytes", ctypes.c_uint64),
        ("flags_offset", ctypes.c_uint64),
        ("send_codes_offset", ctypes.c_uint64),
        ("send_params_offset", ctypes.c_uint64),
        ("recv_codes_offset", ctypes.c_uint64),
        ("recv_params_offset", ctypes.c_uint64),
        ("gsend_codes_offset", ctypes.c_uint64),
        ("gsend_params_offset", ctypes.c_uint64),
        ("grecv_codes_offset", ctypes.c_uint64),
        ("grecv_params_offset", ctypes.c_uint64),
        ("workspace_bytes", ctypes.c_uint64),
        ("state_bytes", ctypes.c_uint64),
    ]


def lib() -> ctypes.CDLL:
    """Load the CUDA library; raises if it was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"Echo CUDA library missing at {LIB_PATH}; build it with "
                               "`python -m bit_error_compensated_group_b200._build`")
        L = ctypes.CDLL(LIB_PATH)
        V, I, I64, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
        PP = ctypes.POINTER(ctypes.c_void_p)
        L.echo_state_bytes.argtypes = [I64, I, I]
        L.echo_state_bytes.restype = ctypes.c_size_t
        L.echo_workspace_bytes.argtypes = [I64, I, I, I]
        L.echo_workspace_bytes.restype = ctypes.c_size_t
        L.echo_query_layout.argtypes = [I64, I, I, I, I, ctypes.POINTER(EchoLayout)]
        L.echo_query_layout.restype = I
        L.echo_init_state.argtypes = [ctypes.POINTER(V), I64, I, I, I, V, V, V]
        L.echo_init_state.restype = I
        L.echo_allreduce_sim.argtypes = [PP, PP, V, I64, I, I, I, F, F, F, F, V]
        L.echo_allreduce_sim.restype = I
        L.echo_allreduce_sim_range.argtypes = [PP, PP, V, I64, I, I, I, F, F, F, F, I64, I64, V]
        L.echo_allreduce_sim_range.restype = I
        L.echo_allreduce_sim_host.argtypes = [PP, V, PP, PP, V, I64, I, I, I, F, F, F, F, I64, V, V, V]
        L.echo_allreduce_sim_host.restype = I
        L.echo_phase_quantize.argtypes = [PP, V, I, F, F, F, F, V]
        L.echo_phase_quantize.restype = I
        L.echo_phase_reduce.argtypes = [PP, PP, V, I, F, F, F, F, V]
        L.echo_phase_reduce.restype = I
        L.echo_phase_gather.argtypes = [PP, V, I, V]
        L.echo_phase_gather.restype = I
        L.echo_check_watchdog.argtypes = [V, ctypes.c_uint32, V]
        L.echo_check_watchdog.restype = I
        L.echo_get_status.argtypes = [V, V, ctypes.POINTER(ctypes.c_uint32)]
        L.echo_get_status.restype = I
        L.echo_set_quantizer.argtypes = [V, I]
        L.echo_set_quantizer.restype = I
        L.echo_query_rank_layout.argtypes = [I64, I, I, I, I, I, ctypes.POINTER(EchoRankLayout)]
        L.echo_query_rank_layout.restype = I
        L.echo_init_rank.argtypes = [ctypes.POINTER(V), I64, I, I, I, I, V, V, V]
        L.echo_init_rank.restype = I
        L.echo_rank_quantize.argtypes = [V, V, I, F, F, F, F, V]
        L.echo_rank_quantize.restype = I
        L.echo_rank_reduce.argtypes = [V, V, V, I, F, F, F, F, V]
        L.echo_rank_reduce.restype = I
        L.echo_rank_decode.argtypes = [V, V, I, V]
        L.echo_rank_decode.restype = I
        L.echo_rank_quantize_chunk.argtypes = [V, V, I, F, F, F, F, I, I, V]
        L.echo_rank_quantize_chunk.restype = I
        L.echo_rank_reduce_chunk.argtypes = [V, V, V, I, F, F, F, F, I, I, V]
        L.echo_rank_reduce_chunk.restype = I
        L.echo_rank_decode_chunk.argtypes = [V, V, I, I, I, V]
        L.echo_rank_decode_chunk.restype = I
        L.echo_query_chunk.argtypes = [I64, I, I, I, I, I, ctypes.POINTER(I64), ctypes.POINTER(I64)]
        L.echo_query_chunk.restype = I
        L.echo_bf16_allreduce_sim.argtypes = [PP, PP, I64, I, V]
        L.echo_bf16_allreduce_sim.restype = I
        L.echo_background_traffic.argtypes = [V, V, ctypes.c_size_t, ctypes.c_uint32, ctypes.c_uint32,
                                              ctypes.c_uint32, V, V]
        L.echo_background_traffic.restype = I
        L.echo_inject_launch_failure.argtypes = [I]
        L.echo_inject_launch_failure.restype = I
        L.echo_set_wait_limit.argtypes = [V, ctypes.c_uint32]
        L.echo_set_wait_limit.restype = I
        L.echo_get_wait_limit.argtypes = [V]
        L.echo_get_wait_limit.restype = ctypes.c_uint32
        L.echo_allreduce_sim_noalloc.argtypes = [PP, PP, V, I64, I, I, I, F, F, F, F,
                                                 ctypes.POINTER(ctypes.c_uint32), V]
        L.echo_allreduce_sim_noalloc.restype = I
        L.echo_free.argtypes = [V]
        L.echo_free.restype = I
        L.echo_status_string.argtypes = [I]
        L.echo_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def echo_status_string(status: int) -> str:
    return lib().echo_status_string(status).decode()


def _check(rc: int, what: str) -> None:
    if rc != ECHO_OK:
        raise EchoError(rc, what)


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("Echo buffers must be contiguous CUDA tensors")
    return t.data_ptr()


def _ptr_array(ts: Sequence) -> ctypes.Array:
    return (ctypes.c_void_p * len(ts))(*[_ptr(t) for t in ts])


# ----------------------------------------------------------------- sizes

def echo_state_bytes(n: int, P: int, group: int) -> int:
    return int(lib().echo_state_bytes(n, P, group))


def echo_workspace_bytes(n: int, P: int, group: int, max_bits: int) -> int:
    return int(lib().echo_workspace_bytes(n, P, group, max_bits))


def echo_query_layout(n: int, P: int, group: int, max_bits: int, bits: int) -> EchoLayout:
    out = EchoLayout()
    _check(lib().echo_query_layout(n, P, group, max_bits, bits, ctypes.byref(out)), "echo_query_layout")
    return out


# ----------------------------------------------------------------- calls

def echo_init_state(n: int, P: int, group: int, max_bits: int, state, workspace, stream=None) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(lib().echo_init_state(ctypes.byref(h), n, P, group, max_bits, _ptr(state), _ptr(workspace),
                                 _stream(stream)), "echo_init_state")
    return h


def echo_allreduce_sim(inputs: Sequence, outputs: Sequence, st, n: int, P: int, bits: int, group: int,
                       eta: float, alpha_long: float, alpha_short: float, w: float, stream=None) -> None:
    _check(lib().echo_allreduce_sim(_ptr_array(inputs), _ptr_array(outputs), st, n, P, bits, group,
                                    eta, alpha_long, alpha_short, w, _stream(stream)), "echo_allreduce_sim")


def echo_allreduce_sim_range(inputs: Sequence, outputs: Sequence, st, n: int, P: int, bits: int, group: int,
                             eta: float, alpha_long: float, alpha_short: float, w: float, group_begin: int,
                             group_end: int, stream=None) -> None:
    _check(lib().echo_allreduce_sim_range(_ptr_array(inputs), _ptr_array(outputs), st, n, P, bits, group,
                                          eta, alpha_long, alpha_short, w, group_begin, group_end,
                                          _stream(stream)), "echo_allreduce_sim_range")


def column_window(rank: int, world: int, G: int):
    """Group columns ``[c0, c1)`` that GPU ``rank`` of ``world`` takes when one
    message is split across GPUs: contiguous ranges ``[floor(rank G / world),
    floor((rank + 1) G / world))``. They tile ``[0, G)`` in rank order; each
    GPU runs ``echo_allreduce_sim_range`` on its window of the same message
    (every column is independent: all P ranks' group j, their payloads and
    EMA rows), so no collective is needed on the data path."""
    if world < 1 or not 0 <= rank < world or G < 0:
        raise ValueError("column_window: need 0 <= rank < world and G >= 0")
    return rank * G // world, (rank + 1) * G // world


def _host_ptr(t) -> int:
    if isinstance(t, int):
        return t
    if t.is_cuda or not t.is_contiguous():
        raise ValueError("host buffers must be contiguous CPU tensors")
    return t.data_ptr()


def echo_allreduce_sim_host(host_inputs: Sequence, host_output, inputs: Sequence, outputs: Sequence, st, n: int,
                            P: int, bits: int, group: int, eta: float, alpha_long: float, alpha_short: float,
                            w: float, chunk_groups: int = 0, stream=None, copy_in=None, copy_out=None) -> None:
    """Host inputs in, host result out, copies overlapped with the kernels
    (pinned host tensors for the overlap). `copy_in` / `copy_out` default to
    `stream` (no overlap)."""
    s = _stream(stream)
    hin = (ctypes.c_void_p * len(host_inputs))(*[_host_ptr(t) for t in host_inputs])
    hout = None if host_output is None else _host_ptr(host_output)
    _check(lib().echo_allreduce_sim_host(hin, hout, _ptr_array(inputs), _ptr_array(outputs), st, n, P, bits, group,
                                         eta, alpha_long, alpha_short, w, chunk_groups, s,
                                         s if copy_in is None else _stream(copy_in),
                                         s if copy_out is None else _stream(copy_out)),
           "echo_allreduce_sim_host")


def echo_phase_quantize(inputs: Sequence, st, bits: int, eta: float, alpha_long: float, alpha_short: float,
                        w: float, stream=None) -> None:
    _check(lib().echo_phase_quantize(_ptr_array(inputs), st, bits, eta, alpha_long, alpha_short, w,
                                     _stream(stream)), "echo_phase_quantize")


def echo_phase_reduce(inputs: Sequence, outputs: Optional[Sequence], st, bits: int, eta: float,
                      alpha_long: float, alpha_short: float, w: float, stream=None) -> None:
    outs = _ptr_array(outputs) if outputs is not None else None
    _check(lib().echo_phase_reduce(_ptr_array(inputs), outs, st, bits, eta, alpha_long, alpha_short, w,
                                   _stream(stream)), "echo_phase_reduce")


def echo_phase_gather(outputs: Sequence, st, bits: int, stream=None) -> None:
    _check(lib().echo_phase_gather(_ptr_array(outputs), st, bits, _stream(stream)), "echo_phase_gather")


def echo_check_watchdog(st, limit_us: int, stream=None) -> None:
    _check(lib().echo_check_watchdog(st, limit_us, _stream(stream)), "echo_check_watchdog")


def echo_get_status(st, stream=None):
    """Returns (status, flags); synchronizes the stream."""
    flags = ctypes.c_uint32(0)
    rc = lib().echo_get_status(st, _stream(stream), ctypes.byref(flags))
    if rc not in (ECHO_OK, ECHO_ERANGE, ECHO_ETIMEOUT):
        raise EchoError(rc, "echo_get_status")
    return rc, int(flags.value)


def echo_allreduce_sim_noalloc(inputs: Sequence, outputs: Sequence, state, n: int, P: int, bits: int,
                               group: int, eta: float, alpha_long: float, alpha_short: float, w: float,
                               stream=None, read_flags: bool = True) -> Optional[int]:
    """echo_allreduce_sim for callers that cannot allocate device memory:
    the payloads live in the library's fixed scratch array, there is no
    handle, and the caller passes the EMA state tensor (or None for no
    feedback). With `read_flags` (which synchronizes the stream) a range or
    timeout flag raised by the call's kernels raises EchoError (ECHO_ERANGE /
    ECHO_ETIMEOUT) and the flag bits (0) are returned; without it nothing
    reports such a failure and None is returned."""
    flags = ctypes.c_uint32(0)
    rc = lib().echo_allreduce_sim_noalloc(_ptr_array(inputs), _ptr_array(outputs), _ptr(state), n, P, bits, group,
                                          eta, alpha_long, alpha_short, w,
                                          ctypes.byref(flags) if read_flags else None, _stream(stream))
    _check(rc, "echo_allreduce_sim_noalloc")
    return int(flags.value) if read_flags else None


def echo_bf16_allreduce_sim(inputs: Sequence, outputs: Sequence, n: int, P: int, stream=None) -> None:
    """The 16-bit baseline all-reduce over P virtual ranks (rank-ordered
    binary32 sum, bf16 result into every output)."""
    _check(lib().echo_bf16_allreduce_sim(_ptr_array(inputs), _ptr_array(outputs), n, P, _stream(stream)),
           "echo_bf16_allreduce_sim")


def echo_background_traffic(src, dst, duty_permille: int, period_us: int, duration_us: int, moved=None,
                            stream=None) -> None:
    """Competing HBM traffic: copy src -> dst (same size, bytes a multiple of
    16) for the duty cycle of every period, for duration_us of wall-clock
    time. `moved`: an int64 CUDA tensor that accumulates the bytes moved."""
    if src.numel() * src.element_size() != dst.numel() * dst.element_size():
        raise ValueError("echo_background_traffic: src and dst differ in size")
    _check(lib().echo_background_traffic(_ptr(src), _ptr(dst), src.numel() * src.element_size(), duty_permille,
                                         period_us, duration_us, _ptr(moved), _stream(stream)),
           "echo_background_traffic")


def echo_set_wait_limit(st, limit_us: int) -> None:
    """Limit of the kernels' bounded device waits for the handle's later
    calls (1 ms .. 60 s; default 1 s)."""
    _check(lib().echo_set_wait_limit(st, limit_us), "echo_set_wait_limit")


def echo_get_wait_limit(st) -> int:
    return int(lib().echo_get_wait_limit(st))


def echo_set_quantizer(st, quantizer: int) -> None:
    """Quantizer form for the handle's later calls (ECHO_QUANT_*)."""
    _check(lib().echo_set_quantizer(st, quantizer), "echo_set_quantizer")


def echo_inject_launch_failure(enable: bool) -> bool:
    """Test hook: while enabled, kernel launches report ECHO_ECUDA (nothing
    fails on the GPU). Returns the previous setting."""
    return bool(lib().echo_inject_launch_failure(1 if enable else 0))


def echo_free(st) -> None:
    lib().echo_free(st)


# ----------------------------------------------------------------- convenience

class EchoAllReduce:
    """Owns (through torch) the EMA state and workspace of one message shape
    and the library handle; ``__call__`` runs echo_allreduce_sim."""

    def __init__(self, n: int, P: int, group: int = 128, max_bits: int = 4, feedback: bool = True,
                 device=None, stream=None, quantizer: int = ECHO_QUANT_DIRECTED):
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.n, self.P, self.group, self.max_bits = n, P, group, max_bits
        self.layout = echo_query_layout(n, P, group, max_bits, max_bits)
        self.workspace = torch.empty(int(self.layout.workspace_bytes), dtype=torch.uint8, device=device)
        self.state = None
        if feedback:
            self.state = torch.empty(int(self.layout.state_bytes) // 4, dtype=torch.float32, device=device)
        self.handle = echo_init_state(n, P, group, max_bits, self.state, self.workspace, stream)
        if quantizer != ECHO_QUANT_DIRECTED:
            echo_set_quantizer(self.handle, quantizer)

    def __call__(self, inputs, outputs, bits: int = 4, eta: float = 1.0, alpha_long: float = 0.05,
                 alpha_short: float = 0.5, w: float = 0.5, stream=None) -> None:
        echo_allreduce_sim(inputs, outputs, self.handle, self.n, self.P, bits, self.group,
                           eta, alpha_long, alpha_short, w, stream)

    # views of the state: [P][2][S] -> (e_long [P][n], e_short [P][n])
    def ema_views(self):
        S = int(self.layout.state_stride)
        st = self.state.view(self.P, 2, S)
        return st[:, 0, :self.n], st[:, 1, :self.n]

    def payload_views(self, bits: int):
        """(a2a_codes [P][G][cb], a2a_params [P][G] int32, gather_codes [G][cb], gather_params [G])."""
        L = echo_query_layout(self.n, self.P, self.group, self.max_bits, bits)
        G, cb, ws = int(L.groups), int(L.code_bytes), self.workspace
        a2a_c = ws[L.a2a_codes_offset:L.a2a_codes_offset + self.P * G * cb].view(self.P, G, cb)
        a2a_p = ws[L.a2a_params_offset:L.a2a_params_offset + self.P * G * 4].view(torch.int32).view(self.P, G)
        g_c = ws[L.gather_codes_offset:L.gather_codes_offset + G * cb].view(G, cb)
        g_p = ws[L.gather_params_offset:L.gather_params_offset + G * 4].view(torch.int32)
        return a2a_c, a2a_p, g_c, g_p

    def status(self, stream=None):
        return echo_get_status(self.handle, stream)

    def close(self) -> None:
        if self.handle is not None:
            echo_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ----------------------------------------------------------------- one rank of a multi-GPU call

def echo_query_rank_layout(n: int, P: int, rank: int, group: int, max_bits: int, bits: int) -> EchoRankLayout:
    out = EchoRankLayout()
    _check(lib().echo_query_rank_layout(n, P, rank, group, max_bits, bits, ctypes.byref(out)),
           "echo_query_rank_layout")
    return out


def echo_init_rank(n: int, P: int, rank: int, group: int, max_bits: int, state, workspace,
                   stream=None) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(lib().echo_init_rank(ctypes.byref(h), n, P, rank, group, max_bits, _ptr(state), _ptr(workspace),
                                _stream(stream)), "echo_init_rank")
    return h


def echo_rank_quantize(x, st, bits: int, eta: float, alpha_long: float, alpha_short: float, w: float,
                       stream=None) -> None:
    _check(lib().echo_rank_quantize(_ptr(x), st, bits, eta, alpha_long, alpha_short, w, _stream(stream)),
           "echo_rank_quantize")


def echo_rank_reduce(x, out, st, bits: int, eta: float, alpha_long: float, alpha_short: float, w: float,
                     stream=None) -> None:
    _check(lib().echo_rank_reduce(_ptr(x), _ptr(out), st, bits, eta, alpha_long, alpha_short, w, _stream(stream)),
           "echo_rank_reduce")


def echo_rank_decode(out, st, bits: int, stream=None) -> None:
    _check(lib().echo_rank_decode(_ptr(out), st, bits, _stream(stream)), "echo_rank_decode")


def echo_rank_quantize_chunk(x, st, bits: int, eta: float, alpha_long: float, alpha_short: float, w: float,
                             chunk: int, chunks: int, stream=None) -> None:
    _check(lib().echo_rank_quantize_chunk(_ptr(x), st, bits, eta, alpha_long, alpha_short, w, chunk, chunks,
                                          _stream(stream)), "echo_rank_quantize_chunk")


def echo_rank_reduce_chunk(x, out, st, bits: int, eta: float, alpha_long: float, alpha_short: float, w: float,
                           chunk: int, chunks: int, stream=None) -> None:
    _check(lib().echo_rank_reduce_chunk(_ptr(x), _ptr(out), st, bits, eta, alpha_long, alpha_short, w, chunk,
                                        chunks, _stream(stream)), "echo_rank_reduce_chunk")


def echo_rank_decode_chunk(out, st, bits: int, chunk: int, chunks: int, stream=None) -> None:
    _check(lib().echo_rank_decode_chunk(_ptr(out), st, bits, chunk, chunks, _stream(stream)),
           "echo_rank_decode_chunk")


def echo_query_chunk(n: int, P: int, group: int, owner: int, chunk: int, chunks: int):
    """(first, count): owner's part of chunk `chunk` of `chunks`, in groups,
    relative to the owner's first group."""
    first, count = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().echo_query_chunk(n, P, group, owner, chunk, chunks, ctypes.byref(first), ctypes.byref(count)),
           "echo_query_chunk")
    return int(first.value), int(count.value)


class ExchangePlan:
    """Views of one rank's workspace for the two exchanges of a multi-GPU
    call and their split sizes, in the argument order of
    torch.distributed.all_to_all_single / all_gather_into_tensor. Built from
    the library's layouts alone, so it serves a workspace on any device."""

    def __init__(self, workspace: torch.Tensor, n: int, P: int, rank: int, group: int, max_bits: int, bits: int):
        L = echo_query_rank_layout(n, P, rank, group, max_bits, bits)
        segs = [int(echo_query_rank_layout(n, P, s, group, max_bits, bits).seg_groups) for s in range(P)]
        G, seg, sm, cb = int(L.groups), int(L.seg_groups), int(L.seg_max), int(L.code_bytes)
        ws = workspace

        def u8(off, nbytes):
            return ws[int(off):int(off) + nbytes]

        def i32(off, count):
            return ws[int(off):int(off) + 4 * count].view(torch.int32)

        self.layout = L
        self.send_codes = u8(L.send_codes_offset, G * cb)
        self.send_params = i32(L.send_params_offset, G)
        self.recv_codes = u8(L.recv_codes_offset, P * seg * cb)
        self.recv_params = i32(L.recv_params_offset, P * seg)
        self.codes_in_splits = [g * cb for g in segs]      # to owner s: its segment of this rank's row
        self.codes_out_splits = [seg * cb] * P             # from every rank: this owner's segment
        self.params_in_splits = list(segs)
        self.params_out_splits = [seg] * P
        self.gsend_codes = u8(L.gsend_codes_offset, sm * cb)
        self.gsend_params = i32(L.gsend_params_offset, sm)
        self.grecv_codes = u8(L.grecv_codes_offset, P * sm * cb)
        self.grecv_params = i32(L.grecv_params_offset, P * sm)
        self._args = (n, P, rank, group, cb, sm)
        self._segs = segs
        self._seg_begin = [int(echo_query_rank_layout(n, P, s, group, max_bits, bits).seg_begin) for s in range(P)]
        self._chunks = {}

    def chunk_pieces(self, chunk: int, chunks: int):
        """Views of this rank's buffers for chunk `chunk` of `chunks` (the
        layout echo_rank_quantize_chunk & co. document): per peer, what to
        send and where to receive, as (codes, params) view pairs.

        a2a_send[s] / a2a_recv[r]: this rank's send slots for owner s's part;
        the slots of this owner's recv row r where rank r's part lands.
        ag_send: this owner's part of its gsend buffer; ag_recv[o]: the slots
        of gathered row o where owner o's part lands."""
        key = (chunk, chunks)
        if key not in self._chunks:
            n, P, rank, group, cb, sm = self._args
            parts = [echo_query_chunk(n, P, group, s, chunk, chunks) for s in range(P)]
            seg = self._segs[rank]
            f_me, c_me = parts[rank]

            def cp(codes, params, slot, count):
                return codes[slot * cb:(slot + count) * cb], params[slot:slot + count]

            a2a_send = [cp(self.send_codes, self.send_params, self._seg_begin[s] + parts[s][0], parts[s][1])
                        for s in range(P)]
            a2a_recv = [cp(self.recv_codes, self.recv_params, r * seg + f_me, c_me) for r in range(P)]
            ag_send = cp(self.gsend_codes, self.gsend_params, f_me, c_me)
            ag_recv = [cp(self.grecv_codes, self.grecv_params, o * sm + parts[o][0], parts[o][1]) for o in range(P)]
            self._chunks[key] = (a2a_send, a2a_recv, ag_send, ag_recv)
        return self._chunks[key]


def exchange_all_to_all(plan: ExchangePlan, group=None) -> None:
    """The all-to-all of the packed payload (codes and parameters)."""
    import torch.distributed as dist
    dist.all_to_all_single(plan.recv_codes, plan.send_codes, plan.codes_out_splits, plan.codes_in_splits,
                           group=group)
    dist.all_to_all_single(plan.recv_params, plan.send_params, plan.params_out_splits, plan.params_in_splits,
                           group=group)


def exchange_all_gather(plan: ExchangePlan, group=None) -> None:
    """The all-gather of the owners' requantized segments."""
    import torch.distributed as dist
    dist.all_gather_into_tensor(plan.grecv_codes, plan.gsend_codes, group=group)
    dist.all_gather_into_tensor(plan.grecv_params, plan.gsend_params, group=group)


def exchange_chunk(plan: ExchangePlan, step: str, chunk: int, chunks: int, rank: int, group=None):
    """One chunk's exchange as point-to-point sends and receives (the pieces
    of a chunk are not contiguous across peers, and their sizes differ by a
    group or so): `step` "all_to_all" sends this rank's part for every other
    owner and receives every other rank's part of its own segment;
    "all_gather" sends its own part to every other rank, receives every other
    owner's part, and copies its own part into its gathered row. Enqueued on
    the current stream; returns the requests (their wait() orders that
    stream after the transfers)."""
    import torch.distributed as dist
    a2a_send, a2a_recv, ag_send, ag_recv = plan.chunk_pieces(chunk, chunks)
    P = len(a2a_send)
    ops = []
    for peer in range(P):
        if peer == rank:
            continue
        # point-to-point ops name the peer by its global rank
        dst = peer if group is None else dist.get_global_rank(group, peer)
        if step == "all_to_all":
            pieces = ((a2a_send[peer], a2a_recv[peer]),)
        elif step == "all_gather":
            pieces = ((ag_send, ag_recv[peer]),)
        else:
            raise ValueError(step)
        for send, recv in pieces:
            for k in range(2):   # codes, then parameter words
                if send[k].numel():
                    ops.append(dist.P2POp(dist.isend, send[k], dst, group))
                if recv[k].numel():
                    ops.append(dist.P2POp(dist.irecv, recv[k], dst, group))
    if step == "all_gather":
        for k in range(2):
            if ag_send[k].numel():
                ag_recv[rank][k].copy_(ag_send[k])
    return dist.batch_isend_irecv(ops) if ops else []


class EchoRank:
    """One rank of a multi-GPU Echo all-reduce (one process per GPU): owns,
    through torch, this rank's EMA state and workspace, and the library
    handle. `allreduce` runs the five steps with torch.distributed
    collectives between the kernels (NCCL for CUDA tensors)."""

    def __init__(self, n: int, P: int, rank: int, group: int = 128, max_bits: int = 4, feedback: bool = True,
                 device=None, stream=None, quantizer: int = ECHO_QUANT_DIRECTED):
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.n, self.P, self.rank, self.group, self.max_bits = n, P, rank, group, max_bits
        L = echo_query_rank_layout(n, P, rank, group, max_bits, max_bits)
        self.workspace = torch.empty(int(L.workspace_bytes), dtype=torch.uint8, device=device)
        self.state = torch.empty(int(L.state_bytes) // 4, dtype=torch.float32, device=device) if feedback else None
        self.handle = echo_init_rank(n, P, rank, group, max_bits, self.state, self.workspace, stream)
        if quantizer != ECHO_QUANT_DIRECTED:
            echo_set_quantizer(self.handle, quantizer)
        self._plans = {}
        self._comm_stream = None   # the chunked call's communication stream, made on first use

    def plan(self, bits: int) -> ExchangePlan:
        if bits not in self._plans:
            self._plans[bits] = ExchangePlan(self.workspace, self.n, self.P, self.rank, self.group, self.max_bits,
                                             bits)
        return self._plans[bits]

    def quantize(self, x, bits=4, eta=1.0, alpha_long=0.05, alpha_short=0.5, w=0.5, stream=None) -> None:
        echo_rank_quantize(x, self.handle, bits, eta, alpha_long, alpha_short, w, stream)

    def reduce(self, x, out, bits=4, eta=1.0, alpha_long=0.05, alpha_short=0.5, w=0.5, stream=None) -> None:
        echo_rank_reduce(x, out, self.handle, bits, eta, alpha_long, alpha_short, w, stream)

    def decode(self, out, bits=4, stream=None) -> None:
        echo_rank_decode(out, self.handle, bits, stream)

    def quantize_chunk(self, x, chunk, chunks, bits=4, eta=1.0, alpha_long=0.05, alpha_short=0.5, w=0.5,
                       stream=None) -> None:
        echo_rank_quantize_chunk(x, self.handle, bits, eta, alpha_long, alpha_short, w, chunk, chunks, stream)

    def reduce_chunk(self, x, out, chunk, chunks, bits=4, eta=1.0, alpha_long=0.05, alpha_short=0.5, w=0.5,
                     stream=None) -> None:
        echo_rank_reduce_chunk(x, out, self.handle, bits, eta, alpha_long, alpha_short, w, chunk, chunks, stream)

    def decode_chunk(self, out, chunk, chunks, bits=4, stream=None) -> None:
        echo_rank_decode_chunk(out, self.handle, bits, chunk, chunks, stream)

    def allreduce(self, x, out, bits=4, eta=1.0, alpha_long=0.05, alpha_short=0.5, w=0.5, group=None,
                  chunks: int = 1, comm_stream=None) -> None:
        """Steps 1-5 with the process group's exchanges in between (every rank
        of the group calls this). chunks = 1: on torch's current stream, the
        collectives between the kernels. chunks > 1: the call in column
        chunks (see echo_rank_quantize_chunk), chunk c's exchanges on
        `comm_stream` (if None, a stream this handle creates once and keeps)
        overlapping chunk c + 1's kernels on the current stream, ordered by
        CUDA events; the current stream continues once the last chunk is
        decoded."""
        fb = (eta, alpha_long, alpha_short, w)
        if chunks <= 1 or self.P == 1:
            self.quantize(x, bits, *fb)
            if self.P > 1:
                exchange_all_to_all(self.plan(bits), group)
            self.reduce(x, out, bits, *fb)
            if self.P > 1:
                exchange_all_gather(self.plan(bits), group)
                self.decode(out, bits)
            return
        plan = self.plan(bits)
        if comm_stream is None:
            if self._comm_stream is None:
                self._comm_stream = torch.cuda.Stream(device=self.workspace.device)
            comm_stream = self._comm_stream

        def comm(step, c):
            for req in exchange_chunk(plan, step, c, chunks, self.rank, group):
                req.wait()

        run_chunked([self], [x], [out], bits, fb, chunks, comm, comm_stream)

    def ema_views(self):
        """(e_long [n], e_short [n]) of this rank."""
        S = -(-self.n // self.group) * self.group
        st = self.state.view(2, S)
        return st[0, :self.n], st[1, :self.n]

    def status(self, stream=None):
        return echo_get_status(self.handle, stream)

    def close(self) -> None:
        if self.handle is not None:
            echo_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def run_chunked(ranks: Sequence["EchoRank"], xs: Sequence, outs: Sequence, bits: int, fb, chunks: int, comm,
                comm_stream=None) -> None:
    """The chunked schedule of a multi-GPU call for the ranks this process
    drives (one per process on P GPUs; all P of them on one GPU in tests and
    one-GPU benchmarks). Compute stream = torch's current stream; chunk c's
    all-to-all runs on the communication stream once its quantize is done,
    its reduce once that all-to-all is done, its all-gather once the reduce
    is done, its decode once the all-gather is done; the compute stream
    issues quantize(c), reduce(c - 1), decode(c - 2) in turn, so one chunk's
    transfers overlap the neighbouring chunks' kernels. `comm(step, c)`
    enqueues chunk c's exchange on the current stream (called with the
    communication stream current)."""
    compute = torch.cuda.current_stream()
    cs = comm_stream if comm_stream is not None else torch.cuda.Stream(device=compute.device)
    ev = {name: [torch.cuda.Event() for _ in range(chunks)] for name in ("q", "a", "r", "g")}
    cs.wait_stream(compute)   # the inputs and the previous call's work
    for t in range(chunks + 2):
        c = t
        if c < chunks:
            for rk, x in zip(ranks, xs):
                rk.quantize_chunk(x, c, chunks, bits, *fb, stream=compute)
            ev["q"][c].record(compute)
            with torch.cuda.stream(cs):
                cs.wait_event(ev["q"][c])
                comm("all_to_all", c)
                ev["a"][c].record(cs)
        c = t - 1
        if 0 <= c < chunks:
            compute.wait_event(ev["a"][c])
            for rk, x in zip(ranks, xs):
                rk.reduce_chunk(x, None, c, chunks, bits, *fb, stream=compute)
            ev["r"][c].record(compute)
            with torch.cuda.stream(cs):
                cs.wait_event(ev["r"][c])
                comm("all_gather", c)
                ev["g"][c].record(cs)
        c = t - 2
        if 0 <= c < chunks:
            compute.wait_event(ev["g"][c])
            for rk, y in zip(ranks, outs):
                rk.decode_chunk(y, c, chunks, bits, stream=compute)
    compute.wait_stream(cs)


def exchange_in_process(plans: Sequence[ExchangePlan], step: str) -> None:
    """Both exchanges for P ranks held by one process on one device (tests and
    one-GPU benchmarks of the rank kernels): stream-ordered copies with the
    semantics of all_to_all_single (`step` "all_to_all": chunk `dst` of the
    sender's input into chunk `src` of the receiver's output) and of
    all_gather_into_tensor (`step` "all_gather": rank order), over the same
    views and split sizes the collectives receive."""
    if step == "all_to_all":
        for dst, pd in enumerate(plans):
            for src, ps in enumerate(plans):
                for send, recv, ins, outs in ((ps.send_codes, pd.recv_codes, ps.codes_in_splits, pd.codes_out_splits),
                                              (ps.send_params, pd.recv_params, ps.params_in_splits,
                                               pd.params_out_splits)):
                    ln = ins[dst]
                    if ln != outs[src]:
                        raise ValueError("exchange plans of different messages")
                    a, b = sum(ins[:dst]), sum(outs[:src])
                    recv[b:b + ln].copy_(send[a:a + ln])
    elif step == "all_gather":
        for pd in plans:
            for s, ps in enumerate(plans):
                for send, recv in ((ps.gsend_codes, pd.grecv_codes), (ps.gsend_params, pd.grecv_params)):
                    k = send.numel()
                    recv[s * k:(s + 1) * k].copy_(send)
    else:
        raise ValueError(step)


def exchange_chunk_in_process(plans: Sequence[ExchangePlan], step: str, chunk: int, chunks: int) -> None:
    """exchange_chunk for P ranks held by one process on one device:
    stream-ordered copies of the same pieces (tests and one-GPU benchmarks)."""
    pieces = [pl.chunk_pieces(chunk, chunks) for pl in plans]
    P = len(plans)
    for dst in range(P):
        for src in range(P):
            if step == "all_to_all":
                if src == dst:
                    continue
                send, recv = pieces[src][0][dst], pieces[dst][1][src]
            elif step == "all_gather":
                send, recv = pieces[src][2], pieces[dst][3][src]
            else:
                raise ValueError(step)
            for k in range(2):
                if send[k].numel() != recv[k].numel():
                    raise ValueError("chunk pieces of different messages")
                if send[k].numel():
                    recv[k].copy_(send[k])
