"""Python access to the oracle (``echo_oracle.c``) through ctypes.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by the package smoke check
and by the benchmark's CPU-baseline leg, never by the product path.

The arrays follow the oracle's own layout: rank-major ``[P][ld]`` with
``ld = jc * group`` elements, for the group columns ``[j0, j0 + jc)`` of a
message of ``n_total`` elements per rank. Everything is numpy on the host.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np

from . import build as _build

RN, RD, RU = 0, 1, 2
FLAG_RANGE = 1
Q_DIRECTED, Q_NEAREST, Q_INT_ZERO = 0, 1, 2   # quantizer forms (readings R4, R10, R11)

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        # ECHO_ORACLE_LIB lets the mutation test load a deliberately broken
        # copy of the oracle; normally the in-tree build is used
        path = os.environ.get("ECHO_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        L.oracle_f32_to_f16.argtypes = [ctypes.c_float, ctypes.c_int]
        L.oracle_f32_to_f16.restype = ctypes.c_uint16
        L.oracle_f16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_f16_to_f32.restype = ctypes.c_float
        L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_f32.restype = ctypes.c_float
        L.oracle_quantize_group.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P, P, P]
        L.oracle_quantize_group.restype = ctypes.c_uint32
        L.oracle_pack_codes.argtypes = [P, ctypes.c_int, ctypes.c_int, P]
        L.oracle_pack_codes.restype = None
        L.oracle_unpack_codes.argtypes = [P, ctypes.c_int, ctypes.c_int, P]
        L.oracle_unpack_codes.restype = None
        L.oracle_segment_begin.argtypes = [ctypes.c_int, ctypes.c_longlong, ctypes.c_int]
        L.oracle_segment_begin.restype = ctypes.c_longlong
        L.oracle_owner.argtypes = [ctypes.c_longlong, ctypes.c_longlong, ctypes.c_int]
        L.oracle_owner.restype = ctypes.c_int
        L.oracle_compensation.argtypes = [ctypes.c_float] * 4
        L.oracle_compensation.restype = ctypes.c_float
        L.oracle_ema_update.argtypes = [P, P, ctypes.c_longlong, ctypes.c_float]
        L.oracle_ema_update.restype = None
        L.oracle_echo_allreduce.argtypes = [
            ctypes.c_int, ctypes.c_longlong, ctypes.c_int, ctypes.c_int,
            ctypes.c_longlong, ctypes.c_longlong,
            P, P, P, P,
            ctypes.c_float, ctypes.c_float, ctypes.c_float, ctypes.c_float,
            P, P, P, P, P, P, P, P,
        ]
        L.oracle_echo_allreduce.restype = ctypes.c_int
        L.oracle_quantize_group_q.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, P]
        L.oracle_quantize_group_q.restype = ctypes.c_uint32
        L.oracle_echo_allreduce_q.argtypes = [
            ctypes.c_int, ctypes.c_longlong, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_longlong, ctypes.c_longlong,
            P, P, P, P,
            ctypes.c_float, ctypes.c_float, ctypes.c_float, ctypes.c_float,
            P, P, P, P, P, P, P, P,
        ]
        L.oracle_echo_allreduce_q.restype = ctypes.c_int
        L.oracle_bf16_allreduce.argtypes = [ctypes.c_int, ctypes.c_longlong, P, P]
        L.oracle_bf16_allreduce.restype = None
        _lib = L
    return _lib


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- scalars

def f32_to_f16(x: float, mode: int = RN) -> int:
    return int(lib().oracle_f32_to_f16(ctypes.c_float(x), mode))


def f16_to_f32(h: int) -> float:
    return float(lib().oracle_f16_to_f32(h))


def f32_to_bf16(x: float) -> int:
    return int(lib().oracle_f32_to_bf16(ctypes.c_float(x)))


def bf16_to_f32(b: int) -> float:
    return float(lib().oracle_bf16_to_f32(b))


def owner(j: int, G: int, P: int) -> int:
    return int(lib().oracle_owner(j, G, P))


def segment_begin(s: int, G: int, P: int) -> int:
    return int(lib().oracle_segment_begin(s, G, P))


def compensation(e_long: float, e_short: float, eta: float, w: float) -> float:
    return float(lib().oracle_compensation(e_long, e_short, eta, w))


def ema_update(e: np.ndarray, rho: np.ndarray, alpha: float) -> None:
    assert e.dtype == np.float32 and rho.dtype == np.float32 and e.shape == rho.shape
    lib().oracle_ema_update(_ptr(e), _ptr(rho), e.size, alpha)


@dataclass
class GroupQuant:
    codes: np.ndarray   # uint8, one code per element
    s_bits: int
    z_bits: int
    vhat: np.ndarray    # float32 dequantized values
    flag: int


def quantize_group(v: np.ndarray, bits: int, quantizer: int = Q_DIRECTED) -> GroupQuant:
    """One group through the quantizer form ``quantizer`` (Q_DIRECTED: fp16
    zero rounded down and step rounded up; Q_NEAREST: both rounded to
    nearest; Q_INT_ZERO: integer zero point, ``z_bits`` then holds zp)."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    m = v.size
    codes = np.zeros(m, np.uint8)
    vhat = np.zeros(m, np.float32)
    s = ctypes.c_uint16()
    z = ctypes.c_uint16()
    if quantizer == Q_DIRECTED:
        flag = lib().oracle_quantize_group(_ptr(v), m, bits, _ptr(codes), ctypes.byref(s),
                                           ctypes.byref(z), _ptr(vhat))
    else:
        flag = lib().oracle_quantize_group_q(_ptr(v), m, bits, quantizer, _ptr(codes), ctypes.byref(s),
                                             ctypes.byref(z), _ptr(vhat))
    return GroupQuant(codes, int(s.value), int(z.value), vhat, int(flag))


def pack_codes(codes: np.ndarray, group: int, bits: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.zeros(group * bits // 8, np.uint8)
    lib().oracle_pack_codes(_ptr(codes), group, bits, _ptr(out))
    return out


def unpack_codes(packed: np.ndarray, group: int, bits: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    out = np.zeros(group, np.uint8)
    lib().oracle_unpack_codes(_ptr(packed), group, bits, _ptr(out))
    return out


# ---------------------------------------------------------------- one call

@dataclass
class CallResult:
    y: np.ndarray               # [P][ld] uint16 bf16 bits
    a2a_codes: np.ndarray       # [P][jc][group*bits/8] uint8
    a2a_params: np.ndarray      # [P][jc][2] uint16 {s, z}
    gather_codes: np.ndarray    # [jc][group*bits/8] uint8
    gather_params: np.ndarray   # [jc][2] uint16
    xprime: Optional[np.ndarray]
    rho: Optional[np.ndarray]
    passes: Optional[np.ndarray]
    flags: int


def echo_allreduce(x: np.ndarray, *, n_total: int, group: int, bits: int,
                   e_long: Optional[np.ndarray] = None, e_short: Optional[np.ndarray] = None,
                   eta: float = 1.0, alpha_long: float = 0.05, alpha_short: float = 0.5,
                   w: float = 0.5, j0: int = 0, jc: Optional[int] = None,
                   debug: bool = False, quantizer: int = Q_DIRECTED) -> CallResult:
    """Run one oracle call on the columns ``[j0, j0 + jc)``.

    ``x`` is ``[P][jc*group]`` uint16 (bf16 bit patterns). ``e_long`` and
    ``e_short`` (``[P][jc*group]`` float32) are updated in place; pass both or
    neither. ``quantizer`` selects the quantizer form (see quantize_group).
    """
    x = np.ascontiguousarray(x, dtype=np.uint16)
    P, ld = x.shape
    G = (n_total + group - 1) // group
    if jc is None:
        jc = G - j0
    assert ld == jc * group, (ld, jc, group)
    if e_long is not None or e_short is not None:
        assert e_long is not None and e_short is not None
        for e in (e_long, e_short):
            assert e.dtype == np.float32 and e.shape == (P, ld) and e.flags["C_CONTIGUOUS"]
    cb = group * bits // 8
    y = np.zeros((P, ld), np.uint16)
    a2a_c = np.zeros((P, jc, cb), np.uint8)
    a2a_p = np.zeros((P, jc, 2), np.uint16)
    g_c = np.zeros((jc, cb), np.uint8)
    g_p = np.zeros((jc, 2), np.uint16)
    xp = np.zeros((P, ld), np.float32) if debug else None
    rho = np.zeros((P, ld), np.float32) if debug else None
    passes = np.zeros((P, ld), np.uint8) if debug else None
    flags = ctypes.c_uint32(0)
    if quantizer == Q_DIRECTED:
        rc = lib().oracle_echo_allreduce(
            P, n_total, group, bits, j0, jc, _ptr(x), _ptr(y), _ptr(e_long), _ptr(e_short),
            eta, alpha_long, alpha_short, w, _ptr(a2a_c), _ptr(a2a_p), _ptr(g_c), _ptr(g_p),
            _ptr(xp), _ptr(rho), _ptr(passes), ctypes.byref(flags))
    else:
        rc = lib().oracle_echo_allreduce_q(
            P, n_total, group, bits, quantizer, j0, jc, _ptr(x), _ptr(y), _ptr(e_long), _ptr(e_short),
            eta, alpha_long, alpha_short, w, _ptr(a2a_c), _ptr(a2a_p), _ptr(g_c), _ptr(g_p),
            _ptr(xp), _ptr(rho), _ptr(passes), ctypes.byref(flags))
    if rc != 0:
        raise ValueError("oracle_echo_allreduce rejected its arguments")
    return CallResult(y, a2a_c, a2a_p, g_c, g_p, xp, rho, passes, int(flags.value))


def library_path() -> str:
    return os.path.abspath(_build.LIB)


def bf16_allreduce(x: np.ndarray) -> np.ndarray:
    """The 16-bit baseline all-reduce over the rows of ``x`` ([P][n] uint16
    bf16 bit patterns): every row of the result is bf16_rn of the binary32
    sum in rank order."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    P, n = x.shape
    y = np.zeros((P, n), np.uint16)
    lib().oracle_bf16_allreduce(P, n, _ptr(x), _ptr(y))
    return y
