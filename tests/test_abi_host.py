"""Host-side checks of the C ABI (no GPU needed, no kernel launched).

* the library builds for sm_100a and loads;
* it exports every function include/echo.h declares;
* size and layout queries follow the documented layout;
* bad arguments are rejected with ECHO_EINVAL before any CUDA call, and with
  no GPU present a valid init fails loudly with ECHO_ECUDA.
"""
import ctypes
import os
import re

import pytest

import bit_error_compensated_group_b200 as E
from bit_error_compensated_group_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    _build.build()
    return E.lib()


def declared_functions():
    with open(os.path.join(ROOT, "include", "echo.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"ECHO_API\s+[\w\s\*]+?\b(echo_\w+)\s*\(", text)))


def test_exports_every_declared_function(L):
    names = declared_functions()
    assert len(names) >= 11, names
    for name in names:
        assert hasattr(L, name), name
    # nothing but the C ABI is exported
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", _build.LIB], capture_output=True, text=True).stdout
    exported = sorted(line.split()[-1] for line in out.splitlines() if " T " in line)
    assert exported == names


def _G(n, g):
    return -(-n // g)


@pytest.mark.parametrize("n,P,g,mb", [(4096, 2, 128, 4), (1000, 3, 32, 8), (1 << 29, 8, 128, 4), (777, 64, 256, 8)])
def test_layout(L, n, P, g, mb):
    G = _G(n, g)
    assert E.echo_state_bytes(n, P, g) == P * 2 * G * g * 4
    for bits in (4, 8):
        if bits > mb:
            with pytest.raises(E.EchoError):
                E.echo_query_layout(n, P, g, mb, bits)
            continue
        lay = E.echo_query_layout(n, P, g, mb, bits)
        assert lay.groups == G and lay.state_stride == G * g
        assert lay.code_bytes == g * bits // 8
        regions = [(lay.flags_offset, 4), (lay.a2a_codes_offset, P * G * g * mb // 8),
                   (lay.a2a_params_offset, P * G * 4), (lay.gather_codes_offset, G * g * mb // 8),
                   (lay.gather_params_offset, G * 4)]
        for (o1, s1), (o2, _) in zip(regions, regions[1:]):
            assert o1 % 256 == 0 and o1 + s1 <= o2
        assert regions[-1][0] + regions[-1][1] <= lay.workspace_bytes
        assert lay.workspace_bytes == E.echo_workspace_bytes(n, P, g, mb)


@pytest.mark.parametrize("n,P,g,mb", [(0, 2, 128, 4), (10, 0, 128, 4), (10, 65, 128, 4),
                                      (10, 2, 48, 4), (10, 2, 128, 5), (1 << 41, 2, 128, 4)])
def test_bad_sizes(L, n, P, g, mb):
    assert E.echo_workspace_bytes(n, P, g, mb) == 0
    lay = E.EchoLayout()
    assert L.echo_query_layout(n, P, g, mb, 4, ctypes.byref(lay)) == E.ECHO_EINVAL
    h = ctypes.c_void_p()
    assert L.echo_init_state(ctypes.byref(h), n, P, g, mb, None, 256, None) == E.ECHO_EINVAL
    assert h.value is None


def test_init_rejects_bad_pointers_before_cuda(L):
    h = ctypes.c_void_p()
    # no workspace / misaligned workspace / misaligned state: rejected on the host
    assert L.echo_init_state(ctypes.byref(h), 1024, 2, 128, 4, None, None, None) == E.ECHO_EINVAL
    assert L.echo_init_state(ctypes.byref(h), 1024, 2, 128, 4, None, 4096 + 8, None) == E.ECHO_EINVAL
    assert L.echo_init_state(ctypes.byref(h), 1024, 2, 128, 4, 4096 + 4, 4096, None) == E.ECHO_EINVAL
    assert L.echo_init_state(None, 1024, 2, 128, 4, None, 4096, None) == E.ECHO_EINVAL


def test_calls_reject_missing_handle(L):
    arr = (ctypes.c_void_p * 2)(4096, 8192)
    assert L.echo_allreduce_sim(arr, arr, None, 1024, 2, 4, 128, 1.0, 0.05, 0.5, 0.5, None) == E.ECHO_EINVAL
    assert L.echo_allreduce_sim_range(arr, arr, None, 1024, 2, 4, 128, 1.0, 0.05, 0.5, 0.5, 0, 8,
                                      None) == E.ECHO_EINVAL
    assert L.echo_allreduce_sim_host(arr, None, arr, arr, None, 1024, 2, 4, 128, 1.0, 0.05, 0.5, 0.5, 0,
                                     None, None, None) == E.ECHO_EINVAL
    assert L.echo_phase_quantize(arr, None, 4, 1.0, 0.05, 0.5, 0.5, None) == E.ECHO_EINVAL
    assert L.echo_phase_reduce(arr, arr, None, 4, 1.0, 0.05, 0.5, 0.5, None) == E.ECHO_EINVAL
    assert L.echo_phase_gather(arr, None, 4, None) == E.ECHO_EINVAL
    assert L.echo_get_status(None, None, None) == E.ECHO_EINVAL
    assert L.echo_set_quantizer(None, E.ECHO_QUANT_NEAREST) == E.ECHO_EINVAL
    assert L.echo_set_wait_limit(None, 1000000) == E.ECHO_EINVAL
    assert L.echo_get_wait_limit(None) == 0
    assert L.echo_check_watchdog(None, 0, None) == E.ECHO_EINVAL
    assert L.echo_free(None) == E.ECHO_OK


def test_status_strings(L):
    for code in range(6):
        assert E.echo_status_string(code)
    assert E.echo_status_string(99) == "unknown status"


def test_no_gpu_fails_loudly(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p()
    rc = L.echo_init_state(ctypes.byref(h), 1024, 2, 128, 4, None, 4096, None)
    assert rc == E.ECHO_ECUDA
    with pytest.raises(E.EchoError) as ei:
        E.echo_init_state(1024, 2, 128, 4, None, 4096, stream=0)
    assert ei.value.status == E.ECHO_ECUDA


@pytest.mark.parametrize("n,P,g,mb,bits", [(1000, 3, 64, 8, 4), (1 << 29, 8, 128, 4, 4), (3 * 128, 4, 128, 4, 4),
                                           (777, 5, 32, 8, 8), (1, 2, 32, 4, 4)])
def test_rank_layout(L, n, P, g, mb, bits):
    """One rank's layout of a multi-GPU call: the segments tile [0, G) in rank
    order, seg_max is the largest, and the workspace regions are 256-byte
    aligned, disjoint and as large as the exchange needs."""
    G = _G(n, g)
    cb, cbm = g * bits // 8, g * mb // 8
    lays = [E.echo_query_rank_layout(n, P, r, g, mb, bits) for r in range(P)]
    begin = 0
    for r, lay in enumerate(lays):
        assert lay.groups == G and lay.code_bytes == cb
        assert lay.seg_begin == begin == r * G // P
        assert lay.seg_groups == (r + 1) * G // P - r * G // P
        begin += lay.seg_groups
        assert lay.seg_max == max(l.seg_groups for l in lays)
        assert lay.state_bytes == 2 * G * g * 4
        seg, sm = lay.seg_groups, lay.seg_max
        regions = [(lay.flags_offset, 4), (lay.send_codes_offset, G * cbm), (lay.send_params_offset, G * 4),
                   (lay.recv_codes_offset, P * seg * cbm), (lay.recv_params_offset, P * seg * 4),
                   (lay.gsend_codes_offset, sm * cbm), (lay.gsend_params_offset, sm * 4),
                   (lay.grecv_codes_offset, P * sm * cbm), (lay.grecv_params_offset, P * sm * 4)]
        for (o1, s1), (o2, _) in zip(regions, regions[1:]):
            assert o1 % 256 == 0 and o1 + s1 <= o2
        assert regions[-1][0] + regions[-1][1] <= lay.workspace_bytes
    assert begin == G


def test_rank_calls_reject_bad_arguments(L):
    lay = E.EchoRankLayout()
    assert L.echo_query_rank_layout(1000, 3, 3, 64, 4, 4, ctypes.byref(lay)) == E.ECHO_EINVAL   # rank >= P
    assert L.echo_query_rank_layout(1000, 3, -1, 64, 4, 4, ctypes.byref(lay)) == E.ECHO_EINVAL
    assert L.echo_query_rank_layout(1000, 3, 0, 64, 4, 8, ctypes.byref(lay)) == E.ECHO_EINVAL   # bits > max_bits
    h = ctypes.c_void_p()
    assert L.echo_init_rank(ctypes.byref(h), 1000, 3, 5, 64, 4, None, 4096, None) == E.ECHO_EINVAL
    assert L.echo_init_rank(ctypes.byref(h), 1000, 3, 1, 64, 4, None, 4096 + 8, None) == E.ECHO_EINVAL
    assert L.echo_rank_quantize(4096, None, 4, 1.0, 0.05, 0.5, 0.5, None) == E.ECHO_EINVAL
    assert L.echo_rank_reduce(4096, 4096, None, 4, 1.0, 0.05, 0.5, 0.5, None) == E.ECHO_EINVAL
    assert L.echo_rank_decode(4096, None, 4, None) == E.ECHO_EINVAL
    assert L.echo_rank_quantize_chunk(4096, None, 4, 1.0, 0.05, 0.5, 0.5, 0, 2, None) == E.ECHO_EINVAL
    assert L.echo_rank_reduce_chunk(4096, 4096, None, 4, 1.0, 0.05, 0.5, 0.5, 0, 2, None) == E.ECHO_EINVAL
    assert L.echo_rank_decode_chunk(4096, None, 4, 0, 2, None) == E.ECHO_EINVAL
    assert h.value is None


@pytest.mark.parametrize("n,P,g", [(1000, 3, 64), (1 << 29, 8, 128), (3 * 128, 4, 128), (777, 5, 32)])
@pytest.mark.parametrize("chunks", [1, 2, 3, 7, 64])
def test_chunk_parts_tile_each_segment(L, n, P, g, chunks):
    """Every owner's parts of chunks 0 .. chunks-1 tile its segment in
    order, their sizes differ by at most one group, and the last group of
    the message (in the last owner's segment) is in the last chunk."""
    G = -(-n // g)
    for s in range(P):
        seg = int(E.echo_query_rank_layout(n, P, s, g, 4, 4).seg_groups)
        parts = [E.echo_query_chunk(n, P, g, s, c, chunks) for c in range(chunks)]
        assert parts[0][0] == 0 and sum(c for _, c in parts) == seg
        for (f0, c0), (f1, _) in zip(parts, parts[1:]):
            assert f0 + c0 == f1
        sizes = [c for _, c in parts]
        assert max(sizes) - min(sizes) <= 1
    if G >= P:
        f, c = E.echo_query_chunk(n, P, g, P - 1, chunks - 1, chunks)
        seg_last = int(E.echo_query_rank_layout(n, P, P - 1, g, 4, 4).seg_groups)
        assert f + c == seg_last and c >= 1


def test_traffic_calls_reject_bad_arguments(L):
    arr = (ctypes.c_void_p * 2)(4096, 8192)
    assert L.echo_bf16_allreduce_sim(arr, arr, 0, 2, None) == E.ECHO_EINVAL        # n < 1
    assert L.echo_bf16_allreduce_sim(arr, arr, 100, 65, None) == E.ECHO_EINVAL     # P > 64
    bad = (ctypes.c_void_p * 2)(4096, 8200)
    assert L.echo_bf16_allreduce_sim(bad, arr, 100, 2, None) == E.ECHO_EINVAL      # misaligned
    assert L.echo_bf16_allreduce_sim(None, arr, 100, 2, None) == E.ECHO_EINVAL
    bt = L.echo_background_traffic
    chunk = 16384                                                                        # the copy's unit
    assert bt(4096, 4096 + 256, chunk, 500, 100, 1000, None, None) == E.ECHO_EINVAL     # overlapping
    assert bt(4096, 1 << 20, chunk + 16, 500, 100, 1000, None, None) == E.ECHO_EINVAL   # not a multiple of 16 KB
    assert bt(4096, 1 << 20, 1024, 500, 100, 1000, None, None) == E.ECHO_EINVAL         # less than one chunk
    assert bt(4096, 1 << 20, chunk, 1001, 100, 1000, None, None) == E.ECHO_EINVAL       # duty > 1000
    assert bt(4096, 1 << 20, chunk, 500, 5, 1000, None, None) == E.ECHO_EINVAL          # period too short
    assert bt(4096, 1 << 20, chunk, 500, 100, 0, None, None) == E.ECHO_EINVAL           # no duration
    assert bt(4096, 1 << 20, chunk, 0, 100, 1000, None, None) == E.ECHO_OK              # duty 0: nothing to launch


def test_chunk_query_rejects_bad_arguments(L):
    f, c = ctypes.c_int64(), ctypes.c_int64()
    for args in ((1000, 3, 64, 3, 0, 2), (1000, 3, 64, -1, 0, 2), (1000, 3, 64, 0, 2, 2), (1000, 3, 64, 0, 0, 0),
                 (1000, 3, 64, 0, 0, E.ECHO_MAX_CHUNKS + 1), (0, 3, 64, 0, 0, 1), (1000, 3, 48, 0, 0, 1)):
        assert L.echo_query_chunk(*args, ctypes.byref(f), ctypes.byref(c)) == E.ECHO_EINVAL, args
    assert L.echo_query_chunk(1000, 3, 64, 0, 0, 1, None, ctypes.byref(c)) == E.ECHO_EINVAL


def test_header_is_c_and_links(L, tmp_path):
    """include/echo.h compiles as pedantic C99 and a C program linked against
    the library gets the same host-only answers as the binding."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(r'''
#include <stdio.h>
#include "echo.h"
int main(void) {
    echo_layout L;
    echo_rank_layout R;
    if (echo_query_layout(1000, 3, 64, 8, 4, &L) != ECHO_OK) return 2;
    if (echo_query_rank_layout(1000, 3, 1, 64, 8, 4, &R) != ECHO_OK) return 3;
    printf("%zu %llu %lld %lld %llu\n", echo_state_bytes(1000, 3, 64),
           (unsigned long long)L.workspace_bytes, (long long)R.seg_begin, (long long)R.seg_groups,
           (unsigned long long)R.workspace_bytes);
    return echo_query_rank_layout(1000, 3, 3, 64, 8, 4, &R) == ECHO_EINVAL ? 0 : 4;
}
''')
    exe = tmp_path / "abi"
    lib = _build.LIB
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), lib, "-o", str(exe)], check=True)
    env = dict(os.environ, LD_LIBRARY_PATH=os.path.dirname(lib))
    out = subprocess.run([str(exe)], capture_output=True, text=True, env=env, check=True).stdout.split()
    lay = E.echo_query_layout(1000, 3, 64, 8, 4)
    rl = E.echo_query_rank_layout(1000, 3, 1, 64, 8, 4)
    assert [int(v) for v in out] == [E.echo_state_bytes(1000, 3, 64), lay.workspace_bytes, rl.seg_begin,
                                     rl.seg_groups, rl.workspace_bytes]


def test_missing_library_fails_loudly(monkeypatch):
    """Without the CUDA library the binding raises at the first call; there is
    no fallback path."""
    import bit_error_compensated_group_b200.echo as EE
    monkeypatch.setattr(EE, "_lib", None)
    monkeypatch.setattr(EE, "LIB_PATH", "/nonexistent/libecho_b200.so")
    with pytest.raises(RuntimeError, match="missing"):
        EE.echo_state_bytes(1024, 2, 128)
    with pytest.raises(RuntimeError, match="missing"):
        EE.EchoAllReduce(1024, 2, device="cpu")


def test_launch_failure_hook_toggles(L):
    assert E.echo_inject_launch_failure(True) is False
    assert E.echo_inject_launch_failure(True) is True
    assert E.echo_inject_launch_failure(False) is True
    assert E.echo_inject_launch_failure(False) is False
