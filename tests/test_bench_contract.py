"""The benchmark's JSON line: the keys its consumers read.

CPU: the reference arm (the oracle timed on the host) prints one line with
the metric, the unit, its cpu_baseline and an e2e entry of zero copies.
GPU: the main arm on a small message of the same shape family prints one line
with the roofline, the clocks, the end-to-end leg, the CPU baseline and the
launch count.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _last_json(out: str) -> dict:
    lines = [l for l in out.splitlines() if l.startswith("{")]
    assert lines, out[-2000:]
    return json.loads(lines[-1])


def test_reference_arm_line():
    sys.path.insert(0, ROOT)
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=600, check=True).stdout
    line = _last_json(out)
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["value"] > 0 and line["cpu_baseline"]["value"] == line["value"]
    import bench
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == bench.host_cores()
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"] == "p8_1GB_student_t"


@pytest.mark.gpu
def test_main_arm_line():
    out = subprocess.run([sys.executable, "bench.py", "--tokens", "2048", "--steps", "3", "--warmup", "3",
                          "--no-variants"], cwd=ROOT, capture_output=True, text=True, timeout=900, check=True).stdout
    line = _last_json(out)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "roofline_call", "clocks", "e2e",
                "gpu_launches", "cpu_baseline", "status", "flags"):
        assert key in line, key
    assert line["status"] == 0 and line["flags"] == 0
    assert line["value"] > 0 and line["gpu_launches"] == 6
    r = line["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and 0 < r["frac"] == pytest.approx(r["achieved"] / r["peak"])
    assert line["e2e"]["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 8 * 2048 * 4096 * 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline_1core"]["cores"] == 1
    assert line["scaling"] == "weak" and line["roofline"]["traffic_source"]


def test_algorithmic_bytes_match_the_roofline_definition():
    """B_min = P n (2 in + 2 out + 16 state) + 2 (P - 1) G PB + 2 G PB: 21.0625
    bytes per element-rank at 4 bits and groups of 128 (PB = 68), 5.0625
    without state; the two kernels' own shares add up to it less the gather
    payload's read-back, which the owners' pass does not need."""
    sys.path.insert(0, ROOT)
    import bench
    P, n, g = 8, 1 << 29, 128
    G = n // g
    ab = bench.algorithmic_bytes(P, n, g, 4)
    assert ab["total"] == P * n * 20 + 2 * (P - 1) * G * 68 + 2 * G * 68 == 90_462_748_672
    assert ab["total"] / (P * n) == 21.0625
    assert bench.algorithmic_bytes(P, n, g, 4, feedback=False)["total"] / (P * n) == 5.0625
    assert ab["quantize"] == (P - 1) * G * 2372 and ab["reduce_gather"] == G * 4896
    assert ab["quantize"] + ab["reduce_gather"] + G * 68 == ab["total"]
    assert bench.algorithmic_bytes(P, n, g, 8)["total"] / (P * n) == 22.0625


@pytest.mark.gpu
def test_background_study_line():
    out = subprocess.run([sys.executable, "bench.py", "--tokens", "2048", "--steps", "3", "--warmup", "2",
                          "--background", "0,50,100"], cwd=ROOT, capture_output=True, text=True, timeout=900,
                         check=True).stdout
    bg = _last_json(out)["background"]
    assert bg["loads_pct"] == [0, 50, 100]
    for key in ("echo", "echo_no_feedback", "bf16", "background_alone"):
        assert len(bg[key]) == 3 and all(v > 0 for v in bg[key][1:]), key
    assert bg["echo_slowdown"][0] == 1.0 and bg["background_alone"][0] == 0.0
    assert bg["background_alone"][2] > bg["background_alone"][1] > 0


@pytest.mark.gpu
def test_shapes_line():
    out = subprocess.run([sys.executable, "bench.py", "--shapes", "--steps", "2", "--warmup", "1"], cwd=ROOT,
                         capture_output=True, text=True, timeout=900, check=True).stdout
    shapes = _last_json(out)["shapes"]
    assert [(s["P"], s["group"], s["bits"]) for s in shapes][:4] == [(2, 128, 4), (4, 128, 4), (8, 128, 4),
                                                                     (16, 128, 4)]
    for s in shapes:
        assert s["status"] == 0 and s["flags"] == 0
        assert s["quantize_ms"] > 0 and s["reduce_ms"] > 0
        assert s["call_ms"] == pytest.approx(s["quantize_ms"] + s["reduce_ms"])
        assert 0 < s["reduce_frac"] < 1.5 and 0 < s["quantize_frac"] < 1.5


def test_oracle_pool_fails_fast_when_a_worker_dies():
    """A worker process that is gone (killed, or crashed at start-up) ends the
    pass with an error within seconds instead of the pool's 600 s limit, and
    closing the pool does not wait on the survivors."""
    import time
    sys.path.insert(0, ROOT)
    import bench
    pool = bench.OraclePool(2, 64)
    try:
        pool.procs[0].terminate()
        pool.procs[0].join(timeout=30)
        t0 = time.monotonic()
        with pytest.raises(RuntimeError, match="exited"):
            pool.run()
        assert time.monotonic() - t0 < 60
    finally:
        t1 = time.monotonic()
        pool.close()
        assert time.monotonic() - t1 < 30
    assert not any(pr.is_alive() for pr in pool.procs)


def test_oracle_pool_pass():
    sys.path.insert(0, ROOT)
    import bench
    pool = bench.OraclePool(2, 64)
    try:
        gbs, dt, er = pool.run()
    finally:
        pool.close()
    assert gbs > 0 and dt > 0 and er == pool.w.P * 64 * pool.w.group
    assert not any(pr.is_alive() for pr in pool.procs)
