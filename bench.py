"""Benchmark: Echo 4-bit error-compensated all-reduce, simulated over P = 8
virtual ranks on one B200, on the 1 GB-per-rank message (131072 x 4096 bf16,
Student-t nu=3 values scaled to unit variance, groups of 128, INT4, feedback
on: alpha_long 0.05, alpha_short 0.5, w 0.5, eta 1).

One step = one full call (two kernels: the non-owners' quantize with fused
feedback and EMA update; the owners' reduce/requantize, which also decodes the
gathered result into all P outputs), inputs resident in HBM.
Metric: GB/s of bf16 input (all P ranks' inputs) per second.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

With N > 1 (launched by torchrun, one process per GPU) the one 1 GB message
is split across the GPUs by group columns (``--split columns``, the default):
rank k runs echo_allreduce_sim_range on columns [floor(kG/N), floor((k+1)G/N))
of the same message -- every column is independent, so there is no collective
on the data path -- and value = the message's input bytes / max-over-ranks
time (strong scaling). ``--split messages`` instead gives every GPU its own
independent 1 GB message (weak scaling, value = all ranks' input bytes /
max-over-ranks time).

``--impl reference`` times the oracle (plain C, single thread) on the host on a
bounded sample of group columns of the same workload, rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import queue
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Echo 4-bit all-reduce sim GB/s of bf16 input (P=8, 1 GB); % HBM roofline"
FALLBACK_HBM_GBS = 6650.0

# group columns of the workload timed on the host (one oracle call each):
# single thread, and on all cores (a chunk of columns per worker process)
CPU_BASELINE_COLS = 1 << 17
CPU_BASELINE_COLS_PER_CORE = 1 << 13
CPU_BASELINE_COLS_MAX = 1 << 18
REFERENCE_STEP_COLS_PER_CORE = 1 << 11
REFERENCE_STEP_COLS_MAX = 1 << 17


_TOKENS = None   # --tokens: a smaller message of the same shape family (profiling only)


def _workload():
    import dataclasses
    import workloads as W
    if _TOKENS is None:
        return W.HEADLINE
    return dataclasses.replace(W.HEADLINE, name=f"{W.HEADLINE.name}_tokens{_TOKENS}", tokens=_TOKENS)


def _peak_hbm():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes(P, n, group, bits, feedback=True):
    """Minimal bytes per call: every tensor crosses HBM once, each payload is
    written once and read once ("total", the roofline of the call). Per
    kernel: quantize; and the owners' reduce, which also writes the P outputs
    (it decodes the gathered bits it just produced, so its own bytes omit the
    re-read of the gather payload that "total" counts)."""
    G = -(-n // group)
    pb = group * bits // 8 + 4                       # payload bytes per group
    st = 16 if feedback else 0                       # two fp32 EMAs read + written
    xb = 2 * group                                   # bf16 input of one group
    q = (P - 1) * G * (xb + st * group + pb)          # non-owned rank-groups
    r = G * (xb + st * group + (P - 1) * pb + pb)      # owners: own x + EMAs, P-1 payloads in, gather out
    g = G * (pb + P * xb)                             # gather payload in, P outputs
    return {"quantize": q, "reduce_gather": r + g - G * pb, "total": q + r + g}


def _kernel_source_hash():
    """Hash of the device code: the kernels and their launch shape (threads,
    ring stages, shared memory) are all defined in these two files."""
    h = hashlib.sha256()
    for f in ("echo_kernels.cuh", "echo_pipeline.cuh"):
        with open(os.path.join(ROOT, "bit_error_compensated_group_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _measured_traffic():
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, or None when the kernel changed since it was captured."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except Exception:
        return None
    if t.get("source_hash") != _kernel_source_hash():
        return None
    return t.get("bytes_per_launch")


class ClockSampler:
    """SM clock and throttle reasons sampled during the timed region: NVML read
    every 20 ms from a thread (falls back to `nvidia-smi -lms 200`). Reads
    only; no setting of the GPU is touched."""
    PERIOD_S = 0.02
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        import threading
        import torch
        self.rows = []          # (sm_mhz, set of reason names)
        self.max_mhz = None
        self.proc = None
        self.thread = None
        self.kind = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            return
        self.uuid = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        try:
            import pynvml as N
            N.nvmlInit()
            self.N = N
            self.h = N.nvmlDeviceGetHandleByUUID(self.uuid)
            self.max_mhz = float(N.nvmlDeviceGetMaxClockInfo(self.h, N.NVML_CLOCK_SM))
            self.bits = {"hw_slowdown": N.nvmlClocksEventReasonHwSlowdown,
                         "hw_thermal_slowdown": N.nvmlClocksEventReasonHwThermalSlowdown,
                         "sw_thermal_slowdown": N.nvmlClocksEventReasonSwThermalSlowdown,
                         "sw_power_cap": N.nvmlClocksEventReasonSwPowerCap}
            self.done = threading.Event()
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.kind = "nvml"
            self.thread.start()
        except Exception:
            self.thread = None
            self._start_smi()

    def _poll(self):
        N = self.N
        while not self.done.is_set():
            try:
                mhz = float(N.nvmlDeviceGetClockInfo(self.h, N.NVML_CLOCK_SM))
                r = N.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.rows.append((mhz, {k for k, b in self.bits.items() if r & b}))
            except Exception:
                pass
            self.done.wait(self.PERIOD_S)

    def _start_smi(self):
        try:
            self.path = f"/tmp/echo_clocks_{os.getpid()}.csv"
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.SMI_FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
            self.kind = "nvidia-smi"
        except Exception:
            self.proc = None

    def _stop_smi(self):
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) != 9 or not parts[1].replace(".", "").isdigit():
                    continue
                if parts[2].replace(".", "").isdigit():
                    self.max_mhz = float(parts[2])
                self.rows.append((float(parts[1]),
                                  {self.REASONS[i] for i in range(4) if parts[5 + i].lower() == "active"}))
        os.unlink(self.path)

    def stop(self):
        if self.thread is not None:
            self.done.set()
            self.thread.join(timeout=5)
            try:
                self.N.nvmlShutdown()
            except Exception:
                pass
        elif self.proc is not None:
            self._stop_smi()
        if not self.rows:
            return None
        return {"sm_mhz": statistics.median(r[0] for r in self.rows), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(set().union(*(r[1] for r in self.rows))), "samples": len(self.rows),
                "sampler": f"{self.kind}, every {int(self.PERIOD_S * 1000) if self.kind == 'nvml' else 200} ms"}


def max_over_ranks(value: float, world: int, device) -> float:
    """The largest `value` over all ranks (every rank gets it); the job's time
    is its slowest rank's."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_gbs(world: int, bytes_per_rank: int, max_ms: float) -> float:
    """Whole-job GB/s: every rank moved its own message in the slowest rank's time."""
    return world * bytes_per_rank / (max_ms * 1e-3) / 1e9


def cpu_sample_rate(cols, seed=123):
    """Time the oracle (single thread, as it stands) on `cols` group columns
    of the workload; returns (GB/s of bf16 input, seconds, element-ranks)."""
    import numpy as np
    import torch
    import oracle as O
    import workloads as W
    w = _workload()
    P, group = w.P, w.group
    G = -(-w.n // group)
    cols = min(cols, w.n // group)                # full groups only (a smaller message when profiling)
    j0 = (G // 2) - cols // 2                     # straddles an owner boundary at P = 8
    m = cols * group
    x = np.empty((P, m), np.uint16)
    for r in range(P):
        x[r] = W.bf16_bits(W.student_t3_unit_f32(m, W.seed_of(w.cid, 7, r)).to(torch.bfloat16))
    el = np.zeros((P, m), np.float32)
    es = np.zeros((P, m), np.float32)
    t0 = time.perf_counter()
    O.echo_allreduce(x, n_total=w.n, group=group, bits=w.bits, e_long=el, e_short=es, eta=w.eta,
                     alpha_long=w.alpha_long, alpha_short=w.alpha_short, w=w.w, j0=j0, jc=cols)
    dt = time.perf_counter() - t0
    return P * m * 2 / dt / 1e9, dt, P * m


# ------------------------------------------------------------ the oracle on all host cores
#
# The oracle stays single-threaded and unchanged; the sample's group columns
# are cut into one contiguous chunk per worker process (spawned, so no CUDA
# state is inherited), every column being independent. Inputs sit in shared
# memory; each worker copies its chunk, waits at a barrier with the others,
# then runs the oracle on its columns. Elapsed = latest end - earliest start.

def _oracle_worker(wid, shm_name, shape, barrier, tasks, results):
    import numpy as np
    from multiprocessing import shared_memory
    import oracle as O
    shm = shared_memory.SharedMemory(name=shm_name)
    try:
        x_all = np.ndarray(shape, dtype=np.uint16, buffer=shm.buf)
        while True:
            task = tasks.get()
            if task is None:
                break
            lo, hi, j0, n_total, group, bits, fb = task
            x = np.ascontiguousarray(x_all[:, lo * group:hi * group])
            el = np.zeros(x.shape, np.float32)
            es = np.zeros(x.shape, np.float32)
            barrier.wait(timeout=120)
            t0 = time.perf_counter()
            if hi > lo:
                O.echo_allreduce(x, n_total=n_total, group=group, bits=bits, e_long=el, e_short=es, eta=fb[0],
                                 alpha_long=fb[1], alpha_short=fb[2], w=fb[3], j0=j0 + lo, jc=hi - lo)
            results.put((wid, t0, time.perf_counter()))
    finally:
        del x_all
        shm.close()


class OraclePool:
    """`workers` spawned processes, each running the oracle on its own chunk
    of group columns: by default a sample of `cols` columns of the benchmark
    workload; with `x` (a [P][cols * group] bf16-bit array of workload `w`,
    columns from `j0`), those columns."""

    def __init__(self, workers, cols, w=None, x=None, j0=None):
        import multiprocessing as mp
        import numpy as np
        import torch
        from multiprocessing import shared_memory
        import workloads as W
        w = _workload() if w is None else w
        self.w = w
        self.workers = workers
        G = -(-w.n // w.group)
        if x is None:
            self.cols = min(cols, w.n // w.group)          # full groups only
            self.j0 = G // 2 - self.cols // 2                # straddles an owner boundary at P = 8
        else:
            self.cols, self.j0 = cols, j0
        m = self.cols * w.group
        self.shm = shared_memory.SharedMemory(create=True, size=w.P * m * 2)
        xs = np.ndarray((w.P, m), dtype=np.uint16, buffer=self.shm.buf)
        for r in range(w.P):
            if x is None:
                xs[r] = W.bf16_bits(W.student_t3_unit_f32(m, W.seed_of(w.cid, 7, r)).to(torch.bfloat16))
            else:
                xs[r] = x[r]
        del xs
        ctx = mp.get_context("spawn")
        self.barrier = ctx.Barrier(workers)
        self.results = ctx.Queue()
        self.tasks = [ctx.Queue() for _ in range(workers)]
        self.procs = [ctx.Process(target=_oracle_worker, daemon=True,
                                  args=(k, self.shm.name, (w.P, m), self.barrier, self.tasks[k], self.results))
                      for k in range(workers)]
        self.broken = False
        for pr in self.procs:
            pr.start()

    def run(self, bits=None):
        """One pass over the columns on all workers: (GB/s of bf16 input,
        seconds, element-ranks)."""
        w = self.w
        fb = (w.eta, w.alpha_long, w.alpha_short, w.w)
        for k in range(self.workers):
            lo, hi = k * self.cols // self.workers, (k + 1) * self.cols // self.workers
            self.tasks[k].put((lo, hi, self.j0, w.n, w.group, w.bits if bits is None else bits, fb))
        got = []
        deadline = time.monotonic() + 600
        while len(got) < self.workers:
            # a worker that died (e.g. at start-up) ends the run at once
            # rather than after the whole time limit
            try:
                got.append(self.results.get(timeout=1.0))
            except queue.Empty:
                dead = [pr.exitcode for pr in self.procs if pr.exitcode is not None]
                if dead:
                    self.broken = True
                    raise RuntimeError(f"oracle worker process exited with {dead}")
                if time.monotonic() > deadline:
                    self.broken = True
                    raise TimeoutError("oracle workers gave no result within 600 s")
        dt = max(g[2] for g in got) - min(g[1] for g in got)
        er = w.P * self.cols * w.group
        return er * 2 / dt / 1e9, dt, er

    def close(self):
        # after a failed pass the survivors may be waiting at the barrier:
        # end them at once; otherwise let every worker leave its loop
        if not self.broken:
            for q in self.tasks:
                q.put(None)
            for pr in self.procs:
                pr.join(timeout=30)
        for pr in self.procs:
            if pr.is_alive():
                pr.terminate()
                pr.join(timeout=10)
        self.shm.close()
        self.shm.unlink()


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def run_reference(args):
    """The oracle as it stands, on all the host's cores: each step one pass
    of the worker processes over a bounded sample of group columns."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = _workload()
    cores = host_cores()
    cols = min(REFERENCE_STEP_COLS_PER_CORE * cores, REFERENCE_STEP_COLS_MAX)
    pool = OraclePool(cores, cols)
    try:
        for _ in range(args.warmup):
            pool.run()
        times = []
        for _ in range(args.steps):
            _, dt, er = pool.run()
            times.append(dt)
    finally:
        pool.close()
    tot = sum(times)
    value = args.steps * er * 2 / tot / 1e9
    sample = (f"{pool.cols} of {-(-w.n // w.group)} group columns x P={w.P} per step ({er} element-ranks), "
              f"{cores} worker processes of the single-threaded oracle, one column chunk each")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": _config(w),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


_FEEDBACK = True   # --feedback off: the main step runs without EMA state (profiling that variant)


def _config(w):
    return {"workload": w.name, "P": w.P, "n": w.n, "tokens": w.tokens, "hidden": w.hidden, "group": w.group,
            "bits": w.bits, "feedback": _FEEDBACK, "eta": w.eta, "alpha_long": w.alpha_long,
            "alpha_short": w.alpha_short, "w": w.w, "values": "Student-t nu=3 / sqrt(3)",
            "l2": "no flush: each step touches %.0f GB, far larger than the 126 MB L2"
                  % (algorithmic_bytes(w.P, w.n, w.group, w.bits, _FEEDBACK)["total"] / 1e9)}


def run_gpu(args):
    import torch
    import torch.distributed as dist
    import workloads as W
    import bit_error_compensated_group_b200 as E

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    w = _workload()
    P, n, group, bits = w.P, w.n, w.group, w.bits
    G = -(-n // group)
    split_cols = world > 1 and args.split == "columns"
    c0, c1 = E.column_window(rank, world, G) if split_cols else (0, G)
    ar = E.EchoAllReduce(n, P, group, bits, feedback=_FEEDBACK, device=dev)
    inputs = []
    for r in range(P):
        # columns: every GPU holds the same message (it touches only its
        # window); messages: each GPU its own message
        inputs.append(W.rank_input(w, r, site=0 if split_cols else rank, device=dev))
    outputs = [torch.empty_like(t) for t in inputs]
    stream = torch.cuda.current_stream(dev)
    h = ar.handle
    fb = (w.eta, w.alpha_long, w.alpha_short, w.w)

    # one step = one echo_allreduce_sim call (with a column split: the
    # echo_allreduce_sim_range call on this GPU's window): the non-owners'
    # quantize pass, then the owners' pass (a programmatic dependent of the
    # first, which also decodes into all P outputs); events only at the step
    # boundaries
    def call():
        if split_cols:
            E.echo_allreduce_sim_range(inputs, outputs, h, n, P, bits, group, *fb, c0, c1, stream=stream)
        else:
            E.echo_allreduce_sim(inputs, outputs, h, n, P, bits, group, *fb, stream=stream)

    # the same two kernels through the phase entry points with an event
    # between them: the per-kernel split for the roofline, in a pass of its own
    def step(evs=None):
        if evs is not None:
            evs[0].record(stream)
        E.echo_phase_quantize(inputs, h, bits, *fb, stream=stream)
        if evs is not None:
            evs[1].record(stream)
        E.echo_phase_reduce(inputs, outputs, h, bits, *fb, stream=stream)
        if evs is not None:
            evs[2].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        call()
    barrier()

    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier()
    t0.record(stream)
    for _ in range(args.steps):
        call()
    t1.record(stream)
    barrier()
    clock_info = clocks.stop()
    rc, flags = ar.status()
    total_ms = t0.elapsed_time(t1)
    max_ms = max_over_ranks(total_ms, world, dev)

    # the per-kernel split (phase entry points over the whole message): with
    # a column split every GPU would time the whole message, so it is left out
    phase_steps = max(3, min(args.steps, 10))
    per_phase = None
    if not split_cols:
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(phase_steps)]
        for i in range(phase_steps):
            step(evs[i])
        barrier()
        per_phase = {"quantize": 0.0, "reduce_gather": 0.0}
        for e in evs:
            per_phase["quantize"] += e[0].elapsed_time(e[1])
            per_phase["reduce_gather"] += e[1].elapsed_time(e[2])

    # the same message without feedback state (x' = x, no EMA traffic): its
    # time and the difference, the cost of compensation (the pages quote
    # 0.90 ms per 1 GB message on 8 A100s, fused into the entry pass)
    variant = None
    if not args.no_variants and _FEEDBACK and not split_cols:
        nf = E.EchoAllReduce(n, P, group, bits, feedback=False, device=dev)
        nf_steps = max(3, min(args.steps, 10))

        def nf_step(ev=None):
            if ev is not None:
                ev[0].record(stream)
            E.echo_phase_quantize(inputs, nf.handle, bits, *fb, stream=stream)
            if ev is not None:
                ev[1].record(stream)
            E.echo_phase_reduce(inputs, outputs, nf.handle, bits, *fb, stream=stream)
            if ev is not None:
                ev[2].record(stream)

        for _ in range(args.warmup):
            nf_step()
        barrier()
        nf_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(nf_steps)]
        for i in range(nf_steps):
            nf_step(nf_evs[i])
        barrier()
        nf_ms = max_over_ranks(nf_evs[0][0].elapsed_time(nf_evs[-1][2]), world, dev) / nf_steps
        nf_phases = {"quantize": sum(e[0].elapsed_time(e[1]) for e in nf_evs) / nf_steps,
                     "reduce_gather": sum(e[1].elapsed_time(e[2]) for e in nf_evs) / nf_steps}
        nf.close()
        del nf
        variant = {"ms_per_step": nf_ms, "steps": nf_steps, "phases_ms": nf_phases,
                   "value": weak_scaling_gbs(world, P * n * 2, nf_ms),
                   "roofline_frac": algorithmic_bytes(P, n, group, bits, feedback=False)["total"] / (nf_ms * 1e-3)
                   / 1e9 / _peak_hbm()[0]}

    # the other quantizer forms (the ablations' variants) on the same call,
    # feedback on: the nearest and integer-zero forms clamp each code
    forms = None
    if not args.no_variants and _FEEDBACK and not split_cols:
        forms = {}
        q_steps = max(3, min(args.steps, 10))
        for name, q in (("nearest", E.ECHO_QUANT_NEAREST), ("int_zero", E.ECHO_QUANT_INT_ZERO)):
            E.echo_set_quantizer(h, q)
            for _ in range(args.warmup):
                step()
            barrier()
            q_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(q_steps)]
            for i in range(q_steps):
                step(q_evs[i])
            barrier()
            q_ms = max_over_ranks(q_evs[0][0].elapsed_time(q_evs[-1][2]), world, dev) / q_steps
            forms[name] = {"ms_per_step": q_ms, "steps": q_steps,
                           "roofline_frac": algorithmic_bytes(P, n, group, bits)["total"] / (q_ms * 1e-3)
                           / 1e9 / _peak_hbm()[0]}
        E.echo_set_quantizer(h, E.ECHO_QUANT_DIRECTED)

    # the early-site 8-bit mode on the same message, feedback on (one code
    # per byte: 22.06 algorithmic bytes per element-rank instead of 21.06)
    int8 = None
    if not args.no_variants and _FEEDBACK and not split_cols:
        a8 = E.EchoAllReduce(n, P, group, 8, feedback=True, device=dev)
        i8_steps = max(3, min(args.steps, 10))

        def i8_step(ev=None):
            if ev is not None:
                ev[0].record(stream)
            E.echo_phase_quantize(inputs, a8.handle, 8, *fb, stream=stream)
            if ev is not None:
                ev[1].record(stream)
            E.echo_phase_reduce(inputs, outputs, a8.handle, 8, *fb, stream=stream)
            if ev is not None:
                ev[2].record(stream)

        for _ in range(args.warmup):
            i8_step()
        barrier()
        i8_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(i8_steps)]
        for i in range(i8_steps):
            i8_step(i8_evs[i])
        barrier()
        i8_ms = max_over_ranks(i8_evs[0][0].elapsed_time(i8_evs[-1][2]), world, dev) / i8_steps
        i8_q = sum(e[0].elapsed_time(e[1]) for e in i8_evs) / i8_steps
        i8_r = sum(e[1].elapsed_time(e[2]) for e in i8_evs) / i8_steps
        ab8 = algorithmic_bytes(P, n, group, 8)
        a8_rc, a8_flags = a8.status()
        a8.close()
        del a8
        torch.cuda.empty_cache()
        int8 = {"ms_per_step": i8_ms, "steps": i8_steps, "phases_ms": {"quantize": i8_q, "reduce_gather": i8_r},
                "value": weak_scaling_gbs(world, P * n * 2, i8_ms),
                "roofline_frac": ab8["total"] / (i8_ms * 1e-3) / 1e9 / _peak_hbm()[0],
                "quantize_frac": ab8["quantize"] / (i8_q * 1e-3) / 1e9 / _peak_hbm()[0],
                "status": a8_rc, "flags": a8_flags}

    # end to end through the public host-buffer call: every step, pinned
    # inputs copied in and the reduced result copied out, chunk by chunk on
    # two copy streams overlapping the kernels (echo_allreduce_sim_host)
    e2e = None
    host_in = host_out = None
    if not args.no_e2e:
        # every rank pins P + 1 message buffers (its window's, with a column
        # split); the leg runs only if all could (a collective decision, so
        # that every rank takes the same steps)
        why = None
        hn = min(c1 * group, n) - c0 * group if split_cols else n
        try:
            host_in = [torch.empty(hn, dtype=torch.bfloat16, pin_memory=True) for _ in range(P)]
            host_out = torch.empty(hn, dtype=torch.bfloat16, pin_memory=True)
        except (RuntimeError, MemoryError) as exc:
            host_in = host_out = None
            why = f"pinned host buffers: {exc}".splitlines()[0][:200]
        if max_over_ranks(0.0 if why is None else 1.0, world, dev) > 0.0:
            e2e = {"unavailable": why or "another rank could not pin its host buffers"}
            host_in = host_out = None
    if host_in is not None and split_cols:
        # a column split: this GPU's window of the inputs in, its window of
        # the result out, around the window's call (serialised on one stream)
        e0, e1 = c0 * group, min(c1 * group, n)   # the pinned buffers hold just this window
        e2e_steps = max(1, min(args.steps, 4))
        for r in range(P):
            host_in[r].copy_(inputs[r][e0:e1])

        def e2e_step():
            for r in range(P):
                inputs[r][e0:e1].copy_(host_in[r], non_blocking=True)
            call()
            host_out.copy_(outputs[0][e0:e1], non_blocking=True)

        e2e_step()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        b.record(stream)
        barrier()
        e2e_ms = max_over_ranks(a.elapsed_time(b), world, dev) / e2e_steps
        e2e = {"value": P * n * 2 / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": P * n * 2, "d2h_bytes_per_step": n * 2,
               "ms_per_step": e2e_ms, "steps": e2e_steps,
               "call": "echo_allreduce_sim_range on each GPU's window, host copies of the window around it"}
        host_in = host_out = None
    if host_in is not None:
        e2e_steps = max(1, min(args.steps, 4))
        for r in range(P):
            host_in[r].copy_(inputs[r])
        cin, cout = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def e2e_step():
            E.echo_allreduce_sim_host(host_in, host_out, inputs, outputs, h, n, P, bits, group, *fb,
                                      args.e2e_chunk, stream=stream, copy_in=cin, copy_out=cout)

        e2e_step()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        b.record(stream)
        barrier()
        e2e_ms = max_over_ranks(a.elapsed_time(b), world, dev) / e2e_steps
        chunk = args.e2e_chunk if args.e2e_chunk > 0 else -(-G // 16)
        e2e = {"value": weak_scaling_gbs(world, P * n * 2, e2e_ms), "unit": "GB/s",
               "h2d_bytes_per_step": P * n * 2, "d2h_bytes_per_step": n * 2,
               "ms_per_step": e2e_ms, "steps": e2e_steps, "call": "echo_allreduce_sim_host",
               "chunks": -(-G // chunk)}
        del host_in, host_out

    if rank == 0:
        ms = max_ms / args.steps
        peak, peak_kind = _peak_hbm()
        ab = algorithmic_bytes(P, n, group, bits, feedback=_FEEDBACK)
        traffic = _measured_traffic() if _FEEDBACK else None
        cfg = _config(w)
        if split_cols:
            # strong scaling: the one message's bytes in the slowest GPU's time;
            # the roofline is the whole call's, per GPU (each moves 1/N of it)
            value = P * n * 2 / (ms * 1e-3) / 1e9
            per_gpu = ab["total"] / world / (ms * 1e-3) / 1e9
            cfg.update(split="columns", windows=[list(E.column_window(k, world, G)) for k in range(world)])
            roof = {"bound": "hbm", "kernel": "call (both kernels, one GPU's window)", "achieved": per_gpu,
                    "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": per_gpu / peak, "traffic": None,
                    "algorithmic_bytes": ab["total"] // world}
            phases = None
        else:
            value = weak_scaling_gbs(world, P * n * 2, ms)
            q_ms = per_phase["quantize"] / phase_steps
            achieved = ab["quantize"] / (q_ms * 1e-3) / 1e9
            if world > 1:
                cfg.update(split="messages")
            roof = {"bound": "hbm", "kernel": "k_quantize", "achieved": achieved, "peak": peak,
                    "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                    "traffic_source": "ncu capture of a 4096-token case, scaled to the full launch by the "
                                      "rank-groups processed (x32)",
                    "algorithmic_bytes": ab["quantize"]}
            phases = {k: v / phase_steps for k, v in per_phase.items()}
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "strong" if split_cols else "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": cfg,
            "roofline": roof,
            "roofline_call": {"bytes": ab["total"], "achieved": ab["total"] / (ms * 1e-3) / 1e9,
                              "frac": ab["total"] / (ms * 1e-3) / 1e9 / peak},
            "phases_ms": phases,
            "phases_steps": phase_steps if phases is not None else 0,
            "elements_per_s": (1 if split_cols else world) * P * n / (ms * 1e-3),
            "gpu_launches": 2 * args.steps if P >= 2 else args.steps,   # the timed calls' two kernels
            "clocks": clock_info, "status": rc, "flags": flags,
            "e2e": e2e,
        }
        if split_cols:
            line["roofline_call"] = {"bytes": ab["total"], "achieved": ab["total"] / (ms * 1e-3) / 1e9,
                                     "frac_of_n_gpus": ab["total"] / (ms * 1e-3) / 1e9 / (peak * world)}
        if variant is not None:
            line["no_feedback"] = variant
            line["compensation_ms"] = ms - variant["ms_per_step"]
        if forms is not None:
            line["quantizer_forms"] = forms
        if int8 is not None:
            line["int8"] = int8
        if world == 1 and not args.no_cpu_baseline:
            cores = host_cores()
            pool = OraclePool(cores, min(CPU_BASELINE_COLS_PER_CORE * cores, CPU_BASELINE_COLS_MAX))
            try:
                gbs, dt, er = pool.run()
            finally:
                pool.close()
            line["cpu_baseline"] = {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
                                    "sample": f"{er // (P * group)} group columns x P={P} ({er} element-ranks, "
                                              f"{dt:.2f} s on {cores} worker processes of the single-threaded "
                                              f"oracle, one column chunk each)"}
            gbs1, dt1, er1 = cpu_sample_rate(CPU_BASELINE_COLS)
            line["cpu_baseline_1core"] = {"value": gbs1, "unit": "GB/s", "cores": 1, "kind": "oracle",
                                          "sample": f"{er1 // (P * group)} group columns x P={P} "
                                                    f"({er1} element-ranks, {dt1:.1f} s, single thread)"}
        print(json.dumps(line), flush=True)
    ar.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_ablation(args):
    """Accuracy ablations on the synthetic chains, through the public API on
    one GPU (the oracle's agreement with these runs is the GPU test suite's
    job). Each entry: RMS and max over elements of the accumulated error
    S_T = sum_t (y_t - sum_r x_t,r) after the last site, in units of q and
    q_max, the RMS and max of the per-site error of the default form at the
    same bits without feedback (the quantizer's own error scale)."""
    import torch
    import workloads as W
    import bit_error_compensated_group_b200 as E
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)

    noise = {}   # per chain: every site's noise, drawn once and kept on the device

    def site_noise(w, t):
        if w.name not in noise:
            noise[w.name] = [W.chain_noise(w, k + 1).to(dev) for k in range(w.sites)]
        return noise[w.name][t]

    def chain(w, feedback=True, quantizer=E.ECHO_QUANT_DIRECTED, group=None, int8_sites=None, wt=None):
        group = group or w.group
        int8 = w.int8_sites if int8_sites is None else int8_sites
        ar = E.EchoAllReduce(w.n, w.P, group, 8 if int8 else 4, feedback, device=dev, quantizer=quantizer)
        x = W.inputs(w, 0, "cpu")
        inputs = [x[r].to(dev) for r in range(w.P)]
        outputs = [torch.empty_like(t) for t in inputs]
        acc = torch.zeros(w.n, dtype=torch.float64, device=dev)
        site_rms, site_max = [], []
        try:
            for t in range(w.sites):
                bits = 8 if t < int8 else w.bits
                ar(inputs, outputs, bits, w.eta, w.alpha_long, w.alpha_short, w.w if wt is None else wt)
                err = outputs[0].double() - torch.stack([i.double() for i in inputs]).sum(0)
                acc += err
                site_rms.append(float(err.pow(2).mean().sqrt()))
                site_max.append(float(err.abs().max()))
                # the chain rule of workloads.chain_next_input, evaluated on the device
                xn = (outputs[0].float() * w.decay / w.P + site_noise(w, t)).to(torch.bfloat16)
                for r in range(w.P):
                    inputs[r].copy_(xn[r])
            rc, _ = ar.status()
            assert rc == E.ECHO_OK, rc
        finally:
            ar.close()
        return float(acc.pow(2).mean().sqrt()), float(acc.abs().max()), site_rms, site_max

    out = {}
    for w, key in ((W.CHAIN56, "chain56_p8_int4"), (W.CHAIN48_MIXED, "chain48_p4")):
        _, _, q_rms, q_max = chain(w, feedback=False, int8_sites=0)
        q, qm = sum(q_rms) / len(q_rms), sum(q_max) / len(q_max)
        runs = {}
        if w is W.CHAIN56:
            for name, qf in (("directed", E.ECHO_QUANT_DIRECTED), ("nearest", E.ECHO_QUANT_NEAREST),
                             ("int_zero", E.ECHO_QUANT_INT_ZERO)):
                runs[f"form={name}"] = chain(w, quantizer=qf)
                runs[f"form={name},no_feedback"] = chain(w, feedback=False, quantizer=qf)
            for g in (64, 256):
                runs[f"group={g}"] = chain(w, group=g)
            runs["ema=long_only(w=0)"] = chain(w, wt=0.0)
            runs["ema=short_only(w=1)"] = chain(w, wt=1.0)
        else:
            for k8, name in ((0, "none"), (12, "first_quarter(12)"), (24, "first_half(24)"), (48, "all")):
                runs[f"int8_sites={name}"] = chain(w, int8_sites=k8)
                runs[f"int8_sites={name},no_feedback"] = chain(w, feedback=False, int8_sites=k8)
        out[key] = {"q": q, "q_max": qm,
                    "runs": {k: {"rms_S_T/q": v[0] / q, "max_S_T/q_max": v[1] / qm} for k, v in runs.items()}}
    print(json.dumps({"ablation": out, "data": "synthetic chains (workloads.CHAIN56, workloads.CHAIN48_MIXED)"}),
          flush=True)


def run_workloads(args):
    """Every workload's call timed on the GPU (inputs resident, state carried
    from call to call) and the oracle's call timed on the host, single thread.
    Chains are timed per site at each bit width they use; the 1 GB message's
    oracle figure is the main line's sampled `cpu_baseline`."""
    import ctypes
    import numpy as np
    import torch
    import oracle as O
    import workloads as W
    import bit_error_compensated_group_b200 as E
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peak, peak_kind = _peak_hbm()
    out = {}
    for w in W.ALL:
        P, n, group = w.P, w.n, w.group
        widths = sorted({w.bits_at(t) for t in range(w.sites)})
        ar = E.EchoAllReduce(n, P, group, max(widths), feedback=True, device=dev)
        inputs = [W.rank_input(w, r, 0, dev) for r in range(P)]
        outputs = [torch.empty_like(t) for t in inputs]
        fb = (w.eta, w.alpha_long, w.alpha_short, w.w)
        entry = {"P": P, "n": n, "sites": w.sites, "int8_sites": w.int8_sites, "per_call": {}}
        # small messages take tens of microseconds: many calls, and the C
        # call made with its pointer arrays built once, so that the host's
        # argument marshalling does not pace the stream
        steps = max(3, args.steps) if P * n > (1 << 26) else max(300, args.steps)
        L = E.lib()
        pin = (ctypes.c_void_p * P)(*[t.data_ptr() for t in inputs])
        pout = (ctypes.c_void_p * P)(*[t.data_ptr() for t in outputs])
        sh = stream.cuda_stream
        for bits in widths:
            def call():
                rc = L.echo_allreduce_sim(pin, pout, ar.handle, n, P, bits, group, *fb, sh)
                assert rc == E.ECHO_OK, rc
            for _ in range(max(3, args.warmup)):
                call()
            torch.cuda.synchronize(dev)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(steps):
                call()
            b.record(stream)
            torch.cuda.synchronize(dev)
            ms = a.elapsed_time(b) / steps
            ab = algorithmic_bytes(P, n, group, bits)["total"]
            rc, flags = ar.status()
            entry["per_call"][f"int{bits}"] = {
                "gpu_ms": ms, "gbs_bf16_input": P * n * 2 / (ms * 1e-3) / 1e9,
                "roofline_frac": ab / (ms * 1e-3) / 1e9 / peak, "algorithmic_bytes": ab, "status": rc,
                "l2_resident": ab < 126e6, "steps": steps}
        ar.close()
        del ar, inputs, outputs
        torch.cuda.empty_cache()
        if w.sites > 1:
            entry["gpu_ms_per_chain"] = sum(entry["per_call"][f"int{w.bits_at(t)}"]["gpu_ms"] for t in range(w.sites))
        if w is not W.HEADLINE and not args.no_cpu_baseline:
            G = -(-n // group)
            x = np.zeros((P, G * group), np.uint16)
            x[:, :n] = W.bf16_bits(W.inputs(w, 0, "cpu"))
            cores = host_cores()
            pool = OraclePool(min(cores, G), G, w=w, x=x, j0=0) if G > 1 else None
            for bits in widths:
                el = np.zeros((P, G * group), np.float32)
                es = np.zeros((P, G * group), np.float32)
                t0 = time.perf_counter()
                O.echo_allreduce(x, n_total=n, group=group, bits=bits, e_long=el, e_short=es, eta=w.eta,
                                 alpha_long=w.alpha_long, alpha_short=w.alpha_short, w=w.w)
                dt = time.perf_counter() - t0
                entry["per_call"][f"int{bits}"]["oracle_ms"] = dt * 1e3
                entry["per_call"][f"int{bits}"]["oracle_cores"] = 1
                if pool is not None:
                    _, dtn, _ = pool.run(bits)
                    entry["per_call"][f"int{bits}"]["oracle_ms_all_cores"] = dtn * 1e3
                    entry["per_call"][f"int{bits}"]["oracle_all_cores"] = pool.workers
            if pool is not None:
                pool.close()
        out[w.name] = entry
    print(json.dumps({"workloads": out, "peak_gbs": peak, "peak_kind": peak_kind, "data": "synthetic"}), flush=True)


def run_background(args):
    """The background-traffic study on one GPU (the Echo abstract and the
    explainer's results section: the gain over a 16-bit all-reduce grows
    with competing traffic). For each load level L (% duty cycle of an HBM
    copy running on its own stream: copy for L % of every 100 us period,
    sleep for the rest), the Echo call (with and without feedback) and the
    16-bit baseline all-reduce of the same message are timed on the main
    stream while the copy runs. The copy's own bandwidth is measured alone
    and during the timed calls."""
    import torch
    import workloads as W
    import bit_error_compensated_group_b200 as E
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = _workload()
    P, n, group, bits = w.P, w.n, w.group, w.bits
    fb = (w.eta, w.alpha_long, w.alpha_short, w.w)
    peak, peak_kind = _peak_hbm()
    inputs = [W.rank_input(w, r, 0, dev) for r in range(P)]
    outputs = [torch.empty_like(t) for t in inputs]
    ar = E.EchoAllReduce(n, P, group, bits, feedback=True, device=dev)
    nf = E.EchoAllReduce(n, P, group, bits, feedback=False, device=dev)
    bg_bytes = 2 << 30
    src = torch.randint(0, 255, (bg_bytes,), dtype=torch.uint8, device=dev)
    dst = torch.empty_like(src)
    moved = torch.zeros(1, dtype=torch.int64, device=dev)
    main, side = torch.cuda.current_stream(dev), torch.cuda.Stream(dev)
    steps = max(3, args.steps)
    calls = {
        "echo": lambda: E.echo_allreduce_sim(inputs, outputs, ar.handle, n, P, bits, group, *fb, stream=main),
        "echo_no_feedback": lambda: E.echo_allreduce_sim(inputs, outputs, nf.handle, n, P, bits, group, *fb,
                                                          stream=main),
        "bf16": lambda: E.echo_bf16_allreduce_sim(inputs, outputs, n, P, stream=main),
    }
    for f in calls.values():                      # warm-up without load
        for _ in range(args.warmup):
            f()
    torch.cuda.synchronize(dev)
    # the foreground time at no load, to size the copy's duration
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(main)
    for f in calls.values():
        for _ in range(steps + 1):
            f()
    b.record(main)
    torch.cuda.synchronize(dev)
    window_us = int(a.elapsed_time(b) * 1e3)
    period_us = 100
    levels = [int(v) for v in str(args.background).split(",") if v.strip()]
    out = {"loads_pct": levels, "period_us": period_us}
    for key in list(calls) + ["background_alone", "background_during_estimate"]:
        out[key] = []
    for lv in levels:
        # the copy alone: its bandwidth at this duty cycle
        moved.zero_()
        alone_us = 20000
        E.echo_background_traffic(src, dst, 10 * lv, period_us, alone_us, moved, stream=side)
        torch.cuda.synchronize(dev)
        out["background_alone"].append(int(moved.item()) / (alone_us * 1e-6) / 1e9)
        # the calls while the copy runs (its duration covers them even if they
        # slow down 3x); the copy's bandwidth during the calls is estimated
        # from its total bytes less what it moved alone after them
        moved.zero_()
        dur_us = 3 * window_us + 20000
        E.echo_background_traffic(src, dst, 10 * lv, period_us, dur_us, moved, stream=side)
        w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        w0.record(main)
        for key, f in calls.items():
            f()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(main)
            for _ in range(steps):
                f()
            e1.record(main)
            e1.synchronize()
            out[key].append(e0.elapsed_time(e1) / steps)
        w1.record(main)
        torch.cuda.synchronize(dev)
        busy_s = w0.elapsed_time(w1) * 1e-3
        alone_gbs = out["background_alone"][-1]
        during = (int(moved.item()) / 1e9 - alone_gbs * max(0.0, dur_us * 1e-6 - busy_s)) / busy_s if lv else 0.0
        out["background_during_estimate"].append(max(0.0, during))
    for key in calls:
        base = out[key][levels.index(0)] if 0 in levels else out[key][0]
        out[key + "_slowdown"] = [t / base for t in out[key]]
    out["bf16_over_echo"] = [bt / et for bt, et in zip(out["bf16"], out["echo"])]
    out["bf16_over_echo_no_feedback"] = [bt / et for bt, et in zip(out["bf16"], out["echo_no_feedback"])]
    ab = algorithmic_bytes(P, n, group, bits)
    out["algorithmic_bytes"] = {"echo": ab["total"],
                                "echo_no_feedback": algorithmic_bytes(P, n, group, bits, feedback=False)["total"],
                                "bf16": 2 * P * n * 2}
    ar.close()
    nf.close()
    rc = 0
    print(json.dumps({"background": out, "unit": "ms per call", "steps": steps, "warmup": args.warmup,
                      "config": _config(w), "peak_gbs": peak, "peak_kind": peak_kind, "data": "synthetic",
                      "status": rc}), flush=True)


def _chunk_counts(args):
    return [int(c) for c in str(args.chunks).split(",") if c.strip()]


def run_ranks(args):
    """One rank's kernels of a real multi-GPU call (rank 0 of P = 8 on the
    1 GB message), on one GPU: the P ranks' handles are set up on this GPU and
    one call is run with the exchanges done in-process (so the payloads are
    real), then rank 0's quantize / reduce / decode are timed. The exchanges
    themselves are not timed (they need P GPUs); their bytes are printed."""
    import torch
    import workloads as W
    import bit_error_compensated_group_b200 as E
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = _workload()
    P, n, group, bits = w.P, w.n, w.group, w.bits
    fb = (w.eta, w.alpha_long, w.alpha_short, w.w)
    peak, peak_kind = _peak_hbm()
    G = -(-n // group)
    pb = group * bits // 8 + 4
    out = {}
    for feedback in (True, False):
        ranks = [E.EchoRank(n, P, r, group, bits, feedback, device=dev) for r in range(P)]
        xs = [W.rank_input(w, r, 0, dev) for r in range(P)]
        ys = [torch.empty_like(t) for t in xs]
        plans = [rk.plan(bits) for rk in ranks]
        for r in range(P):
            ranks[r].quantize(xs[r], bits, *fb)
        E.exchange_in_process(plans, "all_to_all")
        for r in range(P):
            ranks[r].reduce(xs[r], ys[r], bits, *fb)
        E.exchange_in_process(plans, "all_gather")
        for r in range(P):
            ranks[r].decode(ys[r], bits)
        torch.cuda.synchronize(dev)
        r0 = ranks[0]
        s = torch.cuda.current_stream(dev)
        steps = max(3, args.steps)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
        for i in range(args.warmup + steps):
            e = evs[i - args.warmup] if i >= args.warmup else None
            if e:
                e[0].record(s)
            r0.quantize(xs[0], bits, *fb)
            if e:
                e[1].record(s)
            r0.reduce(xs[0], ys[0], bits, *fb)
            if e:
                e[2].record(s)
            r0.decode(ys[0], bits)
            if e:
                e[3].record(s)
        torch.cuda.synchronize(dev)
        ms = [sum(e[k].elapsed_time(e[k + 1]) for e in evs) / steps for k in range(3)]
        seg = int(plans[0].layout.seg_groups)
        st = 16 if feedback else 0
        nbytes = [(G - seg) * (2 * group + st * group + pb),                        # x, EMAs, send row
                  seg * (2 * group + st * group + (P - 1) * pb + pb),               # x, EMAs, received rows, gather send
                  G * (pb + 2 * group)]                                            # gathered rows, output
        # the same kernels of rank 0 cut into column chunks (the chunked call's
        # compute side; its exchanges need P GPUs and are not timed here)
        per_chunks = {}
        for chunks in _chunk_counts(args):
            if chunks == 1:
                continue
            cevs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
            for i in range(args.warmup + steps):
                e = cevs[i - args.warmup] if i >= args.warmup else None
                if e:
                    e[0].record(s)
                for c in range(chunks):
                    r0.quantize_chunk(xs[0], c, chunks, bits, *fb)
                if e:
                    e[1].record(s)
                for c in range(chunks):
                    r0.reduce_chunk(xs[0], ys[0], c, chunks, bits, *fb)
                if e:
                    e[2].record(s)
                for c in range(chunks):
                    r0.decode_chunk(ys[0], c, chunks, bits)
                if e:
                    e[3].record(s)
            torch.cuda.synchronize(dev)
            cms = [sum(e[k].elapsed_time(e[k + 1]) for e in cevs) / steps for k in range(3)]
            per_chunks[str(chunks)] = {"phases_ms": {"quantize": cms[0], "reduce": cms[1], "decode": cms[2]},
                                       "ms": sum(cms)}
        rc, flags = r0.status()
        out["feedback" if feedback else "no_feedback"] = {
            "phases_ms": {"quantize": ms[0], "reduce": ms[1], "decode": ms[2]}, "ms": sum(ms),
            "algorithmic_bytes": {"quantize": nbytes[0], "reduce": nbytes[1], "decode": nbytes[2]},
            "roofline_frac": {k: b / (t * 1e-3) / 1e9 / peak for k, b, t in zip(("quantize", "reduce", "decode"),
                                                                               nbytes, ms)},
            "chunked_kernels": per_chunks,
            "status": rc, "flags": flags}
        for rk in ranks:
            rk.close()
        del ranks, xs, ys, plans
        torch.cuda.empty_cache()
    lay0 = E.echo_query_rank_layout(n, P, 0, group, bits, bits)
    seg0, segm = int(lay0.seg_groups), int(lay0.seg_max)
    print(json.dumps({"ranks": out, "config": {"workload": w.name, "P": P, "n": n, "group": group, "bits": bits,
                                               "rank": 0},
                      "exchange_bytes_per_rank": {"all_to_all_out": (G - seg0) * pb, "all_to_all_in": (P - 1) * seg0 * pb,
                                                  "all_gather_in": (P - 1) * segm * pb},
                      "peak_gbs": peak, "peak_kind": peak_kind, "data": "synthetic"}), flush=True)


def run_dist(args):
    """The real multi-GPU call against NCCL's bf16 all-reduce (the pages'
    comparison): under torchrun, P = world size, one rank per GPU, each with
    its own 1 GB bf16 message (the same workload as the main line; rank r's
    input is the workload's rank r). Times, on each rank's stream and as the
    max over ranks, EchoRank.allreduce with and without feedback -- whole,
    and cut into each of --chunks column chunks with chunk c's exchanges
    overlapping chunk c + 1's kernels -- and torch.distributed.all_reduce
    (SUM) of the same bf16 tensor."""
    import torch
    import torch.distributed as dist
    import workloads as W
    import bit_error_compensated_group_b200 as E
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from datetime import timedelta
    if not dist.is_initialized():
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    w = _workload()
    n, group, bits = w.n, w.group, w.bits
    fb = (w.eta, w.alpha_long, w.alpha_short, w.w)
    x = W.rank_input(w, rank % w.P, 0, dev)
    y = torch.empty_like(x)
    s = torch.cuda.current_stream(dev)
    steps = max(3, args.steps)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        for _ in range(steps):
            fn()
        b.record(s)
        torch.cuda.synchronize(dev)
        dist.barrier()
        return max_over_ranks(a.elapsed_time(b) / steps, world, dev)

    out = {}
    comm = torch.cuda.Stream(dev)
    for feedback in (True, False):
        er = E.EchoRank(n, world, rank, group, bits, feedback, device=dev)
        for chunks in _chunk_counts(args):
            key = ("echo_feedback" if feedback else "echo_no_feedback") + ("" if chunks == 1 else f"_chunks{chunks}")
            out[key] = timed(lambda: er.allreduce(x, y, bits, *fb, chunks=chunks, comm_stream=comm))
        rc, flags = er.status()
        er.close()
        del er
        torch.cuda.empty_cache()
    z = x.clone()
    out["nccl_bf16_all_reduce"] = timed(lambda: dist.all_reduce(z))
    if rank == 0:
        line = {"dist": {k: {"ms_per_call": v, "gbs_bf16_per_rank": n * 2 / (v * 1e-3) / 1e9} for k, v in out.items()},
                "speedup_vs_nccl_bf16": {k: out["nccl_bf16_all_reduce"] / v for k, v in out.items()
                                         if k.startswith("echo")},
                "n_gpus": world, "P": world, "steps": steps, "warmup": args.warmup,
                "config": {"workload": w.name, "n": n, "group": group, "bits": bits}, "data": "synthetic"}
        print(json.dumps(line), flush=True)
    dist.barrier()
    dist.destroy_process_group()


def run_shapes(args):
    """The owners' pass and the quantize pass across P (and group sizes and
    widths): 2^28 N(0,1) elements per rank (512 MB), feedback on, through the
    phase entry points with an event between the two kernels; each kernel's
    fraction of the measured copy peak for its own algorithmic bytes."""
    import torch
    import bit_error_compensated_group_b200 as E
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peak, _ = _peak_hbm()
    n = 1 << 28
    fb = (1.0, 0.05, 0.5, 0.5)
    out = []
    for P, group, bits in [(2, 128, 4), (4, 128, 4), (8, 128, 4), (16, 128, 4), (8, 32, 4), (8, 256, 4),
                           (8, 128, 8)]:
        g = torch.Generator(device=dev)
        g.manual_seed(5)
        inputs = [torch.randn(n, generator=g, device=dev).to(torch.bfloat16) for _ in range(P)]
        outputs = [torch.empty_like(t) for t in inputs]
        ar = E.EchoAllReduce(n, P, group, bits, True)
        try:
            def step(evs=None):
                if evs is not None:
                    evs[0].record(stream)
                E.echo_phase_quantize(inputs, ar.handle, bits, *fb, stream=stream)
                if evs is not None:
                    evs[1].record(stream)
                E.echo_phase_reduce(inputs, outputs, ar.handle, bits, *fb, stream=stream)
                if evs is not None:
                    evs[2].record(stream)
            for _ in range(args.warmup):
                step()
            torch.cuda.synchronize(dev)
            evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
            for e in evs:
                step(e)
            torch.cuda.synchronize(dev)
            rc, flags = ar.status()
        finally:
            ar.close()
        q = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
        r = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
        ab = algorithmic_bytes(P, n, group, bits)
        out.append({"P": P, "group": group, "bits": bits, "quantize_ms": q, "reduce_ms": r, "call_ms": q + r,
                    "call_frac": ab["total"] / ((q + r) * 1e-3) / 1e9 / peak,
                    "quantize_frac": ab["quantize"] / (q * 1e-3) / 1e9 / peak,
                    "reduce_frac": ab["reduce_gather"] / (r * 1e-3) / 1e9 / peak, "status": rc, "flags": flags})
        del inputs, outputs
        torch.cuda.empty_cache()
    print(json.dumps({"shapes": out, "elements_per_rank": n, "steps": args.steps, "warmup": args.warmup,
                      "peak_gbs": peak}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="echo", choices=["echo", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-chunk", type=int, default=0,
                    help="group columns per chunk of the host-buffer call (0: the library's default, G/16)")
    ap.add_argument("--no-variants", action="store_true", help="skip the no-feedback, quantizer-form and 8-bit timings")
    ap.add_argument("--feedback", choices=["on", "off"], default="on",
                    help="off: time the call without EMA state as the main step (profiling)")
    ap.add_argument("--ablation", action="store_true",
                    help="print the accuracy ablations on the synthetic chains instead of timing")
    ap.add_argument("--dist", action="store_true",
                    help="under torchrun: the multi-GPU call (P = world size) against NCCL's bf16 all-reduce")
    ap.add_argument("--ranks", action="store_true",
                    help="print one rank's kernel times of a multi-GPU call (rank 0 of P = 8, 1 GB) instead")
    ap.add_argument("--shapes", action="store_true",
                    help="print each kernel's time and roofline fraction across P, group size and width "
                         "(512 MB per rank) instead")
    ap.add_argument("--workloads", action="store_true",
                    help="print every workload's GPU and oracle time per call instead of the main line")
    ap.add_argument("--background", default=None,
                    help="background-traffic study: comma-separated load levels in %% (e.g. 0,25,50,75,100)")
    ap.add_argument("--chunks", default="1,4,16",
                    help="--dist / --ranks: column-chunk counts of the multi-GPU call (comma-separated)")
    ap.add_argument("--split", choices=["columns", "messages"], default="columns",
                    help="with N > 1 GPUs: split the one message by group columns (strong scaling, default) "
                         "or give every GPU its own message (weak scaling)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="tokens per rank (default 131072, the 1 GB message); smaller values are for profiling")
    args = ap.parse_args()
    global _TOKENS, _FEEDBACK
    _TOKENS = args.tokens
    _FEEDBACK = args.feedback == "on"
    if args.impl == "reference":
        run_reference(args)
    elif args.ablation:
        run_ablation(args)
    elif args.workloads:
        run_workloads(args)
    elif args.shapes:
        run_shapes(args)
    elif args.ranks:
        run_ranks(args)
    elif args.background is not None:
        run_background(args)
    elif args.dist:
        run_dist(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
