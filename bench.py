#!/usr/bin/env python
"""Throughput benchmark of the MRU prefix-product scan on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = one call of mru_scan_fused over the whole workload (lift + chunk
prefixes + chunk-total scan + fix-up, every kernel of the path) with the
embeddings already resident in HBM.  The default workload is the largest
single-GPU configuration the metric is quoted on: the n = 16, B1 H8 L262144
determinant-corrected scan (x [1, 262144, 2048] fp32 in, every S_t
[1, 262144, 8, 16, 16] fp32 out).  Rank 0 prints one JSON line; at N = 1 it
also carries `per_workload`, the same measurement for each of the five
configurations (n4, n16 B8, n32 LDU, n16 long, n64 readout).

Multi-GPU (torchrun, one process per GPU): the (b, h) sequences are
independent, so every rank scans its own replica of the workload with no
data-path collective ("scaling": "weak"); NCCL is used only for the barrier
and the max over ranks of the timed region.

--impl reference times the fp64 CPU oracle on the host cores, on a bounded
sample of the same workload per step (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_rnn_scan_b200 import inputs as gen  # noqa: E402

METRIC = "MRU scan tokens·heads/s and achieved % of HBM/tensor roofline, 1×B200"
UNIT = "token·heads/s"
DEFAULT_WORKLOAD = "n16_detnorm_b1h8l262144"
L2_BYTES = 126 * 1024 * 1024


def env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


class Ranks:
    """One process per GPU, rank and world size from the launcher's
    environment (RANK, WORLD_SIZE, LOCAL_RANK, MASTER_ADDR/PORT).  The only
    collectives are the barrier around the timed regions and the max over
    ranks of their durations; rank 0 prints."""

    def __init__(self, backend: str = "nccl", device=None, timeout_s: float = 120.0):
        self.rank, self.world = env_int("RANK", 0), env_int("WORLD_SIZE", 1)
        self.local = env_int("LOCAL_RANK", 0)
        self.device = device
        self.dist = None
        if self.world > 1:
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
            self.dist = dist

    @property
    def printer(self) -> bool:
        return self.rank == 0

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max(self, v: float) -> float:
        if self.dist is None:
            return v
        import torch
        t = torch.tensor([v], device=self.device, dtype=torch.float64)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist is not None:
            self.dist.destroy_process_group()
            self.dist = None


def aggregate_rate(world: int, units_per_rank: int, ms_max: float) -> float:
    """Whole-job throughput: every rank processed its units within the
    slowest rank's time."""
    return world * units_per_rank / (ms_max / 1e3)


# ------------------------------------------------------------ bookkeeping ---

def step_bytes(w: gen.Workload) -> dict:
    """Algorithmic HBM bytes of one step: embeddings in, results out."""
    nn = w.n * w.n
    xb = 2 if w.x_dtype == "bf16" else 4
    x_bytes = w.token_heads * nn * xb
    if w.readout:
        out = w.token_heads * w.n * max(w.queries, 1) * 4
        if w.snapshot_every:
            out += w.B * (w.L // w.snapshot_every) * w.H * nn * 4
    else:
        out = w.token_heads * nn * 4
    return {"in": x_bytes, "out": out, "total": x_bytes + out}


def kernel_bytes(name: str, w: gen.Workload, chunk: int) -> int:
    """Bytes one launch of a kernel must move by its own design (per launch =
    the whole workload).  Generic path: the chunk kernel reads the embeddings
    and writes the local prefixes Q_t where S_t goes plus the chunk totals;
    the fix-up reads Q_t and writes S_t.  Two-pass paths: the reduce pass
    reads the embeddings and writes the chunk totals; the apply pass reads
    the embeddings and each chain's carry factors and writes S_t; the carry
    kernels touch only chunk totals, in-group prefixes and carries.  The
    one-launch small kernel reads the embeddings and writes S_t (its second
    pass over a sequence's embeddings is meant to hit L2)."""
    nn = w.n * w.n
    sb = step_bytes(w)
    K = -(-w.L // chunk)
    chains = w.B * w.H * K
    tot = chains * nn                       # elements of all chunk totals
    groups = -(-chains // 16)
    if name == "k_small_scan":
        return sb["in"] + sb["out"]
    if name == "k16_fused":
        # embeddings in once (the apply items read them again from L2), S_t
        # out, chunk totals and in-group prefixes, per-token scalars
        cdb = w.token_heads * 8 if w.mode == gen.MODE_DETNORM else 0
        return sb["in"] + sb["out"] + tot * (4 + 4) + cdb
    if "chunk" in name:
        return sb["in"] + sb["out"] + tot * 4
    if "fixup" in name:
        return 2 * sb["out"] + tot * 4
    if "reduce" in name:
        return sb["in"] + tot * 4
    if "apply" in name:
        return sb["in"] + sb["out"] + chains * nn * (8 + 4)
    if name == "k16_carry":
        return tot * (4 + 4) + groups * nn * (8 + 8)
    if name == "k_level":
        return tot * (4 + 4) + groups * nn * 8
    if name in ("k_top", "k_down"):
        return groups * nn * 16
    if name.endswith("carry_local"):
        return tot * (4 + 8)
    if name.endswith("carry_groups"):
        G = max(1, math.isqrt(K - 1) + 1) if K > 1 else 1
        return w.B * w.H * (-(-K // G)) * nn * 16
    if name.endswith("carry_final"):
        return tot * (8 + 8 + 4)
    return 0


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


KERNEL_SOURCES = {"k16_": "mru_n16.cu", "k16b_": "mru_n16.cu", "k32_": "mru_n32.cu", "k32b_": "mru_n32.cu",
                  "k64_": "mru_n64.cu", "k64b_": "mru_n64_bwd.cu",
                  "k_level": "mru_carry.cu", "k_top": "mru_carry.cu", "k_down": "mru_carry.cu"}


def kernel_source(kernel: str) -> str:
    for prefix, f in KERNEL_SOURCES.items():
        if kernel.startswith(prefix):
            return f
    return "mru_scan_v1.cu"


def csrc_hash(kernel: str) -> str:
    """sha256 of the source file that holds the kernel and the shared
    internal header (a capture stays valid while neither changes)."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "linear_rnn_scan_b200", "csrc")
    for name in (kernel_source(kernel), "mru_internal.cuh"):
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rows = json.load(f)
    except Exception:
        return None
    cur = csrc_hash(kernel)
    for r in rows:
        if r.get("workload") == workload and r.get("kernel") == kernel and r.get("csrc_sha256") == cur:
            return float(r["dram_bytes_per_launch"])
    return None


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML during a region."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.period = period_s
        self.samples = []
        self.stop_ev = threading.Event()
        self.thread = None
        self.max_mhz = None
        self.err = None
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = device_index
            if vis:
                ids = [v.strip() for v in vis.split(",") if v.strip()]
                if device_index < len(ids) and ids[device_index].isdigit():
                    idx = int(ids[device_index])
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report the absence
            self.nv = None
            self.err = str(e)

    def _run(self):
        nv = self.nv
        while not self.stop_ev.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((time.time(), sm, rs))
            except Exception as e:
                self.err = str(e)
            self.stop_ev.wait(self.period)

    def __enter__(self):
        if self.nv is not None:
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        return self

    def __exit__(self, *a):
        self.stop_ev.set()
        if self.thread:
            self.thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": self.err or "no samples"}
        mhz = [s[1] for s in self.samples]
        bits = 0
        for s in self.samples:
            bits |= int(s[2])
        reasons = [name for b, name in sorted(self.REASONS.items()) if bits & b and name != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(mhz)), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(mhz), "sm_mhz_min": min(mhz)}


# ------------------------------------------------------------- CPU oracle ---

def oracle_rate(w: gen.Workload, x_np, target_s: float, nthreads: int):
    """Times the fp64 oracle (as it stands) on a bounded sample of the
    workload: the first t_end tokens of every (b, h) sequence (a spread
    subset when there are many more sequences than threads), repeated until
    about target_s seconds of work when the whole workload is quicker."""
    import oracle
    p = oracle.make_problem(w.B, w.H, w.L, w.n, x_dtype=w.x_dtype, mode=w.mode, alpha=w.alpha,
                            add_identity=w.add_identity, ldu_offdiag=w.ldu_offdiag, ldu_diag=w.ldu_diag)
    nbh = w.B * w.H
    seqs = min(nbh, max(4 * nthreads, 1))
    bh = np.linspace(0, nbh - 1, seqs).round().astype(np.int64)
    # calibrate on a short prefix
    t_cal = min(w.L, 16)
    t0 = time.perf_counter()
    oracle.compare(p, x_np, bh=bh, t_end=t_cal, nthreads=nthreads)
    dt = max(time.perf_counter() - t0, 1e-4)
    per_token = dt / t_cal
    t_end = int(min(w.L, max(t_cal, target_s / per_token)))
    reps, units, el = 0, 0, 0.0
    while True:
        t0 = time.perf_counter()
        oracle.compare(p, x_np, bh=bh, t_end=t_end, nthreads=nthreads)
        el += time.perf_counter() - t0
        units += len(bh) * t_end
        reps += 1
        if el >= 0.5 * target_s or reps >= 1000:
            break
    sample = (f"first {t_end} of {w.L} tokens of {len(bh)} of {nbh} (b,h) sequences, x{reps}, fp64, "
              f"{nthreads} threads")
    return units / el, units, el, sample


def run_reference(args, w):
    rank = env_int("RANK", 0)
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    nthreads = os.cpu_count() or 1
    x_np = gen.make_x(w)
    per_step = float(os.environ.get("MRU_REF_STEP_SECONDS", "3.0"))
    for _ in range(args.warmup):
        oracle_rate(w, x_np, 0.2, nthreads)
    rates, units_all, secs_all, sample = [], 0, 0.0, ""
    for _ in range(args.steps):
        r, u, s, sample = oracle_rate(w, x_np, per_step, nthreads)
        rates.append(r)
        units_all += u
        secs_all += s
    value = units_all / secs_all
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * secs_all / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, None),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                         "sample": f"per step: {sample}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, chunk):
    sb = step_bytes(w)
    return {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "n": w.n, "x_dtype": w.x_dtype,
            "mode": ["reshape", "detnorm", "ldu", "cayley", "expm"][w.mode], "readout": w.readout,
            "snapshot_every": w.snapshot_every, "chunk": chunk,
            **({"query_columns": w.queries} if w.queries else {}),
            "l2": ("inputs larger than L2: x %.0f MiB in, %.0f MiB out per step" %
                   (sb["in"] / 2 ** 20, sb["out"] / 2 ** 20)) if sb["total"] > L2_BYTES
            else "inputs smaller than L2: L2 flushed (252 MiB written) between timed steps, outside the events",
            "parallelism": "single GPU; replicas across GPUs (independent (b,h) sequences)"}


# ------------------------------------------------------------------- ours ---

# The five workloads the benchmark's metric is quoted on (n4, n16 B8, n32
# LDU, n16 long, n64 readout), reported together in `per_workload`.
BASELINE_WORKLOADS = ["n4_reshape_l1024", "n16_detnorm_b8h8l4096", "n32_ldu_bf16_b4h16l8192",
                      "n16_detnorm_b1h8l262144", "n64_detnorm_readout_b2h4l16384"]

# Tensor pipe each workload's products run on and its peak in TFLOP/s: the
# contraction's own dtype, from MEASURED_PEAKS.json's bf16 figure times the
# nominal dense ratio (tf32 1.1 / bf16 2.25 PFLOP/s).  The kernels issue
# mma.sync, whose measured ceiling on this part is lower (tf32 279, bf16
# 557 TFLOP/s); every workload is bound by HBM either way.
NOMINAL_TF32_OVER_BF16 = 1.1 / 2.25


def flop_side(w: gen.Workload, peaks) -> dict:
    """Algorithmic scan FLOPs (2 n^3 per token-head) over the peak of the
    pipe the path's products use."""
    flops = 2.0 * w.n ** 3 * w.token_heads
    if w.n == 32 and w.x_dtype == "bf16":
        pipe, tf = "bf16 tensor (split bf16)", peaks["bf16_tflops"]
    elif w.n in (16, 64):
        pipe, tf = "tf32 tensor", peaks["bf16_tflops"] * NOMINAL_TF32_OVER_BF16
    else:
        pipe, tf = "fp32 FMA (SIMT, nominal 74.4)", 74.4
    return {"flops_per_step": flops, "pipe": pipe, "peak_tflops": tf, "min_ms": flops / (tf * 1e12) * 1e3}


def roofline_min_ms(w: gen.Workload, peaks) -> dict:
    """The slower of the bytes at HBM peak and the scan FLOPs at the pipe's
    peak: the roofline time of one step."""
    sb = step_bytes(w)
    hbm_ms = sb["total"] / (peaks["hbm_gbs"] * 1e9) * 1e3
    fl = flop_side(w, peaks)
    bound = "hbm" if hbm_ms >= fl["min_ms"] else "tensor"
    return {"bytes_per_step": sb["total"], "hbm_min_ms": hbm_ms, "flop": fl, "bound": bound,
            "min_ms": max(hbm_ms, fl["min_ms"])}


class Case:
    """One workload resident on the device: inputs, outputs, workspace and
    the call, through the C-ABI."""

    def __init__(self, w, dev, stream, seed_offset=0, x_np=None):
        import torch

        from linear_rnn_scan_b200 import mru
        self.w, self.mru = w, mru
        self.p = mru.problem_from_workload(w)
        self.chunk = mru.chosen_chunk(self.p, w.readout)
        self.stream = stream
        if x_np is None:
            x_np = gen.make_x(w, seed=w.seed + seed_offset)
        if w.x_dtype == "bf16":
            x_host = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16)
        else:
            x_host = torch.from_numpy(x_np)
        self.x_pin = x_host.pin_memory()
        self.x_dev = self.x_pin.to(dev)
        self.ws = mru.workspace_t(self.p, dev)
        self.ro = None
        if w.readout:
            self.u = torch.from_numpy(gen.make_u(w)).to(dev)
            o = torch.empty((w.B, w.L, w.H, w.n) + ((w.queries,) if w.queries else ()), dtype=torch.float32,
                            device=dev)
            snaps = (torch.empty((w.B, w.L // w.snapshot_every, w.H, w.n, w.n), dtype=torch.float32, device=dev)
                     if w.snapshot_every else None)
            self.ro = mru.Readout(self.u.data_ptr(), w.snapshot_every,
                                  snaps.data_ptr() if snaps is not None else None, w.queries, 1 if w.queries else 0)
            self.outs_dev = [o] + ([snaps] if snaps is not None else [])
        else:
            self.outs_dev = [torch.empty((w.B, w.L, w.H, w.n, w.n), dtype=torch.float32, device=dev)]
        self.names = mru.kernel_names(self.p, w.readout)
        self.launches = mru.launch_count(self.p, w.readout)

    def step(self):
        mru, o = self.mru, self.outs_dev[0]
        if self.ro is not None:
            rc = mru.scan_fused(self.p, self.x_dev.data_ptr(), None, self.ro, None, o.data_ptr(), self.ws.data_ptr(),
                                self.ws.numel(), self.stream.cuda_stream)
        else:
            rc = mru.scan_fused(self.p, self.x_dev.data_ptr(), None, None, o.data_ptr(), None, self.ws.data_ptr(),
                                self.ws.numel(), self.stream.cuda_stream)
        if rc != mru.OK:
            raise mru.MruError(rc, "mru_scan_fused")

    def check_status(self, what):
        st = self.mru.last_device_status(self.ws.data_ptr(), self.stream.cuda_stream)
        if st != self.mru.OK:
            raise self.mru.MruError(st, what)

    def time_steps(self, steps, dev, clocks=None):
        """Device time of `steps` calls (CUDA events on the launching
        stream); workloads smaller than L2 get an L2 flush (a write of twice
        its size) between steps, outside the per-step events."""
        import torch
        stream = self.stream
        if step_bytes(self.w)["total"] > L2_BYTES:
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ev0.record(stream)
            for _ in range(steps):
                self.step()
            ev1.record(stream)
            ev1.synchronize()
            return ev0.elapsed_time(ev1) / steps
        flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
        pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for a, b in pairs:
            flush.zero_()
            a.record(stream)
            self.step()
            b.record(stream)
        pairs[-1][1].synchronize()
        return sum(a.elapsed_time(b) for a, b in pairs) / steps

    def kernel_times(self, steps):
        """Mean device time of each of the call's launches over `steps`
        calls, from the library's event hook."""
        import torch
        n_k = self.launches
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * n_k)] for _ in range(steps)]
        for row in evs:
            for e in row:
                e.record(self.stream)           # creates the handles
        torch.cuda.synchronize()
        for row in evs:
            self.mru.set_profile_events([e.cuda_event for e in row])
            self.step()
        self.mru.set_profile_events(None)
        torch.cuda.synchronize()
        return [statistics.mean(row[2 * i].elapsed_time(row[2 * i + 1]) for row in evs) for i in range(n_k)]


def roofline_entry(w, ms, per_kernel, names, chunk, peaks):
    """The dominant kernel's roofline (algorithmic bytes of the whole step,
    which that kernel's launch processes, over its launch time) and the whole
    call's fraction of the step's roofline time."""
    rl = roofline_min_ms(w, peaks)
    dom = int(np.argmax(per_kernel))
    dom_name = names[dom]
    sb = step_bytes(w)
    achieved = sb["total"] / (per_kernel[dom] / 1e3) / 1e9
    whole = rl["min_ms"] / ms
    roof = {"bound": rl["bound"], "kernel": dom_name, "achieved": achieved, "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
            "frac_whole_call": whole,
            "traffic": recorded_traffic(w.name, dom_name),
            "algorithmic_bytes_per_launch": sb["total"], "avg_launch_ms": per_kernel[dom],
            "kernel_own_bytes_per_launch": kernel_bytes(dom_name, w, chunk),
            "flop_side": {"flops_per_step": rl["flop"]["flops_per_step"], "pipe": rl["flop"]["pipe"],
                          "peak_tflops": round(rl["flop"]["peak_tflops"], 1),
                          "achieved_tflops": rl["flop"]["flops_per_step"] / (ms / 1e3) / 1e12,
                          "min_ms": rl["flop"]["min_ms"]},
            "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json hbm_gbs)" if peaks["source"] == "measured"
            else "fallback 6.65 TB/s"}
    path = {"algorithmic_bytes_per_step": sb["total"], "achieved_gbs": sb["total"] / (ms / 1e3) / 1e9,
            "frac_of_hbm_peak": sb["total"] / (ms / 1e3) / 1e9 / peaks["hbm_gbs"],
            "roofline_ms": rl["min_ms"], "frac_of_roofline": whole}
    return roof, path


def measure_case(case, args, dev, clocks=None):
    """Warm-up, the timed region (K steps), then the per-kernel split."""
    for _ in range(args.warmup):
        case.step()
    case.check_status("device status after warm-up")
    import torch
    torch.cuda.synchronize()
    ms = case.time_steps(args.steps, dev)
    case.check_status("device status after timing")
    per_kernel = case.kernel_times(min(args.steps, 10))
    return ms, per_kernel


def per_workload_lines(args, dev, stream, peaks, skip_name, skip_entry):
    """Every workload the metric is quoted on, one entry each (rank 0 at
    N = 1): step time, throughput, the whole call's fraction of its roofline,
    the dominant kernel and its fraction, and the per-kernel split."""
    import torch
    out = {}
    for name in BASELINE_WORKLOADS:
        if name == skip_name:
            out[name] = skip_entry
            continue
        w = gen.WORKLOADS[name]
        case = Case(w, dev, stream)
        ms, per_kernel = measure_case(case, args, dev)
        roof, path = roofline_entry(w, ms, per_kernel, case.names, case.chunk, peaks)
        out[name] = {"ms_per_step": ms, "value": w.token_heads / (ms / 1e3), "unit": UNIT,
                     "frac_whole_call": roof["frac_whole_call"], "bound": roof["bound"],
                     "dominant_kernel": roof["kernel"], "dominant_kernel_frac": roof["frac"],
                     "roofline_ms": path["roofline_ms"], "chunk": case.chunk,
                     "kernels_ms": {case.names[i]: round(per_kernel[i], 5) for i in range(len(per_kernel))}}
        del case
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return out


def run_ours(args, w):
    import torch

    from linear_rnn_scan_b200 import mru

    local = env_int("LOCAL_RANK", 0)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    rank, world = ranks.rank, ranks.world
    barrier, max_over_ranks = ranks.barrier, ranks.max

    # CPU baseline first (rank 0, one GPU), before any CUDA work.
    cpu = None
    x_np = gen.make_x(w, seed=w.seed + rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        nthreads = os.cpu_count() or 1
        r, units, el, sample = oracle_rate(w, x_np, args.cpu_seconds, nthreads)
        cpu = {"value": r, "unit": UNIT, "cores": nthreads, "kind": "oracle", "sample": sample,
               "seconds": round(el, 2)}

    stream = torch.cuda.current_stream()
    case = Case(w, dev, stream, x_np=x_np)
    del x_np
    peaks = read_peaks()
    for _ in range(args.warmup):
        case.step()
    case.check_status("device status after warm-up")

    # timed region: exactly K steps, device-resident inputs
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        ms = case.time_steps(args.steps, dev)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(ms)
    value = aggregate_rate(world, w.token_heads, ms)
    case.check_status("device status after timing")

    per_kernel = case.kernel_times(min(args.steps, 10))
    roofline, path = roofline_entry(w, ms, per_kernel, case.names, case.chunk, peaks)
    kernels_ms = {case.names[i]: round(per_kernel[i], 5) for i in range(len(per_kernel))}

    # e2e: the C-ABI call with HOST buffers (mru_scan_fused_host): the upload
    # of x, the scan and the download of every output, pipelined over pieces
    # on three streams, all inside the timed region
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    outs_host = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in case.outs_dev]
    h2d = case.x_pin.numel() * case.x_pin.element_size()
    d2h = sum(t.numel() * t.element_size() for t in outs_host)
    s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    snaps_host = outs_host[1].data_ptr() if len(outs_host) > 1 else None

    def call_host():
        rc = mru.scan_fused_host(case.p, case.x_pin.data_ptr(), None, case.ro, outs_host[0].data_ptr(), snaps_host,
                                 case.x_dev.data_ptr(), case.outs_dev[0].data_ptr(), case.ws.data_ptr(),
                                 case.ws.numel(), 0, stream.cuda_stream, s_h2d.cuda_stream, s_d2h.cuda_stream)
        if rc != mru.OK:
            raise mru.MruError(rc, "mru_scan_fused_host")

    call_host()                                   # warm-up of the pipelined path
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        call_host()
    e1.record(stream)
    e1.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps)
    case.check_status("device status after the end-to-end timing")
    launches = case.launches
    chunk = case.chunk
    del case, outs_host
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    per_workload = None
    if world == 1 and not args.no_per_workload:
        head = {"ms_per_step": ms, "value": value, "unit": UNIT, "frac_whole_call": roofline["frac_whole_call"],
                "bound": roofline["bound"], "dominant_kernel": roofline["kernel"],
                "dominant_kernel_frac": roofline["frac"], "roofline_ms": path["roofline_ms"], "chunk": chunk,
                "kernels_ms": kernels_ms}
        per_workload = per_workload_lines(args, dev, stream, peaks, w.name, head)

    if rank == 0:
        cfg = workload_config(w, chunk)
        clk = clocks.summary()
        if clk.get("sm_mhz"):
            clk["ms_x_sm_mhz"] = ms * clk["sm_mhz"]
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded N(0,1) embeddings)",
            "config": cfg, "clocks": clk,
            "e2e": {"value": aggregate_rate(world, w.token_heads, e2e_ms), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "api": "mru_scan_fused_host (pinned host buffers; upload, scan and download "
                           "pipelined over pieces on three streams)",
                    "ms_per_step": e2e_ms},
            "gpu_launches": launches * args.steps,
            "roofline": roofline, "path_roofline": path, "kernels_ms": kernels_ms,
        }
        if per_workload is not None:
            line["per_workload"] = per_workload
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    ranks.close()
    return 0


def bwd_kernel_names(w):
    """The three launches of mru_scan_backward for this workload: the tensor-core
    passes where the library has them (n = 16 fp32 reshape / corrected with the
    identity / Cayley map, n = 32 LDU bf16, n = 64 fp32 reshape / corrected in
    tf32), the
    generic kernels otherwise; the chunk-gradient
    scan between them is always the generic one ("chunk_scan": k_bwd_carry
    serially, or k_bwd_group, k_bwd_top and k_bwd_fix in groups for larger
    problems)."""
    if w.n == 16 and w.x_dtype == "f32" and (w.mode in (gen.MODE_RESHAPE, gen.MODE_CAYLEY) or
                                              (w.mode == gen.MODE_DETNORM and w.add_identity)):
        return ["k16b_local", "chunk_scan", "k16b_apply"]
    if w.n == 32 and w.x_dtype == "bf16" and w.mode == gen.MODE_LDU:
        return ["k32b_local", "chunk_scan", "k32b_apply"]
    if w.n == 64 and w.x_dtype == "f32" and w.math == "tf32" and w.mode in (gen.MODE_RESHAPE, gen.MODE_DETNORM):
        return ["k64b_local", "chunk_scan", "k64b_apply"]
    return ["k_bwd_local", "chunk_scan", "k_bwd_apply"]


def run_backward(args, w):
    """One step = one mru_scan_backward over the whole workload (gradients of
    sum <dS, S> with respect to the embeddings), with x, the forward states
    and the upstream gradients resident in HBM.  Not part of the default run."""
    import torch

    from linear_rnn_scan_b200 import mru

    if w.readout:
        return run_backward_readout(args, w)
    local = env_int("LOCAL_RANK", 0)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    p = mru.problem_from_workload(w)
    x_np = gen.make_x(w, seed=w.seed + ranks.rank)
    if w.x_dtype == "bf16":
        x = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).to(dev)
    else:
        x = torch.from_numpy(x_np).to(dev)
    S = mru.scan_fused_t(p, x)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed + 17)
    dS = torch.randn(S.shape, generator=g, device=dev, dtype=torch.float32)
    dx = torch.empty((w.B, w.L, w.H * w.n * w.n), dtype=torch.float32, device=dev)
    ws = torch.empty(mru.backward_workspace_size(p), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        rc = mru.scan_backward(p, x.data_ptr(), None, S.data_ptr(), dS.data_ptr(), dx.data_ptr(), None,
                               ws.data_ptr(), ws.numel(), stream.cuda_stream)
        if rc != mru.OK:
            raise mru.MruError(rc, "mru_scan_backward")

    for _ in range(args.warmup):
        step()
    st = mru.last_device_status(ws.data_ptr(), stream.cuda_stream)
    if st != mru.OK:
        raise mru.MruError(st, "device status after warm-up")
    torch.cuda.synchronize()
    ranks.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        ev1.synchronize()
    torch.cuda.synchronize()
    ranks.barrier()
    ms = ranks.max(ev0.elapsed_time(ev1) / args.steps)
    names = bwd_kernel_names(w)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    for e in evs:
        e.record(stream)
    torch.cuda.synchronize()
    mru.set_profile_events([e.cuda_event for e in evs])
    step()
    mru.set_profile_events(None)
    torch.cuda.synchronize()
    kms = {names[i]: round(evs[2 * i].elapsed_time(evs[2 * i + 1]), 5) for i in range(3)}
    # algorithmic bytes per token-head: x in, forward state in, upstream
    # gradient in, embedding gradient out
    nn = w.n * w.n
    xb = 2 if w.x_dtype == "bf16" else 4
    unit_bytes = nn * (xb + 4 + 4 + 4)
    peaks = read_peaks()
    dom = max(kms, key=kms.get)
    achieved = unit_bytes * w.token_heads / (kms[dom] / 1e3) / 1e9
    if ranks.printer:
        print(json.dumps({
            "metric": "MRU scan backward token·heads/s, 1×B200", "direction": "backward",
            "value": aggregate_rate(ranks.world, w.token_heads, ms), "unit": UNIT, "n_gpus": ranks.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded N(0,1) embeddings "
            "and upstream gradients)", "config": workload_config(w, None), "clocks": clocks.summary(),
            "gpu_launches": 3 * args.steps, "kernels_ms": kms,
            "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "algorithmic_bytes_per_launch": unit_bytes * w.token_heads}}), flush=True)
    ranks.close()
    return 0


def run_backward_readout(args, w):
    """One step = one mru_scan_backward_readout over the whole workload: the
    gradients of the readout outputs (o_t = S_t U, and the snapshots) to the
    embeddings, no forward state kept by the caller (the call recomputes the
    states in its workspace).  Not part of the default run."""
    import torch

    from linear_rnn_scan_b200 import mru

    local = env_int("LOCAL_RANK", 0)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    p = mru.problem_from_workload(w)
    x_np = gen.make_x(w, seed=w.seed + ranks.rank)
    if w.x_dtype == "bf16":
        x = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).to(dev)
    else:
        x = torch.from_numpy(x_np).to(dev)
    del x_np
    u = torch.from_numpy(gen.make_u(w)).to(dev)
    q = max(w.queries, 1)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed + 17)
    d_o = torch.randn((w.B, w.L, w.H, w.n, q), generator=g, device=dev, dtype=torch.float32)
    d_sn = (torch.randn((w.B, w.L // w.snapshot_every, w.H, w.n, w.n), generator=g, device=dev,
                        dtype=torch.float32) if w.snapshot_every else None)
    dx = torch.empty((w.B, w.L, w.H * w.n * w.n), dtype=torch.float32, device=dev)
    ws = torch.empty(mru.backward_readout_workspace_size(p), dtype=torch.uint8, device=dev)
    ro = mru.Readout(u.data_ptr(), w.snapshot_every, None, w.queries, 1 if w.queries else 0)
    stream = torch.cuda.current_stream()

    def step():
        rc = mru.scan_backward_readout(p, x.data_ptr(), None, ro, d_o.data_ptr(),
                                       d_sn.data_ptr() if d_sn is not None else None, dx.data_ptr(), None,
                                       ws.data_ptr(), ws.numel(), stream.cuda_stream)
        if rc != mru.OK:
            raise mru.MruError(rc, "mru_scan_backward_readout")

    for _ in range(args.warmup):
        step()
    st = mru.last_device_status(ws.data_ptr(), stream.cuda_stream)
    if st != mru.OK:
        raise mru.MruError(st, "device status after warm-up")
    torch.cuda.synchronize()
    ranks.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        ev1.synchronize()
    torch.cuda.synchronize()
    ranks.barrier()
    ms = ranks.max(ev0.elapsed_time(ev1) / args.steps)
    # algorithmic bytes per token-head: x in, the readout gradient in, dx out
    nn = w.n * w.n
    xb = 2 if w.x_dtype == "bf16" else 4
    unit_bytes = nn * xb + w.n * q * 4 + nn * 4
    snap_bytes = (w.B * (w.L // w.snapshot_every) * w.H * nn * 4) if w.snapshot_every else 0
    algo = unit_bytes * w.token_heads + snap_bytes
    peaks = read_peaks()
    achieved = algo / (ms / 1e3) / 1e9
    if ranks.printer:
        print(json.dumps({
            "metric": "MRU readout backward token·heads/s, 1×B200", "direction": "backward_readout",
            "value": aggregate_rate(ranks.world, w.token_heads, ms), "unit": UNIT, "n_gpus": ranks.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded N(0,1) embeddings and readout gradients)", "config": workload_config(w, None),
            "clocks": clocks.summary(),
            "roofline": {"bound": "hbm", "scope": "whole call", "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "algorithmic_bytes_per_step": algo,
                         "note": "the call recomputes every state into its workspace (the forward's full-state "
                                 "scan), forms dL/dS_t = do_t U^T there, and runs the scan's backward"}}),
              flush=True)
    ranks.close()
    return 0


def run_decode(args, w):
    """One step = one decode token for every (b, h) sequence of the workload:
    mru_scan_fused with L = 1 started from the previous step's state (S0),
    the single-launch path.  Reports the device time per step."""
    import torch

    from linear_rnn_scan_b200 import mru

    if w.readout:
        print(json.dumps({"impl": "ours", "direction": "decode", "unavailable":
                          "decode is timed on the full-state output"}), flush=True)
        return 0
    local = env_int("LOCAL_RANK", 0)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    wd = w.with_(L=1)
    p = mru.problem_from_workload(wd)
    total = args.warmup + args.steps
    xs = gen.make_x(w.with_(L=total), seed=w.seed + ranks.rank)      # one token per step, [B, total, D]
    if w.x_dtype == "bf16":
        xt = torch.from_numpy(xs.view(np.int16)).view(torch.bfloat16)
    else:
        xt = torch.from_numpy(xs)
    x_steps = [xt[:, t:t + 1].contiguous().to(dev) for t in range(total)]
    state = [torch.empty((w.B, 1, w.H, w.n, w.n), dtype=torch.float32, device=dev) for _ in range(2)]
    state[0].copy_(torch.eye(w.n, device=dev).expand(w.B, 1, w.H, w.n, w.n))
    ws = mru.workspace_t(p, dev)
    stream = torch.cuda.current_stream()

    def step(t):
        src, dst = state[t % 2], state[(t + 1) % 2]
        rc = mru.scan_fused(p, x_steps[t].data_ptr(), src.data_ptr(), None, dst.data_ptr(), None,
                            ws.data_ptr(), ws.numel(), stream.cuda_stream)
        if rc != mru.OK:
            raise mru.MruError(rc, "mru_scan_fused (decode)")

    for t in range(args.warmup):
        step(t)
    torch.cuda.synchronize()
    ranks.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for t in range(args.warmup, total):
            step(t)
        ev1.record(stream)
        ev1.synchronize()
    torch.cuda.synchronize()
    ranks.barrier()
    ms = ranks.max(ev0.elapsed_time(ev1) / args.steps)
    st = mru.last_device_status(ws.data_ptr(), stream.cuda_stream)
    if st != mru.OK:
        raise mru.MruError(st, "device status after decode timing")
    # the same steps captured once in a CUDA graph and replayed: the device
    # time per step without the host's per-call cost
    graph_ms, graph_err = None, None
    try:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                cap = torch.cuda.current_stream().cuda_stream
                for t in range(args.warmup, total):
                    src, dst = state[t % 2], state[(t + 1) % 2]
                    rc = mru.scan_fused(p, x_steps[t].data_ptr(), src.data_ptr(), None, dst.data_ptr(), None,
                                        ws.data_ptr(), ws.numel(), cap)
                    if rc != mru.OK:
                        raise mru.MruError(rc, "mru_scan_fused (graph capture)")
        stream.wait_stream(side)
        g.replay()
        torch.cuda.synchronize()
        ranks.barrier()
        ev0.record(stream)
        g.replay()
        ev1.record(stream)
        ev1.synchronize()
        graph_ms = ranks.max(ev0.elapsed_time(ev1) / args.steps)
        del g
    except (RuntimeError, mru.MruError) as exc:       # capture refused: report the eager figure only
        graph_err = str(exc).splitlines()[0][:200]
        ranks.max(0.0)
    if ranks.printer:
        units = w.B * w.H
        print(json.dumps({
            "metric": "MRU decode token·heads/s (one token per (b,h) sequence per step, from S0), 1×B200",
            "direction": "decode", "value": aggregate_rate(ranks.world, units, ms), "unit": UNIT,
            "n_gpus": ranks.world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "us_per_step": ms * 1e3,
            "graph": ({"us_per_step": graph_ms * 1e3, "value": aggregate_rate(ranks.world, units, graph_ms)}
                      if graph_ms else {"unavailable": graph_err}),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic (seeded N(0,1) embeddings)",
            "config": dict(workload_config(wd, mru.chosen_chunk(p, wd.readout)), sequences=units),
            "clocks": clocks.summary(), "gpu_launches": mru.launch_count(p) * args.steps,
            "kernels": mru.kernel_names(p)}), flush=True)
    ranks.close()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(gen.WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the per_workload entries (the other configurations the metric is quoted on)")
    ap.add_argument("--backward", action="store_true", help="time mru_scan_backward instead (not the default)")
    ap.add_argument("--decode", action="store_true",
                    help="time single-token decode steps from S0 instead (not the default)")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="run the workload with this sequence length instead of its own (small cases for "
                         "profiler captures; the workload's name gets the suffix _l<L>)")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)      # at least 3 untimed warm-up steps, always
    w = gen.WORKLOADS[args.workload]
    if args.seq_len > 0:
        import dataclasses
        w = dataclasses.replace(w, L=args.seq_len, name=f"{w.name}_l{args.seq_len}")
    if args.impl == "reference":
        return run_reference(args, w)
    if args.backward:
        return run_backward(args, w)
    if args.decode:
        return run_decode(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
