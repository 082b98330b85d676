#!/usr/bin/env python3
"""Benchmark of the activation-sparse int4 GEMV on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--path auto|list|thresh|mask] [--sparsity 0.5] [--no-ffn]

Workload: the Llama-3-8B FFN down_proj GEMV (K = 14336 input channels,
N = 4096 outputs), int4 asymmetric weights in groups of 128 along K with fp16
scale and zero, batch 1, x = SiLU(g) * u with g, u ~ N(0, 1) in bf16, and a
magnitude threshold at the 50th percentile of |x| (50% activation sparsity).
All inputs are synthetic and seeded; weights ~ N(0, 0.02).

A step is one pass of the hot path over one activation vector: gathering the
active channels and the sparse GEMV over them (select + gemv, or the fused
threshold-GEMV). Steps cycle through R copies of the packed weights whose total
size is more than 4x the L2 cache, so every step reads its weights from HBM.
The K timed steps run as CUDA-graph replays on one stream, timed with CUDA
events, bracketed by a barrier and a device synchronize. Every graph of the
timed region is replayed once before the warm-up (its first replay uploads
it), and a bounded device delay ahead of the start event keeps the host's
submission of the graphs outside the event window. The kernel-alone and
call-alone timings (roofline kernel, dense GEMV, select, each entry point,
the sparsity sweep, the ReGLU FFN, the tiny case) use a fixed 2000 launches
whatever --steps is.

Further legs on the same protocol: the sparsity sweep 0/30/50/70/90% of the
same GEMV with a roofline fraction per row, the ReGLU FFN (natural ReLU zeros
and an 88% stand-in), the tiny case (latency), the Llama-3-8B FFN and decode
layer, the Qwen3-32B FFN at batch 1..16 and the 2:4 weight-sparse GEMV
(--no-ffn skips them all).

Metric: HBM GB/s on active bytes (and us per GEMV). Active bytes per GEMV are
the weight bytes of the active channels (a*N/2), the scale/zero bytes of the
groups they touch (4*N per group), the index and activation bytes (6*a) and
the output (2*N).

Multi-GPU: the path does not shard across GPUs in this workload (one GEMV per
step); `--gpus N` under torchrun runs N independent replicas, each timing its
own steps, and reports the units of all ranks over the slowest rank's time
(weak scaling).

`--impl reference` times the CPU oracle (the plain fp64 C restatement under
oracle/, its OpenMP form over every host core) on a bounded sample of the
same workload; it is a deliberately slow reference arm, not a target. The
cpu_baseline key of the main line times the oracle twice: on one thread and
on every core.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from activation_sparse_quantized_b200 import sgq                     # noqa: E402
from activation_sparse_quantized_b200 import workloads as wl         # noqa: E402

METRIC = "µs/GEMV and HBM GB/s on active bytes, int4 sparse GEMV, 8B FFN, 50% sparsity"
UNIT = "GB/s"
WORKLOAD = ("Llama-3-8B FFN down_proj GEMV: K=14336, N=4096, int4 asymmetric group 128 "
            "(fp16 scale+zero), x = SiLU(g)*u bf16, batch 1, 50% magnitude sparsity")


# ---------------------------------------------------------------------------
# process / device plumbing
# ---------------------------------------------------------------------------

class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.dev = "cuda"

    def init(self, backend="nccl"):
        # reductions run on the device for NCCL, on the host for gloo
        self.dev = "cuda" if backend == "nccl" else "cpu"
        if self.world > 1:
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", self.local)
                                    if backend == "nccl" else None)
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=self.dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def sum(self, v: float) -> float:
        if not self.pg:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=self.dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.SUM)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock"}

    def __init__(self, index: int, period_s: float = 0.005):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - NVML may be missing on the host
            self.err = str(e)

    def _sample(self):
        self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
        try:
            r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            r = self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.reasons |= int(r)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._sample()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._thread.join()
            self._sample()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def read_peak_gbs(nbytes: int = 2 << 30, reps: int = 10) -> float:
    """A read-only streaming peak measured here: device time of a reduction
    over a buffer much larger than L2 (torch's fp32 sum: one read of the
    buffer, no conversion pass), the best of several runs."""
    buf = torch.ones(nbytes // 4, dtype=torch.float32, device="cuda")
    torch.sum(buf)
    torch.cuda.synchronize()
    best = 1e30
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch.sum(buf)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    del buf
    torch.cuda.empty_cache()
    return nbytes / (best * 1e-3) / 1e9


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "activation_sparse_quantized_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, src_hash: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)[kernel]
        if d.get("source_hash") == src_hash:
            return float(d["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ---------------------------------------------------------------------------
# the workload
# ---------------------------------------------------------------------------

N, K, GROUP = wl.LLAMA8B_DOWN["N"], wl.LLAMA8B_DOWN["K"], wl.LLAMA8B_DOWN["group"]


def active_bytes(a: int, touched_groups: int, n: int = N, B: int = 1) -> int:
    return a * n // 2 + touched_groups * n * 4 + a * (4 + 2 * B) + 2 * B * n


class Replica:
    """R packed weight copies (> 4x L2 in total) and R activation vectors."""

    def __init__(self, sparsity: float, seed: int = 0):
        self.sparsity = sparsity
        W = wl.weight(N, K, seed)
        qw0, sz0 = sgq.alloc_packed(N, K, GROUP)
        sgq.sgq_pack(W.cuda(), N, K, GROUP, qw0, sz0)
        l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
        per = qw0.numel() + sz0.numel() * 4
        self.R = max(2, int(math.ceil(4 * l2 / per)) + 1)
        self.qw = [qw0] + [qw0.clone() for _ in range(self.R - 1)]
        self.sz = [sz0] + [sz0.clone() for _ in range(self.R - 1)]
        self.bytes_resident = self.R * per
        self.l2 = l2
        self.x_host = [wl.x_silu_gated(1, K, 1000 + r) for r in range(self.R)]
        self.x = [x.cuda() for x in self.x_host]
        self.y = torch.empty(1, N, dtype=torch.bfloat16, device="cuda")
        self.ws = sgq.alloc_workspace(N, K, 1)
        self.sidx, self.scnt = sgq.alloc_select(K)
        self.smask = sgq.alloc_mask(K)
        self.yacc = torch.zeros(1, N, dtype=torch.float32, device="cuda")
        self.idx = [sgq.alloc_select(K) for _ in range(self.R)]
        self.mask = [sgq.alloc_mask(K) for _ in range(self.R)]
        self.set_sparsity(sparsity)

    def set_sparsity(self, sparsity: float):
        """Thresholds for `sparsity` on every copy's x, with the per-copy index
        lists and bitmasks (for timing the GEMV kernel alone) and the active
        byte counts."""
        self.sparsity = sparsity
        self.t = [wl.percentile_threshold(x[0], sparsity) for x in self.x_host]
        self.cnt, self.abytes, self.active, self.groups = [], [], [], []
        for r in range(self.R):
            idx, cnt = self.idx[r]
            sgq.sgq_select(self.x[r], 1, K, [self.t[r]], idx, cnt)
            a = int(cnt.item())
            groups = int(np.unique(idx[:a].cpu().numpy() // GROUP).size)
            self.cnt.append(cnt)
            self.active.append(a)
            self.groups.append(groups)
            self.abytes.append(active_bytes(a, groups))
            sgq.sgq_select_mask(self.x[r], 1, K, [self.t[r]], self.mask[r])
        torch.cuda.synchronize()

    def kernel_bytes(self, which: str) -> float:
        """Algorithmic bytes per launch of one timed form, mean over the copies:
        the fused threshold forms read all of x (2K) and no index list; the
        accumulating forms write fp32 y (4N)."""
        a = float(np.mean(self.active))
        base = float(np.mean(self.abytes))
        if which in ("thresh", "thresh_acc"):
            base = base - 6 * a + 2 * K
        if which == "mask":
            base = base - 4 * a + K // 8
        if which in ("thresh_acc", "gemv_acc"):
            base = base + 2 * N
        return base

    def step(self, r: int, path: str):
        """One pass of the hot path on copy r (kernels launched: 2 or 1)."""
        if path == "list":
            sgq.sgq_select(self.x[r], 1, K, [self.t[r]], self.sidx, self.scnt)
            sgq.sgq_gemv(self.qw[r], self.sz[r], N, K, GROUP, self.x[r], 1, self.sidx,
                         self.scnt, self.y, None, self.ws)
        elif path == "mask":
            sgq.sgq_select_mask(self.x[r], 1, K, [self.t[r]], self.smask)
            sgq.sgq_gemv_mask(self.qw[r], self.sz[r], N, K, GROUP, self.x[r], 1, self.smask,
                              self.y, None, self.ws)
        else:
            sgq.sgq_gemv_thresh(self.qw[r], self.sz[r], N, K, GROUP, self.x[r], self.t[r],
                                self.y, None, self.ws)

    def kernel_only(self, r: int, which: str):
        if which == "gemv":
            sgq.sgq_gemv(self.qw[r], self.sz[r], N, K, GROUP, self.x[r], 1, self.idx[r][0],
                         self.cnt[r], self.y, None, self.ws)
        elif which == "dense":
            sgq.sgq_gemv_dense(self.qw[r], self.sz[r], N, K, GROUP, self.x[r], 1, self.y, None,
                               self.ws)
        elif which == "thresh":
            sgq.sgq_gemv_thresh(self.qw[r], self.sz[r], N, K, GROUP, self.x[r], self.t[r],
                                self.y, None, self.ws)
        elif which == "select":
            sgq.sgq_select(self.x[r], 1, K, [self.t[r]], self.sidx, self.scnt)
        elif which == "mask":
            sgq.sgq_gemv_mask(self.qw[r], self.sz[r], N, K, GROUP, self.x[r], 1, self.mask[r],
                              self.y, None, self.ws)
        elif which == "select_mask":
            sgq.sgq_select_mask(self.x[r], 1, K, [self.t[r]], self.smask)
        elif which == "thresh_acc":   # the GEMV kernel alone (adds into fp32, no epilogue)
            sgq.sgq_gemv_thresh_acc(self.qw[r], self.sz[r], N, K, GROUP, self.x[r], self.t[r],
                                    self.yacc)
        elif which == "gemv_acc":
            sgq.sgq_gemv_acc(self.qw[r], self.sz[r], N, K, GROUP, self.x[r], 1, self.idx[r][0],
                             self.cnt[r], self.yacc)


class GraphRunner:
    """Runs exactly n calls of fn(i) as replays of captured CUDA graphs."""

    def __init__(self, fn, period: int, stream):
        self.fn, self.period, self.stream = fn, period, stream
        self.graphs = {}

    def _graph(self, length: int, offset: int):
        key = (length, offset)
        if key not in self.graphs:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(self.stream):
                with torch.cuda.graph(g, stream=self.stream):
                    for i in range(length):
                        self.fn(offset + i)
            self.graphs[key] = g
        return self.graphs[key]

    def _parts(self, n: int):
        full, rem = divmod(n, self.period)
        return [self.period] * full + ([rem] if rem else [])

    def prepare(self, n: int):
        for length in set(self._parts(n)):
            self._graph(length, 0)

    def prewarm(self, n: int):
        """Replays, once and untimed, every graph that run(n) replays (the
        first replay of a graph uploads it to the device)."""
        with torch.cuda.stream(self.stream):
            for length in set(self._parts(n)):
                self._graph(length, 0).replay()
        torch.cuda.synchronize()

    def run(self, n: int):
        for length in self._parts(n):
            self._graph(length, 0).replay()


# Launches for every kernel-alone or call-alone timing, whatever --steps is.
FIXED_LAUNCHES = 2000


def device_delay(stream, us: float = 300.0):
    """A bounded spin (torch's own sleep kernel, a fixed number of clock
    cycles) enqueued before a start event, so that the host's submission of
    the timed graphs happens while the device is still busy and is not inside
    the event window."""
    with torch.cuda.stream(stream):
        torch.cuda._sleep(int(us * 2.0e3))   # cycles at ~2 GHz


def whole_job(bytes_local: float, ms_local: float, dist: Dist):
    """Whole-job GB/s: the bytes of every rank over the slowest rank's device
    time (replicas: weak scaling). Returns (GB/s, max ms)."""
    ms = dist.max(ms_local)
    return dist.sum(bytes_local) / (ms * 1e-3) / 1e9, ms


def time_calls(fn, n: int, period: int, dist: Dist | None = None, warm: int = 3):
    """Device time (ms) of exactly n calls of fn(i), via CUDA graphs: every
    graph replayed once untimed, warm-up calls, then a bounded device delay
    ahead of the start event and the n calls."""
    stream = torch.cuda.Stream()
    gr = GraphRunner(fn, period, stream)
    gr.prepare(n)
    gr.prepare(max(warm, 1))
    gr.prewarm(n)
    with torch.cuda.stream(stream):
        gr.run(max(warm, 1))
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    device_delay(stream)
    with torch.cuda.stream(stream):
        e0.record(stream)
        gr.run(n)
        e1.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    return e0.elapsed_time(e1)


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------

def run_ours(args, dist: Dist):
    torch.cuda.set_device(dist.local)
    sgq.load()
    rep = Replica(args.sparsity)
    R = rep.R
    path = args.path
    if path == "auto":
        path = "thresh"
    # kernels per step: every GEMV call is the GEMV kernel plus its split-K
    # epilogue kernel; the list and mask paths add their select kernel
    kernels_per_step = {"thresh": 2, "list": 3, "mask": 3}[path]
    period = R * max(1, 64 // R)

    # warm-up (untimed) then exactly K timed steps
    # (every graph of the timed region is replayed once before the warm-up,
    # so the timed replays are not the graphs' first; a bounded device delay
    # ahead of the start event keeps the host's submission out of the window)
    stream = torch.cuda.Stream()
    runner = GraphRunner(lambda i: rep.step(i % R, path), period, stream)
    runner.prepare(args.steps)
    runner.prepare(args.warmup)
    runner.prewarm(args.steps)
    with torch.cuda.stream(stream):
        runner.run(args.warmup)
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dist.local) as clk:
        device_delay(stream)
        with torch.cuda.stream(stream):
            e0.record(stream)
            runner.run(args.steps)
            e1.record(stream)
        torch.cuda.synchronize()
    dist.barrier()
    ms_local = e0.elapsed_time(e1)
    value, ms = whole_job(sum(rep.abytes[i % R] for i in range(args.steps)), ms_local, dist)
    us_per_gemv = ms * 1e3 / args.steps

    # the dominant kernel alone, same rotation, for the roofline: the GEMV
    # kernel through its accumulating form (the same kernel adding its
    # split-K sums into an fp32 buffer, so no epilogue kernel follows it);
    # the mask path has no accumulating form and is timed as the whole call
    dom = {"thresh": "thresh_acc", "list": "gemv_acc", "mask": "mask"}[path]
    nk = FIXED_LAUNCHES
    kms = time_calls(lambda i: rep.kernel_only(i % R, dom), nk, period)
    k_us = kms * 1e3 / nk
    k_bytes = rep.kernel_bytes(dom)
    peak, peak_kind = measured_peak()
    rpk = read_peak_gbs()
    achieved = k_bytes / (k_us * 1e-6) / 1e9
    src = source_hash("gemv.cu", "gemv_rows.cuh", "sgq_device.cuh")
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                "traffic": profiled_traffic({"thresh_acc": "thresh", "gemv_acc": "gemv"}.get(dom, dom), src),
                "kernel": {"thresh_acc": "gemv_kernel<ROWS_THRESH> (select fused)",
                           "gemv_acc": "gemv_kernel<ROWS_LIST>",
                           "mask": "sgq_gemv_mask call"}[dom],
                "kernel_us": round(k_us, 3), "algorithmic_bytes": int(k_bytes),
                "frac_of_8TBps": round(achieved / 8000.0, 4),
                "read_peak_gbs": round(rpk, 1), "frac_of_read_peak": round(achieved / rpk, 4),
                "timed": ("the GEMV kernel alone on its stream, launched through the "
                          "accumulating entry point (sgq_gemv_thresh_acc / sgq_gemv_acc): the "
                          "same kernel, its split-K sums added into fp32 y, no epilogue kernel; "
                          "the bf16 call with its epilogue kernel is call_us")
                         if dom != "mask" else "the sgq_gemv_mask call (GEMV + epilogue kernel)"}

    # comparison points on the same rotation: dense int4 GEMV, select alone
    nc = FIXED_LAUNCHES
    dense_ms = time_calls(lambda i: rep.kernel_only(i % R, "dense"), nc, period)
    sel_ms = time_calls(lambda i: rep.kernel_only(i % R, "select"), nc, period)
    cmp_us = {}
    for name in ("gemv", "thresh", "mask", "select_mask", "thresh_acc"):
        cms = time_calls(lambda i: rep.kernel_only(i % R, name), nc, period)
        cmp_us[name] = round(cms * 1e3 / nc, 3)

    e2e = run_e2e(rep, path, 500, args.warmup, dist)
    sweep = None if args.no_ffn else run_sweep(rep)
    rep.set_sparsity(args.sparsity)
    reglu = None if args.no_ffn else run_reglu()
    tiny = None if args.no_ffn else run_tiny()
    layer = None if args.no_ffn else run_layer()
    batch = None if args.no_ffn else run_batch()
    nm = None if args.no_ffn else run_nm()

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded; weights N(0,0.02), x = SiLU(g)*u)",
        "config": {"workload": WORKLOAD, "K": K, "N": N, "group": GROUP, "batch": 1,
                   "sparsity": args.sparsity, "active_channels": int(np.mean(rep.active)),
                   "path": {"list": "select+gemv", "mask": "select_mask+gemv_mask",
                            "thresh": "gemv_thresh (select fused)"}[path],
                   "l2": f"inputs larger than L2: {R} rotating weight copies, "
                         f"{rep.bytes_resident / 1e6:.0f} MB vs L2 {rep.l2 / 1e6:.0f} MB",
                   "parallelism": f"replicas x{dist.world}" if dist.world > 1 else "single GPU"},
        "us_per_gemv": round(us_per_gemv, 3),
        "active_bytes_per_gemv": int(np.mean(rep.abytes)),
        "roofline": roofline,
        "dense_int4_gemv_us": round(dense_ms * 1e3 / nc, 3),
        "select_us": round(sel_ms * 1e3 / nc, 3),
        "call_us": {"gemv_list": cmp_us["gemv"], "gemv_thresh": cmp_us["thresh"],
                    "gemv_mask": cmp_us["mask"], "select_mask": cmp_us["select_mask"],
                    "gemv_thresh_acc": cmp_us["thresh_acc"],
                    "note": "one C-ABI call each on the same rotation; a GEMV call is the "
                            "GEMV kernel plus its split-K epilogue kernel"},
        "e2e": e2e,
        "gpu_launches": args.steps * kernels_per_step,
        "clocks": clk.summary(),
    }
    if layer is not None:
        line.update(layer)
    if batch is not None:
        line["batch_ffn"] = batch
    if nm is not None:
        line["nm_2of4"] = nm
    if sweep is not None:
        line["sparsity_sweep"] = sweep
    if reglu is not None:
        line["reglu_ffn"] = reglu
    if tiny is not None:
        line["tiny"] = tiny
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    return line


def run_e2e(rep: Replica, path: str, steps: int, warmup: int, dist: Dist):
    """The same metric through the public API with host buffers: every step
    copies x from pinned host memory, runs the path, reads y back into pinned
    host memory and waits for it. Each step is one CUDA graph holding those
    three operations (captured once per weight copy), so a step costs one
    graph launch and one synchronize; the same steps issued as separate calls
    are reported as us_per_gemv_eager."""
    xs = [x.pin_memory() for x in rep.x_host]
    yh = torch.empty(1, N, dtype=torch.bfloat16).pin_memory()
    yh_bits = yh.view(torch.int16).numpy()      # the same pinned bytes, read from the host
    xd = torch.empty(1, K, dtype=torch.bfloat16, device="cuda")
    R = rep.R

    def body(r):
        xd.copy_(xs[r], non_blocking=True)
        if path == "list":
            sgq.sgq_select(xd, 1, K, [rep.t[r]], rep.sidx, rep.scnt)
            sgq.sgq_gemv(rep.qw[r], rep.sz[r], N, K, GROUP, xd, 1, rep.sidx, rep.scnt, rep.y,
                         None, rep.ws)
        elif path == "mask":
            sgq.sgq_select_mask(xd, 1, K, [rep.t[r]], rep.smask)
            sgq.sgq_gemv_mask(rep.qw[r], rep.sz[r], N, K, GROUP, xd, 1, rep.smask, rep.y, None,
                              rep.ws)
        else:
            sgq.sgq_gemv_thresh(rep.qw[r], rep.sz[r], N, K, GROUP, xd, rep.t[r], rep.y, None,
                                rep.ws)
        yh.copy_(rep.y, non_blocking=True)

    stream = torch.cuda.Stream()
    graphs = []
    with torch.cuda.stream(stream):
        for r in range(R):
            body(r)                      # warm the path on this stream before capture
        stream.synchronize()
        for r in range(R):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                body(r)
            graphs.append(g)
    torch.cuda.synchronize()

    def step_graph(i):
        graphs[i % R].replay()
        stream.synchronize()
        return int(yh_bits[0, 0])

    def step_eager(i):
        body(i % R)
        stream.synchronize()
        return int(yh_bits[0, 0])

    def timed(fn):
        with torch.cuda.stream(stream):
            for i in range(max(3, warmup)):
                fn(i)
        torch.cuda.synchronize()
        dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(steps):
                fn(i)
            e1.record(stream)
        torch.cuda.synchronize()
        return dist.max(e0.elapsed_time(e1))

    ms = timed(step_graph)
    ms_eager = timed(step_eager)
    b = dist.sum(sum(rep.abytes[i % R] for i in range(steps)))
    return {"value": round(b / (ms * 1e-3) / 1e9, 1), "unit": UNIT,
            "us_per_gemv": round(ms * 1e3 / steps, 3), "steps": steps,
            "us_per_gemv_eager": round(ms_eager * 1e3 / steps, 3),
            "h2d_bytes_per_step": 2 * K, "d2h_bytes_per_step": 2 * N}


# ---------------------------------------------------------------------------
# Layer leg: the decode FFN and the whole decode layer around the GEMV
# (secondary numbers; attention and norms are not part of the path)
# ---------------------------------------------------------------------------

class LayerReplica:
    """R copies of one Llama-3-8B decode layer's projections, int4 g128:
    q 4096->4096, k/v 4096->1024, o 4096->4096, gate/up 4096->14336,
    down 14336->4096. Fused forms: [W_q; W_k; W_v] stacked (one GEMV, y = q|k|v)
    and [W_g; W_u] stacked (one GEMV with the SiLU-GLU epilogue); unfused forms:
    every projection separately plus sgq_glu. R x bytes > 4x L2.

    Inputs: x ~ N(0, 1) into q/k/v and gate/up, an independent N(0, 1) stand-in
    for the attention output into o, each with a 50% threshold; the down
    projection skips |h| <= t_h, t_h the 50th percentile of |h| (found once
    per copy, untimed)."""

    def __init__(self, sparsity: float = 0.5, seed: int = 7):
        L = wl.LLAMA8B_LAYER
        self.H, self.I, self.g = L["gate"]["K"], L["gate"]["N"], L["gate"]["group"]
        self.nq, self.nkv = L["q"]["N"], L["k"]["N"]
        H, I, g = self.H, self.I, self.g
        W = {n: wl.weight(L[n]["N"], L[n]["K"], seed + j) for j, n in enumerate(L)}
        base = {
            "qkv": self._pack(torch.cat([W["q"], W["k"], W["v"]], 0)),
            "q": self._pack(W["q"]), "k": self._pack(W["k"]), "v": self._pack(W["v"]),
            "o": self._pack(W["o"]),
            "gu": self._pack(torch.cat([W["gate"], W["up"]], 0)),
            "gate": self._pack(W["gate"]), "up": self._pack(W["up"]), "down": self._pack(W["down"]),
        }
        per = sum(a.numel() * a.element_size() for t in base.values() for a in t)
        l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
        self.R = max(2, int(math.ceil(4 * l2 / per)) + 1)
        self.w = [base] + [{k: tuple(a.clone() for a in t) for k, t in base.items()}
                           for _ in range(self.R - 1)]
        self.bytes_resident = self.R * per
        xa = [wl.x_gaussian(1, H, 2000 + r) for r in range(self.R)]
        xo = [wl.x_gaussian(1, H, 3000 + r) for r in range(self.R)]
        self.xa, self.xo = [x.cuda() for x in xa], [x.cuda() for x in xo]
        self.ta = [wl.percentile_threshold(x[0], sparsity) for x in xa]
        self.to = [wl.percentile_threshold(x[0], sparsity) for x in xo]
        dev = lambda n: torch.empty(1, n, dtype=torch.bfloat16, device="cuda")
        self.h, self.yg, self.yu = dev(I), dev(I), dev(I)
        self.y, self.yqkv, self.yo = dev(H), dev(self.nq + 2 * self.nkv), dev(H)
        self.yq, self.yk, self.yv = dev(self.nq), dev(self.nkv), dev(self.nkv)
        self.ws = sgq.alloc_workspace(2 * I, max(H, I), 1)     # largest B*N of any call
        self.wsf = sgq.alloc_ffn_workspace(H, I)
        idx, cnt = sgq.alloc_select(max(H, I))
        self.th, self.ffn_bytes, self.layer_bytes = [], [], []

        def active(x, t, K):
            sgq.sgq_select(x, 1, K, [t], idx, cnt)
            a = int(cnt.item())
            return a, int(np.unique(idx[:a].cpu().numpy() // g).size)

        for r in range(self.R):
            self.gate_up(r)
            self.th.append(wl.percentile_threshold(self.h[0].cpu(), sparsity))
            a_in, g_in = active(self.xa[r], self.ta[r], H)
            a_o, g_o = active(self.xo[r], self.to[r], H)
            a_h, g_h = active(self.h, self.th[r], I)
            nqkv = self.nq + 2 * self.nkv
            # active bytes: codes of the active channels, (s, z) of touched groups, x, y
            ffn = (a_in * I + g_in * 2 * I * 4 + 2 * H + 2 * I
                   + a_h * H // 2 + g_h * H * 4 + 2 * I + 2 * H)
            attn = (a_in * nqkv // 2 + g_in * nqkv * 4 + 2 * H + 2 * nqkv
                    + a_o * H // 2 + g_o * H * 4 + 2 * H + 2 * H)
            self.ffn_bytes.append(ffn)
            self.layer_bytes.append(ffn + attn)
        torch.cuda.synchronize()

    def _pack(self, W):
        N, K = W.shape
        qw, sz = sgq.alloc_packed(N, K, self.g)
        sgq.sgq_pack(W.cuda(), N, K, self.g, qw, sz)
        return qw, sz

    def _thresh(self, w, N, K, x, t, y):
        sgq.sgq_gemv_thresh(w[0], w[1], N, K, self.g, x, t, y, None, self.ws)

    def gate_up(self, r):
        qw, sz = self.w[r]["gu"]
        sgq.sgq_gemv_glu_thresh(qw, sz, self.I, self.H, self.g, self.xa[r], self.ta[r],
                                sgq.SGQ_ACT_SILU, self.h, None, self.ws)

    def ffn_fused(self, r):                      # 4 launches
        self.gate_up(r)
        self._thresh(self.w[r]["down"], self.H, self.I, self.h, self.th[r], self.y)

    def ffn_3k(self, r):                         # 3 launches: sgq_ffn
        w = self.w[r]
        sgq.sgq_ffn(w["gu"][0], w["gu"][1], w["down"][0], w["down"][1], self.H, self.I, self.g,
                    self.xa[r], self.ta[r], sgq.SGQ_ACT_SILU, self.th[r], self.y, None, None,
                    self.wsf)

    def ffn_unfused(self, r):                    # 7 launches
        w, H, I = self.w[r], self.H, self.I
        self._thresh(w["gate"], I, H, self.xa[r], self.ta[r], self.yg)
        self._thresh(w["up"], I, H, self.xa[r], self.ta[r], self.yu)
        sgq.sgq_glu(self.yg, self.yu, self.h, 1, I, sgq.SGQ_ACT_SILU)
        self._thresh(w["down"], H, I, self.h, self.th[r], self.y)

    def layer_fused(self, r):                    # 7 launches
        w, H = self.w[r], self.H
        self._thresh(w["qkv"], self.nq + 2 * self.nkv, H, self.xa[r], self.ta[r], self.yqkv)
        self._thresh(w["o"], H, H, self.xo[r], self.to[r], self.yo)
        self.ffn_3k(r)

    def layer_unfused(self, r):                  # 15 launches
        w, H = self.w[r], self.H
        for n, N, y in (("q", self.nq, self.yq), ("k", self.nkv, self.yk),
                        ("v", self.nkv, self.yv)):
            self._thresh(w[n], N, H, self.xa[r], self.ta[r], y)
        self._thresh(w["o"], H, H, self.xo[r], self.to[r], self.yo)
        self.ffn_unfused(r)


def run_layer(n_steps: int = 1000):
    """us per decode FFN and per decode layer (projections only), fused and
    unfused, on the rotation."""
    f = LayerReplica()
    R = f.R
    period = R * max(1, 32 // R)
    n = max(n_steps, 2 * period)
    us = {}
    for name in ("ffn_3k", "ffn_fused", "ffn_unfused", "layer_fused", "layer_unfused"):
        fn = getattr(f, name)
        us[name] = time_calls(lambda i: fn(i % R), n, period) * 1e3 / n
    fb, lb = float(np.mean(f.ffn_bytes)), float(np.mean(f.layer_bytes))
    return {
        "ffn": {"workload": "Llama-3-8B FFN decode, batch 1: gate/up 4096->14336 at 50% input "
                            "sparsity, SiLU, down 14336->4096 over the 50% largest |h|; int4 g128",
                "us_per_ffn_3_kernels": round(us["ffn_3k"], 3), "launches_3_kernels": 3,
                "us_per_ffn_fused": round(us["ffn_fused"], 3), "launches_fused": 4,
                "us_per_ffn_unfused": round(us["ffn_unfused"], 3), "launches_unfused": 7,
                "active_bytes_per_ffn": int(fb),
                "GBps_active_3_kernels": round(fb / (us["ffn_3k"] * 1e-6) / 1e9, 1),
                "tokens_per_s_equiv_ffn_only_32_layers": round(1e6 / (32 * us["ffn_3k"]), 1)},
        "layer": {"workload": "Llama-3-8B decode layer projections, batch 1: q/k/v (stacked), "
                              "o, then the FFN as sgq_ffn (gate/up stacked, h formed and selected "
                              "in the down projection); 50% sparsity per projection input; "
                              "attention and norms excluded",
                  "us_per_layer_fused": round(us["layer_fused"], 3), "launches_fused": 7,
                  "us_per_layer_unfused": round(us["layer_unfused"], 3), "launches_unfused": 15,
                  "active_bytes_per_layer": int(lb),
                  "fused_GBps_active": round(lb / (us["layer_fused"] * 1e-6) / 1e9, 1),
                  "tokens_per_s_equiv_32_layers_projections_only":
                      round(1e6 / (32 * us["layer_fused"]), 1)},
        "rotation": f"{R} copies, {f.bytes_resident / 1e6:.0f} MB",
    }


def run_sweep(rep: "Replica", sparsities=wl.SPARSITY_SWEEP):
    """The same down_proj GEMV over the sparsity sweep: per sparsity, the bf16
    call (fused threshold GEMV + epilogue kernel) and the GEMV kernel alone
    (accumulating form), each over FIXED_LAUNCHES launches on the rotation,
    with the kernel's roofline fraction on its algorithmic bytes."""
    peak, _ = measured_peak()
    R = rep.R
    period = R * max(1, 64 // R)
    rows = []
    for sp in sparsities:
        rep.set_sparsity(sp)
        n = FIXED_LAUNCHES
        call_us = time_calls(lambda i: rep.kernel_only(i % R, "thresh"), n, period) * 1e3 / n
        k_us = time_calls(lambda i: rep.kernel_only(i % R, "thresh_acc"), n, period) * 1e3 / n
        kb = rep.kernel_bytes("thresh_acc")
        cb = rep.kernel_bytes("thresh")
        rows.append({"sparsity": sp, "active_channels": int(np.mean(rep.active)),
                     "us_per_gemv": round(call_us, 3), "kernel_us": round(k_us, 3),
                     "algorithmic_bytes": int(kb),
                     "GBps_call": round(cb / (call_us * 1e-6) / 1e9, 1),
                     "GBps_kernel": round(kb / (k_us * 1e-6) / 1e9, 1),
                     "frac_kernel": round(kb / (k_us * 1e-6) / 1e9 / peak, 4),
                     "frac_kernel_of_8TBps": round(kb / (k_us * 1e-6) / 1e9 / 8000.0, 4)})
    return {"workload": "Llama-3-8B down_proj (K=14336, N=4096, int4 g128), x = SiLU(g)*u, "
                        "batch 1, magnitude threshold at each sparsity; fused select",
            "rows": rows, "launches_per_row": FIXED_LAUNCHES,
            "rotation": f"{R} copies, {rep.bytes_resident / 1e6:.0f} MB"}


class ReGluReplica:
    """R copies of a ReGLU FFN (hidden 4096, intermediate 11008, int4 g128):
    stacked [W_g; W_u] and W_d; R x bytes > 4x L2. x ~ N(0, 1) (dense: every
    channel of the gate/up input is read), h = ReLU(W_g x) * (W_u x) whose
    zeros the down projection skips (t = 0). Random weights leave about half
    of h zero; the stand-in h = ReLU(g - beta) * u with 88% zeros stands for a
    trained ReGLU model's ~90%."""

    def __init__(self, seed: int = 21):
        cfg = wl.REGLU_FFN
        self.H, self.I, self.g = cfg["hidden"], cfg["inter"], cfg["group"]
        H, I, g = self.H, self.I, self.g
        gu = self._pack(torch.cat([wl.weight(I, H, seed), wl.weight(I, H, seed + 1)], 0))
        down = self._pack(wl.weight(H, I, seed + 2))
        per = sum(a.numel() * a.element_size() for t in (gu, down) for a in t)
        l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
        self.R = max(2, int(math.ceil(4 * l2 / per)) + 1)
        self.gu = [gu] + [tuple(a.clone() for a in gu) for _ in range(self.R - 1)]
        self.down = [down] + [tuple(a.clone() for a in down) for _ in range(self.R - 1)]
        self.bytes_resident = self.R * per
        self.x = [wl.x_gaussian(1, H, 5000 + r).cuda() for r in range(self.R)]
        self.h88 = [wl.x_relu_shifted(1, I, 6000 + r).cuda() for r in range(self.R)]
        self.h = torch.empty(1, I, dtype=torch.bfloat16, device="cuda")
        self.hs = torch.empty(1, I, dtype=torch.bfloat16, device="cuda")
        self.y = torch.empty(1, H, dtype=torch.bfloat16, device="cuda")
        self.ws = sgq.alloc_workspace(2 * I, max(H, I), 1)
        self.wsf = sgq.alloc_ffn_workspace(H, I)
        idx, cnt = sgq.alloc_select(I)
        # gate/up (dense) bytes and down bytes at each h
        gub = 2 * I * H // 2 + (H // g) * 2 * I * 4 + 2 * H
        self.nat_down, self.s88_down, self.nat_frac, self.s88_frac = [], [], [], []
        for r in range(self.R):
            self.gate_up(r, self.h)
            for hv, out, fr in ((self.h, self.nat_down, self.nat_frac),
                                (self.h88[r], self.s88_down, self.s88_frac)):
                sgq.sgq_select(hv, 1, I, [0.0], idx, cnt)
                a = int(cnt.item())
                gr = int(np.unique(idx[:a].cpu().numpy() // g).size)
                out.append(a * H // 2 + gr * H * 4 + 2 * I + 2 * H)
                fr.append(1.0 - a / I)
        self.gu_bytes = gub
        torch.cuda.synchronize()

    def _pack(self, W):
        N, K = W.shape
        qw, sz = sgq.alloc_packed(N, K, self.g)
        sgq.sgq_pack(W.cuda(), N, K, self.g, qw, sz)
        return qw, sz

    def gate_up(self, r, h):
        qw, sz = self.gu[r]
        sgq.sgq_gemv_glu_dense(qw, sz, self.I, self.H, self.g, self.x[r], 1, sgq.SGQ_ACT_RELU,
                               h, None, self.ws)

    def ffn_natural(self, r):                    # 3 launches: sgq_ffn
        qg, sg = self.gu[r]
        qd, sd = self.down[r]
        sgq.sgq_ffn(qg, sg, qd, sd, self.H, self.I, self.g, self.x[r], -1.0, sgq.SGQ_ACT_RELU,
                    0.0, self.y, None, None, self.wsf)

    def ffn_standin(self, r):                    # 4 launches
        self.gate_up(r, self.hs)
        qd, sd = self.down[r]
        sgq.sgq_gemv_thresh(qd, sd, self.H, self.I, self.g, self.h88[r], 0.0, self.y, None,
                            self.ws)

    def down_only(self, r, h):
        qd, sd = self.down[r]
        sgq.sgq_gemv_thresh(qd, sd, self.H, self.I, self.g, h, 0.0, self.y, None, self.ws)


def run_reglu():
    """us per ReGLU FFN (natural ReLU zeros and the 88% stand-in) and per down
    projection alone, each over FIXED_LAUNCHES calls on the rotation."""
    f = ReGluReplica()
    R = f.R
    period = R * max(1, 32 // R)
    n = FIXED_LAUNCHES
    peak, _ = measured_peak()
    us = {"ffn_natural": time_calls(lambda i: f.ffn_natural(i % R), n, period) * 1e3 / n,
          "ffn_standin": time_calls(lambda i: f.ffn_standin(i % R), n, period) * 1e3 / n}
    # the down projection alone over the stand-in h (per copy) and over the
    # natural h of copy 0 (gate/up output, computed once)
    f.gate_up(0, f.h)
    us["down_natural"] = time_calls(lambda i: f.down_only(i % R, f.h), n, period) * 1e3 / n
    us["down_standin"] = time_calls(lambda i: f.down_only(i % R, f.h88[i % R]), n,
                                    period) * 1e3 / n
    nat = f.gu_bytes + float(np.mean(f.nat_down))
    s88 = f.gu_bytes + float(np.mean(f.s88_down))
    return {"workload": "ReGLU FFN decode, batch 1: hidden 4096, intermediate 11008, int4 "
                        "g128; x ~ N(0,1) dense into the stacked gate/up GEMV with the ReLU "
                        "GLU; down_proj over h's nonzeros (t = 0)",
            "h_zero_frac_natural": round(float(np.mean(f.nat_frac)), 3),
            "h_zero_frac_standin": round(float(np.mean(f.s88_frac)), 3),
            "us_per_ffn_natural": round(us["ffn_natural"], 3), "launches_natural": 3,
            "us_per_ffn_standin": round(us["ffn_standin"], 3), "launches_standin": 4,
            "active_bytes_natural": int(nat), "active_bytes_standin": int(s88),
            "GBps_natural": round(nat / (us["ffn_natural"] * 1e-6) / 1e9, 1),
            "GBps_standin": round(s88 / (us["ffn_standin"] * 1e-6) / 1e9, 1),
            "down_us_natural": round(us["down_natural"], 3),
            "down_us_standin": round(us["down_standin"], 3),
            "down_frac_standin": round(float(np.mean(f.s88_down)) /
                                       (us["down_standin"] * 1e-6) / 1e9 / peak, 4),
            "note": "natural: sgq_ffn (h formed and selected inside the down projection); "
                    "stand-in: the gate/up GLU GEMV, then the down GEMV over a synthetic h "
                    "with 88% zeros (h = ReLU(g - beta) * u, not the GLU's output)",
            "rotation": f"{R} copies, {f.bytes_resident / 1e6:.0f} MB"}


def run_tiny():
    """The tiny GEMV (K=256, N=512, g64, 50%): latency of one fused call (its
    48 KB of inputs stay in L2; correctness case, not a bandwidth case)."""
    shp = wl.TINY
    n_, k_, g_ = shp["N"], shp["K"], shp["group"]
    case = wl.gemv_case(n_, k_, g_, sparsity=0.5, seed=0)
    qw, sz = sgq.alloc_packed(n_, k_, g_)
    sgq.sgq_pack(case.W.cuda(), n_, k_, g_, qw, sz)
    x = case.x.cuda()
    y = torch.empty(1, n_, dtype=torch.bfloat16, device="cuda")
    ws = sgq.alloc_workspace(n_, k_, 1)
    t = case.t[0]
    n = FIXED_LAUNCHES
    us = time_calls(lambda i: sgq.sgq_gemv_thresh(qw, sz, n_, k_, g_, x, t, y, None, ws), n,
                    64) * 1e3 / n
    return {"workload": "tiny GEMV K=256, N=512, int4 g64, x ~ N(0,1), 50% sparsity, fused "
                        "select; inputs resident in L2 (latency only)",
            "us_per_gemv": round(us, 3), "launches": n}


class BatchFfnReplica:
    """R copies of one Qwen3-32B FFN (hidden 5120, intermediate 25600, int4
    g128): stacked [W_g; W_u] and W_d; R x bytes > 4x L2. At batch B, x has B
    rows of SiLU(g) * u, each with its own 50% threshold; gate/up and down read
    the union of the rows' active sets (index lists from sgq_select), the down
    projection over each row's 50% largest |h|."""

    def __init__(self, seed: int = 11):
        cfg = wl.QWEN32B_FFN
        self.H, self.I, self.g = cfg["hidden"], cfg["inter"], cfg["group"]
        H, I, g = self.H, self.I, self.g
        pk = lambda W: self._pack(W)
        gu = pk(torch.cat([wl.weight(I, H, seed), wl.weight(I, H, seed + 1)], 0))
        down = pk(wl.weight(H, I, seed + 2))
        per = sum(a.numel() * a.element_size() for t in (gu, down) for a in t)
        l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
        self.R = max(2, int(math.ceil(4 * l2 / per)) + 1)
        self.gu = [gu] + [tuple(a.clone() for a in gu) for _ in range(self.R - 1)]
        self.down = [down] + [tuple(a.clone() for a in down) for _ in range(self.R - 1)]
        self.bytes_resident = self.R * per
        self.ws = sgq.alloc_workspace(2 * I, H, sgq.SGQ_MAX_BATCH)
        self.idx_x, self.cnt_x = sgq.alloc_select(H)
        self.idx_h, self.cnt_h = sgq.alloc_select(I)

    def _pack(self, W):
        N, K = W.shape
        qw, sz = sgq.alloc_packed(N, K, self.g)
        sgq.sgq_pack(W.cuda(), N, K, self.g, qw, sz)
        return qw, sz

    def setup(self, B: int):
        H, I = self.H, self.I
        xh = [wl.x_silu_gated(B, H, 4000 + 17 * B + r) for r in range(self.R)]
        self.B = B
        self.x = [x.cuda() for x in xh]
        self.t = [[wl.percentile_threshold(x[b], 0.5) for b in range(B)] for x in xh]
        self.h = torch.empty(B, I, dtype=torch.bfloat16, device="cuda")
        self.y = torch.empty(B, H, dtype=torch.bfloat16, device="cuda")
        self.th, self.union_x, self.union_h = [], [], []
        for r in range(self.R):
            self.front(r)
            hc = self.h.cpu()
            self.th.append([wl.percentile_threshold(hc[b], 0.5) for b in range(B)])
            self.union_x.append(int(self.cnt_x.item()) / H)
            sgq.sgq_select(self.h, B, I, self.th[r], self.idx_h, self.cnt_h)
            self.union_h.append(int(self.cnt_h.item()) / I)
        torch.cuda.synchronize()

    def front(self, r):
        B, H, I, g = self.B, self.H, self.I, self.g
        sgq.sgq_select(self.x[r], B, H, self.t[r], self.idx_x, self.cnt_x)
        qw, sz = self.gu[r]
        sgq.sgq_gemv_glu(qw, sz, I, H, g, self.x[r], B, self.idx_x, self.cnt_x,
                         sgq.SGQ_ACT_SILU, self.h, None, self.ws)

    def ffn_fused(self, r):                      # 4 launches
        """The rows' union found inside each GEMV (sgq_gemv_glu_thresh_batch,
        sgq_gemv_thresh_batch): two GEMVs and their epilogue kernels."""
        B, H, I, g = self.B, self.H, self.I, self.g
        qw, sz = self.gu[r]
        sgq.sgq_gemv_glu_thresh_batch(qw, sz, I, H, g, self.x[r], B, self.t[r],
                                      sgq.SGQ_ACT_SILU, self.h, None, self.ws)
        qd, sd = self.down[r]
        sgq.sgq_gemv_thresh_batch(qd, sd, H, I, g, self.h, B, self.th[r], self.y, None, self.ws)

    def ffn(self, r):                            # 6 launches
        B, H, I, g = self.B, self.H, self.I, self.g
        self.front(r)
        sgq.sgq_select(self.h, B, I, self.th[r], self.idx_h, self.cnt_h)
        qd, sd = self.down[r]
        sgq.sgq_gemv(qd, sd, H, I, g, self.h, B, self.idx_h, self.cnt_h, self.y, None, self.ws)


def run_batch(batches=(1, 2, 4, 8, 16), n_steps: int = 64):
    """us per FFN at each batch size on the rotation (Qwen3-32B shapes)."""
    f = BatchFfnReplica()
    R = f.R
    out = []
    for B in batches:
        f.setup(B)
        n = max(n_steps, 2 * R)
        us6 = time_calls(lambda i: f.ffn(i % R), n, R) * 1e3 / n
        us = time_calls(lambda i: f.ffn_fused(i % R), n, R) * 1e3 / n
        ux, uh = float(np.mean(f.union_x)), float(np.mean(f.union_h))
        wbytes = ux * f.H * f.I + uh * f.I * f.H / 2    # codes of the union rows (gate+up, down)
        # algorithmic bytes of the FFN: codes and (scale, zero) of every group
        # the union rows touch (all of them at these densities), x, h and y
        G_in, G_h = f.H // f.g, f.I // f.g
        abytes = (wbytes + G_in * 2 * f.I * 4 + G_h * f.H * 4
                  + 2 * B * f.H + 2 * B * f.I * 2 + 2 * B * f.H)
        peak, _ = measured_peak()
        out.append({"batch": B, "us_per_ffn": round(us, 2), "launches": 4,
                    "us_per_ffn_select_kernels": round(us6, 2), "launches_select_kernels": 6,
                    "union_active_in": round(ux, 3),
                    "union_active_h": round(uh, 3),
                    "weight_code_GBps": round(wbytes / (us * 1e-6) / 1e9, 1),
                    "algorithmic_bytes": int(abytes),
                    "frac_of_measured_peak": round(abytes / (us * 1e-6) / 1e9 / peak, 4),
                    "tokens_per_s_equiv_ffn_only_64_layers": round(B * 1e6 / (64 * us), 1)})
    return {"workload": "Qwen3-32B FFN decode (hidden 5120, intermediate 25600, int4 g128, "
                        "SiLU): per-row 50% thresholds, union active sets found inside each GEMV "
                        "(sgq_gemv_glu_thresh_batch, sgq_gemv_thresh_batch: 4 launches); "
                        "us_per_ffn_select_kernels: the same with sgq_select before each GEMV "
                        "(6 launches)",
            "rows": out, "rotation": f"{R} copies, {f.bytes_resident / 1e6:.0f} MB"}


def run_nm(n_steps: int = 4000, sparsity: float = 0.5):
    """The 8B down_proj with 2:4 weight sparsity (sgq_pack_nm) composed with
    50% activation sparsity, fused threshold path, on its own rotation."""
    W = wl.weight(N, K, 0)
    qb, kb, sb = sgq.sgq_packed_sizes_nm(N, K, GROUP)
    qw0, kp0, sz0 = sgq.alloc_packed_nm(N, K, GROUP)
    sgq.sgq_pack_nm(W.cuda(), N, K, GROUP, qw0, kp0, sz0)
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    R = max(2, int(math.ceil(4 * l2 / (qb + kb + sb))) + 1)
    cp = [(qw0, kp0, sz0)] + [(qw0.clone(), kp0.clone(), sz0.clone()) for _ in range(R - 1)]
    xh = [wl.x_silu_gated(1, K, 1000 + r) for r in range(R)]
    x = [v.cuda() for v in xh]
    t = [wl.percentile_threshold(v[0], sparsity) for v in xh]
    y = torch.empty(1, N, dtype=torch.bfloat16, device="cuda")
    ws = sgq.alloc_workspace(N, K, 1)
    idx, cnt = sgq.alloc_select(K)
    ab = []
    for r in range(R):
        sgq.sgq_select(x[r], 1, K, [t[r]], idx, cnt)
        a = int(cnt.item())
        gr = int(np.unique(idx[:a].cpu().numpy() // GROUP).size)
        ab.append(a * N // 4 + gr * (N // 2) * 4 + gr * N // 8 + 2 * K + 2 * N)

    def call(i):
        r = i % R
        q, k_, s_ = cp[r]
        sgq.sgq_gemv_nm_thresh(q, k_, s_, N, K, GROUP, x[r], t[r], y, None, ws)

    period = R * max(1, 64 // R)
    n = max(n_steps, 2 * period)
    us = time_calls(call, n, period) * 1e3 / n
    b = float(np.mean(ab))
    return {"workload": "Llama-3-8B down_proj (K=14336, N=4096, g128) with static 2:4 weight "
                        "sparsity along the outputs (sgq_pack_nm) and 50% activation sparsity, "
                        "select fused; batch 1",
            "us_per_gemv": round(us, 3), "active_bytes_per_gemv": int(b),
            "GBps_active": round(b / (us * 1e-6) / 1e9, 1),
            "rotation": f"{R} copies, {R * (qb + kb + sb) / 1e6:.0f} MB"}


# ---------------------------------------------------------------------------
# CPU oracle timings (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------

class OracleSample:
    """The oracle's select + GEMV on the benchmark workload (setup untimed)."""

    def __init__(self, sparsity: float):
        import oracle
        self.o = oracle
        self.W = wl.weight(N, K, 0)
        self.x = wl.x_silu_gated(1, K, 1000)
        self.t = [wl.percentile_threshold(self.x[0], sparsity)]
        wb = self.W.view(torch.int16).numpy().view(np.uint16)
        self.q, self.s, self.z = oracle.quantize(wb, GROUP)
        self.xb = wl.bits(self.x)
        idx = oracle.select(self.xb, self.t)
        self.a = int(idx.size)
        self.groups = int(np.unique(idx // GROUP).size)

    def run(self, rows: np.ndarray, threads: int | None = None):
        """select + GEMV for the given outputs (on `threads` OpenMP threads, or
        the one-thread form); returns the active bytes covered."""
        idx = self.o.select(self.xb, self.t)
        self.o.gemv(self.q[rows], self.s[rows], self.z[rows], GROUP, self.xb, idx,
                    threads=threads)
        n = len(rows)
        return active_bytes(self.a, self.groups, n=n)


def host_cores() -> int:
    return len(os.sched_getaffinity(0))


def cpu_baseline(seconds: float):
    """The oracle's select + GEMV on the benchmark workload, timed twice on the
    host: the one-thread form, and the OpenMP form over every core of the
    affinity mask (each output keeps its summation order: same results). Each
    runs whole GEMVs for about `seconds` (at most 50)."""
    smp = OracleSample(0.5)
    rows = np.arange(N)
    cores = host_cores()

    def timed(threads):
        done, reps, t0 = 0, 0, time.perf_counter()
        while True:
            done += smp.run(rows, threads)
            reps += 1
            el = time.perf_counter() - t0
            if el >= seconds or reps >= 50:
                return done / el / 1e9, reps, el

    v1, r1, e1 = timed(None)
    vm, rm, em = timed(cores)
    return {"value": round(vm, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{rm} full GEMVs (select + fp64 GEMV, all {N} outputs) in {em:.1f} s "
                      f"on {cores} OpenMP threads (outputs shared out, sums unchanged)",
            "single_thread": {"value": round(v1, 4), "unit": UNIT, "cores": 1,
                              "sample": f"{r1} full GEMVs in {e1:.1f} s on one thread"}}


def run_reference(args, dist: Dist):
    """The reference arm: the CPU oracle as it stands (its OpenMP form on every
    core of the affinity mask), on a bounded sample of the workload per step
    (a slice of the outputs), K steps after W warm-up."""
    smp = OracleSample(args.sparsity)
    cores = host_cores()
    budget = 60.0 / max(args.steps + args.warmup, 1)
    t0 = time.perf_counter()
    smp.run(np.arange(8 * cores), cores)
    per_row = (time.perf_counter() - t0) / (8 * cores)
    nrows = int(max(1, min(N, budget / max(per_row, 1e-9))))
    rng = np.random.default_rng(0)
    for _ in range(args.warmup):
        smp.run(np.sort(rng.choice(N, nrows, replace=False)), cores)
    done = 0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        done += smp.run(np.sort(rng.choice(N, nrows, replace=False)), cores)
    el = time.perf_counter() - t0
    value = done / el / 1e9
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
            "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "K": K, "N": N, "group": GROUP, "batch": 1,
                       "sparsity": args.sparsity,
                       "path": f"CPU oracle: select + fp64 GEMV (plain C, OpenMP over the "
                               f"outputs, {cores} threads)"},
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": cores,
                             "kind": "oracle",
                             "sample": f"each step: {nrows} of {N} outputs of the GEMV"},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--path", choices=["auto", "list", "thresh", "mask"], default="auto")
    ap.add_argument("--sparsity", type=float, default=0.5)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-ffn", action="store_true",
                    help="skip the secondary FFN / decode-layer leg (fused vs unfused)")
    ap.add_argument("--profile-batch", type=int, default=0, metavar="B",
                    help="profiling aid: run only the Qwen3-32B FFN at batch B for --steps "
                         "FFNs and exit (prints one line of timing, no JSON contract line)")
    args = ap.parse_args(argv)
    if args.profile_batch:
        torch.cuda.set_device(0)
        f = BatchFfnReplica()
        f.setup(args.profile_batch)
        for i in range(max(3, args.warmup)):
            f.ffn(i % f.R)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for i in range(args.steps):
            f.ffn(i % f.R)
        torch.cuda.synchronize()
        print(f"Qwen3-32B FFN batch {args.profile_batch}: "
              f"{(time.perf_counter() - t0) * 1e6 / args.steps:.1f} us per FFN (host clock)")
        return 0
    if args.warmup < 3:
        args.warmup = 3
    dist = Dist()
    if dist.world != args.gpus and dist.world > 1:
        args.gpus = dist.world
    if args.impl == "reference":
        if dist.rank == 0:
            print(json.dumps(run_reference(args, dist)), flush=True)
        return 0
    dist.init("nccl")
    try:
        line = run_ours(args, dist)
        if dist.rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
