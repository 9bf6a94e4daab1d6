#!/usr/bin/env python
"""Benchmark of the IQ8R rotated W8A8 linear (libiq8r) on B200.

A step is one pass of the whole hot path over one batch: rotate + int8
quantise the activations, then the int8 linear with its fused scale
epilogue. For M <= 8 that is one launch (iq8r_linear_bf16: the GEMV rotates
and quantises x itself); above, iq8r_rotate_quant_act then the tcgen05
tensor-core GEMM (iq8r_linear). The default workload is the decode GEMV
(M=1, K=5120, N=17408, trunk format), reported in HBM GB/s, with a
"prefill" object (M=8192, int8 TOPS) in the same line; --config picks
another workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config decode]
    python bench.py --impl reference ...   # the CPU oracle, same metric

Timing: inputs resident in HBM; several weight copies are rotated so that
the bytes touched between two uses of a copy exceed 3x L2 (or one copy when
a step alone moves more than that); the K steps replay CUDA graphs on one
stream, bracketed by a barrier and synchronize; per-kernel durations come
from CUDA events recorded inside the same graphs. Multi-GPU runs are
independent replicas (one process per GPU, no data-path collective): the
whole-job value is the units all ranks processed over the slowest rank's
time.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "IQ8R W8A8 linear: decode HBM GB/s and prefill int8 TOPS vs B200 peak"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
INT8_OVER_BF16 = 2.0  # nominal dense ratio (4.5 POPS int8 / 2.25 PFLOP/s bf16)

# workloads reported beside the decode line by default
SUB_CONFIGS = ("prefill", "verify16", "lm_head1", "lm_head8")

CONFIGS = {
    # name: (m, k, n, fmt, default steps)
    "pr1": (4, 512, 256, "g256", 2000),
    "decode": (1, 5120, 17408, "g256", 20000),
    "verify8": (8, 17408, 5120, "g256", 5000),
    "verify16": (16, 17408, 5120, "g256", 2000),
    "verify128": (128, 17408, 5120, "g256", 500),
    "prefill": (8192, 5120, 17408, "g256", 20),
    "decode_g128": (1, 5120, 17408, "g128", 20000),
    "prefill_g128": (8192, 5120, 17408, "g128", 20),
    # the drafter's codebook format at the trunk's shape (the pages give no
    # drafter sizes)
    "draft_cb4": (1, 5120, 17408, "cb4", 20000),
    "lm_head1": (1, 5120, 151936, "g128", 2000),
    "lm_head8": (8, 5120, 151936, "g128", 1000),
}


# ------------------------------------------------------------------ bytes

def act_bytes(m, k):
    """Rotate-quantise: bf16 in, int8 codes and one fp32 scale per token out."""
    return 2 * m * k + m * k + 4 * m


def linear_bytes(m, k, n, fmt):
    """Weights (codes + scales), int8 activations + scales in, bf16 out."""
    if fmt == "g256":
        w = n * k + n * (k // 256) + 2 * n
    elif fmt == "cb4":
        w = n * k // 2 + 2 * n * (k // 128)
    else:
        w = n * k + 2 * n * (k // 128)
    return w + m * k + 4 * m + 2 * m * n


def fused_bytes(m, k, n, fmt):
    """One-launch layer: bf16 activations in, weights, bf16 out."""
    return linear_bytes(m, k, n, fmt) - m * k - 4 * m + 2 * m * k


# token rows of a large output (prefill) compared with the oracle
CHECK_ROWS = 16

# iq8r_linear_bf16 is one launch (activation quantiser fused into the GEMV)
# for M <= 2 and for M <= 8 with M * K <= 16384; iq8r_linear picks the GEMV
# for M <= 2 (both as documented in include/iq8r.h)
FUSE_MAX_M, FUSE_MAX_ELEMS, GEMV_MAX_M = 8, 16384, 2


def one_launch(m, k, fmt="g256"):
    if fmt == "cb4":  # the codebook format has no fused quantiser: two launches
        return False
    return m <= GEMV_MAX_M or (m <= FUSE_MAX_M and m * k <= FUSE_MAX_ELEMS)


def step_bytes(m, k, n, fmt, fused=None):
    """Algorithmic bytes of one step: the fused layer (one launch), else the
    activation kernel plus the linear."""
    if fused is None:
        fused = one_launch(m, k, fmt)
    if fused:
        return fused_bytes(m, k, n, fmt)
    return act_bytes(m, k) + linear_bytes(m, k, n, fmt)


def graph_kernel_nodes(g):
    """Kernel nodes in a captured torch CUDA graph (None if it cannot be
    inspected)."""
    if g is None:
        return 0
    try:
        from cuda.bindings import runtime as rt
        h = rt.cudaGraph_t(init_value=g.raw_cuda_graph())
        err, _, num = rt.cudaGraphGetNodes(h, 0)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        err, nodes, num = rt.cudaGraphGetNodes(h, num)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        kinds = [rt.cudaGraphNodeGetType(nd) for nd in nodes[:num]]
        return sum(1 for e, t in kinds if e == rt.cudaError_t.cudaSuccess
                   and t == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel)
    except Exception:
        return None


def max_over_ranks(ms, world, device):
    """The slowest rank's time: every rank takes the same all-reduce (MAX),
    so the job's throughput is all ranks' work over this time."""
    if world <= 1:
        return ms
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_value(units_per_rank, world, ms_max):
    """Whole-job throughput: the units all ranks processed per second of the
    slowest rank."""
    return world * units_per_rank / (ms_max * 1e-3)


def is_hbm_bound(m, k, n, fmt, fused=None):
    """The step's bound: HBM below the ridge point (int8 ops per algorithmic
    byte at which the int8 tensor peak and the HBM peak take equal time),
    the tensor cores above it. Decode and verify steps are HBM-bound and are
    reported in GB/s; prefill is tensor-bound and reported in int8 TOPS."""
    if fused is None:
        fused = one_launch(m, k, fmt)
    hbm, bf16_tf, _ = peaks()
    lin_b = fused_bytes(m, k, n, fmt) if fused else linear_bytes(m, k, n, fmt)
    return 2.0 * m * n * k / lin_b < bf16_tf * INT8_OVER_BF16 * 1e12 / (hbm * 1e9)


# ------------------------------------------------------------------ peaks

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def sustained_bf16():
    """The measured bf16 rate of a seconds-long loop under the power cap."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"])
    except Exception:
        return 1400.0


def kernel_source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "quantised_fwht128_act_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload, files):
    """DRAM bytes per launch from a committed ncu summary, if the kernel's
    sources are unchanged since it was taken; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d[kernel][workload]
        if e.get("source_hash") != kernel_source_hash(files):
            return None
        return int(e["dram_bytes_per_launch"])
    except Exception:
        return None


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples (every 100 ms) while the benchmark runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.idx)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        def num(s):
            try:
                return float(s)
            except ValueError:
                return None

        inside = [p for t, p in self.samples if t0 <= t <= t1]
        window = "timed region"
        if not inside:
            inside = [p for _, p in self.samples]
            window = "whole run (the timed region was shorter than one sample)"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "window": "no nvidia-smi"}
        sm = [num(p[1]) for p in inside if num(p[1]) is not None]
        smax = [num(p[2]) for p in inside if num(p[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for p in inside for i in range(4) if p[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(inside), "window": window}


# ------------------------------------------------------------- workload

_PACKED = {}


def make_inputs(cfg_name, m_override=None):
    """Host inputs: x copies (bf16 bits) and the packed weight (host packer).
    The packed weight is kept for workloads that draw the same weight (same
    seed and shape: verify8/16/128, lm_head1/8)."""
    import quantised_fwht128_act_b200 as iq8r
    from iq8r_inputs import WORKLOADS, gen_workload
    m, k, n, fmt, _ = CONFIGS[cfg_name]
    m = m_override or m
    wl = WORKLOADS.get(cfg_name, WORKLOADS["decode"])
    x0, w = gen_workload(wl, m=m, n=n, k=k)
    key = (wl.seed, wl.w_outlier_frac, n, k, fmt)
    if key not in _PACKED:
        _PACKED.clear()
        _PACKED[key] = iq8r.iq8r_pack(w, fmt, True)
    del w
    return x0, _PACKED[key], wl


def run_ours(args, rank, world, local_rank):
    import torch
    import quantised_fwht128_act_b200 as iq8r
    from iq8r_inputs import f32_to_bf16_bits, gen_act

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    m, k, n, fmt, _ = CONFIGS[args.config]
    m = getattr(args, "m", None) or m
    K, W = args.steps, args.warmup
    x0, (codes, sub, scale), wl = make_inputs(args.config, m)

    # rotating copies so that consecutive uses of one copy are > 3x L2 apart
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    footprint = step_bytes(m, k, n, fmt)
    R = 1 if footprint > 3 * l2 else int(math.ceil(3 * l2 / footprint)) + 1
    weights = []
    base = iq8r.IQ8RWeight.from_packed(codes, sub, scale, fmt, True, device=dev)
    weights.append(base)
    for _ in range(R - 1):
        weights.append(iq8r.IQ8RWeight(base.fmt, base.rotated, base.n, base.k, base.codes.clone(),
                                       None if base.sub_scale is None else base.sub_scale.clone(),
                                       base.scale.clone()))
    rng = np.random.default_rng(1000 + rank)
    xs_host = [x0] + [f32_to_bf16_bits(gen_act(rng, m, k, wl.x_outliers, wl.x_outlier_mult)) for _ in range(R - 1)]
    x_dev = [torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16) for x in xs_host]
    xq = [torch.empty((m, k), dtype=torch.int8, device=dev) for _ in range(R)]
    xsc = [torch.empty((m,), dtype=torch.float32, device=dev) for _ in range(R)]
    y = [torch.empty((m, n), dtype=torch.bfloat16, device=dev) for _ in range(R)]
    path = {"auto": iq8r.IQ8R_PATH_AUTO, "gemv": iq8r.IQ8R_PATH_GEMV, "tc": iq8r.IQ8R_PATH_TC}[args.path]
    # the GEMV rotates and quantises x itself (not for the codebook format)
    fused = one_launch(m, k, fmt) and args.path == "auto"

    def linear(r):
        iq8r.iq8r_linear_ex(xq[r], xsc[r], weights[r], y[r], path=path)

    def step(j):
        r = j % R
        if fused:
            iq8r.iq8r_linear_bf16(x_dev[r], weights[r], y[r])
        else:
            iq8r.iq8r_rotate_quant_act(x_dev[r], True, xq[r], xsc[r])
            linear(r)

    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for j in range(max(W, 1)):
            step(j)
    stream.synchronize()
    iq8r.iq8r_get_device_error(stream)

    # graphs: a main chunk of C steps (a multiple of R) and a tail, captured
    # bare, so consecutive kernels keep their programmatic (overlapping)
    # dependency, as a caller's stream would: the timed region replays these.
    # A step of two kernels is also captured once with external events
    # around each kernel (an event between two kernels removes their
    # overlap), replayed outside the timed region for the per-kernel times.
    C = min(K, max(R, (512 // R) * R))
    n_main, tail = divmod(K, C)

    def capture(nsteps, offset, with_events=False):
        try:
            g = torch.cuda.CUDAGraph(keep_graph=True)  # kept so its kernel nodes can be counted
        except TypeError:
            g = torch.cuda.CUDAGraph()
        evs = None if not with_events else [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)]
                                            for _ in range(nsteps)]
        with torch.cuda.graph(g, stream=stream):
            for j in range(nsteps):
                r = (offset + j) % R
                if fused:
                    iq8r.iq8r_linear_bf16(x_dev[r], weights[r], y[r])
                    continue
                if with_events:
                    evs[j][0].record()
                iq8r.iq8r_rotate_quant_act(x_dev[r], True, xq[r], xsc[r])
                if with_events:
                    evs[j][1].record()
                linear(r)
                if with_events:
                    evs[j][2].record()
        g.instantiate()
        return g, evs

    g_main, _ = capture(C, 0) if n_main else (None, None)
    g_tail, _ = capture(tail, 0) if tail else (None, None)
    g_ev, evs_ev = (None, None) if fused else capture(min(K, C), 0, with_events=True)
    # this library's kernel launches inside the timed region: the kernel
    # nodes of each captured graph times its replays
    counts = [graph_kernel_nodes(g) for g in (g_main, g_tail)]
    gpu_launches = (None if any(c is None for c, g in zip(counts, (g_main, g_tail)) if g is not None)
                    else n_main * (counts[0] or 0) + (counts[1] or 0))
    # one untimed replay of each graph (upload, first-touch), which also
    # sizes how many times the timed region is taken
    est0 = torch.cuda.Event(enable_timing=True)
    est1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        est0.record()
        for g in (g_main, g_tail):
            if g is not None:
                for _ in range(n_main if g is g_main else 1):
                    g.replay()
        est1.record()
    stream.synchronize()
    region_est_ms = est0.elapsed_time(est1)

    # The timed region: the K steps, bracketed by a barrier and a synchronize,
    # taken `reps` times back to back (the same count on every rank); the
    # line reports the median region. A short region (K = 20 decode steps
    # is under half a millisecond) is otherwise dominated by one start-up.
    reps = timed_reps(region_est_ms, tensor_bound=not is_hbm_bound(m, k, n, fmt, fused))
    if world > 1:  # every rank takes the region the same number of times
        t = torch.tensor([reps], dtype=torch.int64, device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        reps = int(t.item())
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    regions, act_ms, lin_ms = [], [], []
    t_start_wall = time.time()
    for _ in range(reps):
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            start.record()
            for _ in range(n_main):
                g_main.replay()
            if g_tail is not None:
                g_tail.replay()
            end.record()
        stream.synchronize()
        torch.cuda.synchronize()
        regions.append(max_over_ranks(start.elapsed_time(end), world, dev))
        if fused:
            lin_ms.append(regions[-1] / K)
    t_end_wall = time.time()
    if world > 1:
        torch.distributed.barrier()
    time.sleep(0.25)
    sampler.stop()
    iq8r.iq8r_get_device_error(stream)
    if fused:
        act_ms = [0.0]
    else:
        # per-kernel durations, each kernel on its own (outside the timed region)
        for _ in range(3):
            with torch.cuda.stream(stream):
                g_ev.replay()
            stream.synchronize()
            act_ms.append(float(np.mean([e[0].elapsed_time(e[1]) for e in evs_ev])))
            lin_ms.append(float(np.mean([e[1].elapsed_time(e[2]) for e in evs_ev])))
    elapsed_ms = float(np.median(regions))
    del g_main, g_tail, g_ev

    # end to end through the public API: every step is one call of
    # iq8r_linear_bf16_host, which queues the pinned H2D copy of x, the layer
    # and the D2H copy of y on the stream (eager launches, no graph)
    e2e = None
    if not args.no_e2e:
        xh = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in xs_host]
        yh = [torch.empty((m, n), dtype=torch.bfloat16).pin_memory() for _ in range(R)]
        xin = [torch.empty((m, k), dtype=torch.bfloat16, device=dev) for _ in range(R)]
        sh = stream.cuda_stream
        stage = [(None, None) if fused else (xq[r], xsc[r]) for r in range(R)]

        def e2e_step(j):
            r = j % R
            iq8r.iq8r_linear_bf16_host(xh[r], weights[r], xin[r], y[r], yh[r], stage[r][0], stage[r][1], sh)

        Ke = K
        for j in range(max(W, 3)):
            e2e_step(j)
        stream.synchronize()
        e_regions = []
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        for _ in range(reps):
            if world > 1:
                torch.distributed.barrier()
            torch.cuda.synchronize()
            with torch.cuda.stream(stream):
                s0.record()
                for j in range(Ke):
                    e2e_step(j)
                s1.record()
            stream.synchronize()
            e_regions.append(max_over_ranks(s0.elapsed_time(s1), world, dev))
        e_ms = float(np.median(e_regions))
        e_hbm = is_hbm_bound(m, k, n, fmt, fused)
        e_val = (job_value(step_bytes(m, k, n, fmt, fused) * Ke, world, e_ms) / 1e9 if e_hbm
                 else job_value(2.0 * m * n * k * Ke, world, e_ms) / 1e12)
        e2e = {"value": e_val, "unit": "GB/s" if e_hbm else "TOPS",
               "h2d_bytes_per_step": 2 * m * k, "d2h_bytes_per_step": 2 * m * n, "steps": Ke,
               "ms_per_step": e_ms / Ke,
               "how": ("one iq8r_linear_bf16_host call a step (pinned host x in, pinned host y out, both copies "
                       f"and the layer queued on one stream), eager; the K-step region timed {reps} times, "
                       "median reported")}

    hbm, bf16_tf, peak_src = peaks()
    lin_avg_ms = float(np.median(lin_ms))
    act_avg_ms = float(np.median(act_ms))
    lin_b = fused_bytes(m, k, n, fmt) if fused else linear_bytes(m, k, n, fmt)
    ops = 2.0 * m * n * k
    peak_i8 = bf16_tf * INT8_OVER_BF16
    # the kernel's bound: HBM below the ridge point (int8 ops per byte at
    # which the tensor peak and the HBM peak take equal time), tensor above
    hbm_bound = is_hbm_bound(m, k, n, fmt, fused)
    on_tc = args.path == "tc" or (args.path == "auto" and not fused and m > GEMV_MAX_M)
    on_tc = on_tc and fmt != "cb4"  # the codebook format has its own GEMV only
    # one or two tokens stream through the register-load GEMV, more (when
    # forced onto the GEMV) through the shared-memory-stage one
    reg = m <= 2
    kname = ("cb4_gemv_kernel" if fmt == "cb4" else
             "gemm_tc_kernel (tcgen05 kind::i8)" if on_tc else
             ("gemv_reg_kernel" if reg else "gemv_kernel") + (" (fused act, one launch per step)" if fused else ""))
    kfiles = (["cb4_gemv.cuh", "iq8r_device.cuh"] if fmt == "cb4" else
              ["gemm_tc.cuh", "iq8r_device.cuh"] if on_tc else
              (["gemv_reg.cuh"] if reg else []) + ["gemv.cuh", "act_quant.cuh", "iq8r_device.cuh"])
    ktraffic = recorded_traffic(kname.split(" ")[0], args.config, kfiles)
    if hbm_bound:
        achieved = lin_b / (lin_avg_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": kname, "achieved": achieved,
                "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "peak_source": f"{peak_src} HBM copy (MEASURED_PEAKS.json hbm_gbs)"
                if peak_src == "measured" else "fallback 6.65 TB/s",
                "traffic": ktraffic,
                "algorithmic_bytes_per_launch": lin_b, "avg_launch_ms": lin_avg_ms,
                "int8_tops": ops / (lin_avg_ms * 1e-3) / 1e12}
    else:
        # a dense int8 contraction on the tensor cores: its roofline is the int8
        # tensor peak, the measured bf16 peak times the nominal int8/bf16 ratio;
        # the burst figure for a short timed region, the sustained one when the
        # clock record shows the power cap during it
        achieved_t = ops / (lin_avg_ms * 1e-3) / 1e12
        ck = sampler.summary(t_start_wall, t_end_wall)
        capped = ("sw_power_cap" in (ck.get("reasons") or []) and ck.get("sm_mhz") is not None
                  and ck.get("sm_max_mhz") is not None and ck["sm_mhz"] < ck["sm_max_mhz"])
        bf16_use = sustained_bf16() if capped else bf16_tf
        peak_i8 = bf16_use * INT8_OVER_BF16
        roof = {"bound": "tensor", "kernel": kname, "achieved": achieved_t,
                "peak": peak_i8, "unit": "TOPS", "frac": achieved_t / peak_i8,
                "peak_source": (f"{peak_src} cuBLAS bf16 {bf16_use:.1f} TFLOP/s (MEASURED_PEAKS.json "
                                f"{'bf16_tflops_sustained: the power cap held the median clock below its maximum' if capped else 'bf16_tflops'}) "
                                f"x {INT8_OVER_BF16:g} (nominal dense int8/bf16)"),
                # both measured denominators, whichever the line's frac uses
                "frac_of_burst": achieved_t / (bf16_tf * INT8_OVER_BF16),
                "frac_of_sustained": achieved_t / (sustained_bf16() * INT8_OVER_BF16),
                "frac_of_datasheet_4500": achieved_t / 4500.0,
                "hbm_gbs": lin_b / (lin_avg_ms * 1e-3) / 1e9,
                "traffic": ktraffic,
                "algorithmic_ops_per_launch": ops, "algorithmic_bytes_per_launch": lin_b,
                "avg_launch_ms": lin_avg_ms}
    if not fused:
        roof["act_kernel"] = {"avg_launch_ms": act_avg_ms, "bytes": act_bytes(m, k),
                              "achieved_gbs": act_bytes(m, k) / (act_avg_ms * 1e-3) / 1e9,
                              "frac_of_hbm": act_bytes(m, k) / (act_avg_ms * 1e-3) / 1e9 / hbm}

    value = job_value(step_bytes(m, k, n, fmt, fused) * K, world, elapsed_ms) / 1e9
    unit = "GB/s"
    if not hbm_bound:  # tensor-bound (prefill) steps are reported in int8 TOPS
        value = job_value(ops * K, world, elapsed_ms) / 1e12
        unit = "TOPS"
    clocks = sampler.summary(t_start_wall, t_end_wall)
    out = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": elapsed_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8", "data": "synthetic",
        "config": workload_config(args.config, m),
        "method": {"step": "iq8r_linear_bf16 (one launch)" if fused else "iq8r_rotate_quant_act + iq8r_linear",
                   "bytes_per_step": step_bytes(m, k, n, fmt, fused), "path": args.path,
                   "l2": f"{R} rotating weight/input copies ({R * footprint / 1e6:.0f} MB > 3x L2)" if R > 1
                   else "a step moves more than 3x L2",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "timing": (("CUDA graphs of the K launches (programmatic dependent launch); events around "
                               "the timed region, average launch = region / K") if fused else
                              ("CUDA graphs of the K steps, kernels back to back (programmatic dependent launch); "
                               "per-kernel times from a copy of the graph with events around each kernel, "
                               "replayed outside the timed region"))
                             + f"; the K-step region timed {reps} times back to back, median reported"},
        "roofline": roof,
        "clocks": clocks,
        "gpu_launches": gpu_launches,
        "e2e": e2e,
        "cpu_baseline": None,
    }
    # for the oracle leg (outside the timed region): the first input copy,
    # the packed weight and the layer's output for them, on the host
    out["_check"] = {"config": args.config, "x": xs_host[0], "packed": (codes, sub, scale),
                     "y": y[0].view(torch.int16).cpu().numpy().view(np.uint16) if m * n <= (1 << 24) else
                     y[0][:CHECK_ROWS].view(torch.int16).cpu().numpy().view(np.uint16)}
    return out


def workload_config(name, m=None):
    """The workload as both arms name it: shape, format and rotation only."""
    m0, k, n, fmt, _ = CONFIGS[name]
    return {"workload": name, "m": m or m0, "k": k, "n": n, "format": fmt, "rotated": True}


def timed_reps(region_ms, tensor_bound=False):
    """How many times the K-step region is timed back to back: at least 3,
    and enough to span about 0.4 s (several clock samples) for a
    memory-bound step. A tensor-bound step (prefill) keeps to 3 regions
    unless one region already exceeds 0.1 s: a longer run at full tensor
    rate meets the power cap, and the line then says so and uses the
    sustained peak."""
    if tensor_bound:
        return 3
    return int(min(2000, max(3, math.ceil(400.0 / max(region_ms, 1e-3)))))


def run_rescore(args, rank, world, local_rank):
    """Candidate rescoring (iq8r_rescore): args.rescore weight rows a token,
    drawn at random over the whole weight, on the workload's weight and
    tokens. One launch a step; the activation codes are computed once."""
    import torch
    import quantised_fwht128_act_b200 as iq8r

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    m, k, n, fmt, _ = CONFIGS[args.config]
    m = getattr(args, "m", None) or m
    C, K, W = args.rescore, args.steps, args.warmup
    x0, (codes, sub, scale), wl = make_inputs(args.config, m)
    weight = iq8r.IQ8RWeight.from_packed(codes, sub, scale, fmt, True, device=dev)
    xd = torch.from_numpy(x0.view(np.int16)).to(dev).view(torch.bfloat16)
    xq, xs = iq8r.iq8r_rotate_quant_act(xd, True)
    R = 8
    g = torch.Generator(device="cpu").manual_seed(77 + rank)
    cands = [torch.randint(0, n, (m, C), generator=g, dtype=torch.int32).to(dev) for _ in range(R)]
    outs = [torch.empty((m, C), dtype=torch.bfloat16, device=dev) for _ in range(R)]
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for j in range(W):
            iq8r.iq8r_rescore(xq, xs, weight, cands[j % R], outs[j % R])
    stream.synchronize()
    iq8r.iq8r_get_device_error(stream)
    try:
        graph = torch.cuda.CUDAGraph(keep_graph=True)
    except TypeError:
        graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for j in range(K):
            iq8r.iq8r_rescore(xq, xs, weight, cands[j % R], outs[j % R])
    graph.instantiate()
    with torch.cuda.stream(stream):
        graph.replay()
    stream.synchronize()
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0w = time.time()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record()
        graph.replay()
        end.record()
    stream.synchronize()
    t1w = time.time()
    sampler.stop()
    iq8r.iq8r_get_device_error(stream)
    ms = max_over_ranks(start.elapsed_time(end), world, dev)
    row = k + (k // 256 + 2 if fmt == "g256" else 2 * (k // 128))
    step_b = m * C * row + m * k + 4 * m + 4 * m * C + 2 * m * C
    hbm, _, peak_src = peaks()
    avg = ms / K
    value = job_value(step_b * K, world, ms) / 1e9
    launches = graph_kernel_nodes(graph)
    del graph
    return {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": avg, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8", "data": "synthetic",
        "config": {"workload": f"{args.config} rescoring", "m": m, "k": k, "n": n, "format": fmt, "rotated": True,
                   "candidates_per_token": C, "step": "iq8r_rescore (one launch)", "bytes_per_step": step_b,
                   "l2": "candidate rows drawn at random over the whole weight", "parallelism": "single GPU"
                   if world == 1 else f"replicas x{world}",
                   "timing": "one CUDA graph of the K launches; events around the replay"},
        "roofline": {"bound": "hbm", "kernel": "rescore_kernel", "achieved": value / world, "peak": hbm,
                     "unit": "GB/s", "frac": value / world / hbm,
                     "peak_source": f"{peak_src} HBM copy (MEASURED_PEAKS.json hbm_gbs)", "traffic": None,
                     "algorithmic_bytes_per_launch": step_b, "avg_launch_ms": avg},
        "clocks": sampler.summary(t0w, t1w),
        "gpu_launches": None if launches is None else launches * 1,
        "e2e": None,
        "cpu_baseline": None,
    }


# ------------------------------------------------------------ CPU oracle

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def run_oracle(cfg_name, budget_s, steps=None):
    """Time the oracle (as it stands) on a bounded sample of the workload.

    A sample step is the oracle's act_quant over all M tokens plus its
    linear over a slice of the N weight rows, sized to the budget. Returns
    (value, unit, sample description, steps, s/step), the value in the
    workload's own unit: GB/s of algorithmic bytes for HBM-bound workloads,
    int8 TOPS (2 M N K per step) for tensor-bound ones.
    """
    import oracle
    from iq8r_inputs import WORKLOADS, gen_workload
    m, k, n, fmt, _ = CONFIGS[cfg_name]
    wl = WORKLOADS.get(cfg_name, WORKLOADS["decode"])
    m_s = min(m, 64)
    n_probe = min(n, 256)
    x, w = gen_workload(wl, m=m_s, n=n_probe, k=k)
    packed = oracle.pack(w, fmt, True) if fmt != "cb4" else (oracle.pack_cb4(w, True)[0], None, oracle.pack_cb4(w, True)[1])
    t = time.perf_counter()
    q, a = oracle.act_quant(x)
    oracle.linear(q, a, fmt, *packed, rotated=True)
    probe = time.perf_counter() - t
    per_row = probe / n_probe
    if steps is None:
        n_s = int(min(n, max(8, budget_s / 5 / max(per_row, 1e-9))))
        reps = max(1, int(budget_s / max(per_row * n_s, 1e-9)))
    else:
        n_s = int(min(n, max(8, budget_s / steps / max(per_row, 1e-9))))
        reps = steps
    x, w = gen_workload(wl, m=m_s, n=n_s, k=k)
    packed = oracle.pack(w, fmt, True) if fmt != "cb4" else (oracle.pack_cb4(w, True)[0], None, oracle.pack_cb4(w, True)[1])
    del w
    t = time.perf_counter()
    for _ in range(reps):
        q, a = oracle.act_quant(x)
        oracle.linear(q, a, fmt, *packed, rotated=True)
    dt = time.perf_counter() - t
    if is_hbm_bound(m, k, n, fmt):
        b = step_bytes(m_s, k, n_s, fmt, fused=one_launch(m, k, fmt))
        value, unit, what = b * reps / dt / 1e9, "GB/s", "algorithmic bytes"
    else:
        value, unit, what = 2.0 * m_s * n_s * k * reps / dt / 1e12, "TOPS", "int8 ops (2 M N K)"
    sample = (f"{reps} oracle steps of act_quant over {m_s} tokens + linear over {n_s} of {n} weight rows "
              f"(K={k}, {fmt}); value = {what} of that slice per second")
    return value, unit, sample, reps, dt / reps


def oracle_check(chk):
    """Part of the CPU-baseline leg: the layer's output on the bench's own
    first input copy and weight against the oracle. Reports the literal
    max |y - y64| / RMS(y64), the share of outputs equal to the oracle's bf16
    result, and whether every output is within the tolerance reading
    |y - y64| <= 1e-2 RMS(y64) + half a bf16 ulp (a bf16 output cannot meet
    1e-2 of RMS alone: its own rounding is up to 2^-8 of |y|). A large output
    is checked on its first CHECK_ROWS token rows."""
    import oracle
    _, _, _, fmt, _ = CONFIGS[chk["config"]]
    y = np.asarray(chk["y"], np.uint16)
    x = chk["x"][:y.shape[0]]
    q, a = oracle.act_quant(x)
    codes, sub, scale = chk["packed"]
    y64 = oracle.linear(q, a, fmt, codes, sub, scale, rotated=True)
    ref = oracle.linear_bf16(y64)
    yg = (y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    rms = float(np.sqrt(np.mean(y64 ** 2)))
    err = np.abs(yg - y64)
    e = np.floor(np.log2(np.maximum(np.abs(y64), 2.0 ** -126)))
    half_ulp = np.ldexp(1.0, (e - 8).astype(int))
    return {"rows_checked": int(y.shape[0]), "outputs": int(y.size),
            "max_err_over_rms": float(err.max() / rms) if rms > 0 else float(err.max()),
            "bit_equal_frac": float(np.mean(y.reshape(-1) == ref.reshape(-1))),
            "within_tolerance": bool(np.all(err <= 1e-2 * rms + half_ulp)),
            "tolerance": "|y - y64| <= 1e-2 RMS(y64) + ulp_bf16(y64)/2 per output"}


def run_reference(args, rank, world):
    m, k, n, fmt, _ = CONFIGS[args.config]
    K, W = args.steps, args.warmup
    budget = float(os.environ.get("IQ8R_REF_BUDGET_S", "60"))
    # warm-up: W oracle steps of the same slice, untimed, within the budget
    run_oracle(args.config, min(budget / 10, 5.0), steps=max(1, min(W, 3)))
    value, unit, sample, reps, s_per = run_oracle(args.config, budget, steps=K)
    cores = blas_threads()
    return {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": s_per * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8", "data": "synthetic", "impl": "reference",
        "config": workload_config(args.config),
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------ main

def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", choices=sorted(CONFIGS), default="decode")
    ap.add_argument("--path", choices=["auto", "gemv", "tc"], default="auto",
                    help="force the linear's kernel (auto: the library's choice)")
    ap.add_argument("--m", type=int, default=None, help="override the workload's token count M")
    ap.add_argument("--rescore", type=int, default=0,
                    help="time candidate rescoring (this many weight rows a token) instead of the layer")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="same as --no-sub")
    ap.add_argument("--no-sub", action="store_true",
                    help="decode run only: skip the prefill, verify16 and lm_head sub-objects")
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    args = ap.parse_args(argv)
    steps_given = args.steps is not None
    if args.steps is None:
        args.steps = CONFIGS[args.config][4]
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        out = run_reference(args, rank, world)
        print(json.dumps(out), flush=True)
        return 0

    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        if args.rescore:
            out = run_rescore(args, rank, world, local_rank)
            if rank == 0:
                print(json.dumps(out), flush=True)
            return 0
        out = run_ours(args, rank, world, local_rank)
        subs = {}
        if args.config == "decode" and not (args.no_prefill or args.no_sub):
            # the metric's second half (prefill int8 TOPS on the tensor cores)
            # and the other workloads of the pages' model: a speculative
            # verify block and the lm_head at one and eight tokens; the same
            # K and timing rules, each its own roofline and end-to-end number
            import torch
            for name in SUB_CONFIGS:
                pargs = argparse.Namespace(**vars(args))
                pargs.config = name
                pargs.m = None
                if not steps_given:
                    pargs.steps = CONFIGS[name][4]
                pargs.warmup = min(args.warmup, 5)
                torch.cuda.empty_cache()
                sub = run_ours(pargs, rank, world, local_rank)
                subs[name] = sub
                out[name] = {k_: sub[k_] for k_ in ("value", "unit", "steps", "warmup", "ms_per_step", "config",
                                                      "method", "roofline", "gpu_launches", "clocks", "e2e")}
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            # the CPU-baseline leg: the oracle timed on a bounded sample of each
            # workload, and the layer's outputs checked against it
            value, unit, sample, reps, _ = run_oracle(args.config, args.cpu_budget_s)
            out["cpu_baseline"] = {"value": value, "unit": unit, "cores": blas_threads(), "kind": "oracle",
                                   "sample": sample}
            out["parity"] = oracle_check(out["_check"])
            for name, sub in subs.items():
                v, u, smp, _, _ = run_oracle(name, min(args.cpu_budget_s, 6.0))
                out[name]["cpu_baseline"] = {"value": v, "unit": u, "cores": blas_threads(), "kind": "oracle",
                                             "sample": smp}
                out[name]["parity"] = oracle_check(sub["_check"])
        out.pop("_check", None)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
