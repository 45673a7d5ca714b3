#!/usr/bin/env python
"""Benchmark of relative-position attention, forward + backward, on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = relpos_attn_fwd + relpos_attn_bwd of the whole workload (default:
Transformer-XL, causal, B=1, H=8, L=8192, d=64, bf16) on inputs already resident
in HBM.  The L2 cache (126 MB) is flushed by writing a 256 MB buffer before every
timed step (outside the timed interval); each step is timed with CUDA events on
the launching stream, and the reported time is the max over ranks.  With N > 1
(torchrun) every rank runs its own batch of the workload (weak scaling) and the
relative-table gradients, shared by all ranks, are summed with one NCCL
all-reduce, as in data-parallel training.

Prints one JSON line (rank 0).  ``--impl reference`` times the fp64 CPU oracle
(test infrastructure, the only reference there is) on a bounded sample of the
same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from attention_fwd_bwd_flashattention_b200 import binding as bd  # noqa: E402
from attention_fwd_bwd_flashattention_b200 import dist as rdist  # noqa: E402
from attention_fwd_bwd_flashattention_b200.inputs import ALIBI, DEBERTA, SHAW, T5, TXL, WORKLOADS, make_inputs  # noqa: E402

DEFAULT_WORKLOAD = "txl_causal_L8192_bf16"
METRIC = "fwd+bwd TFLOP/s and tokens/s at L=8192, % of B200 BF16 tensor peak"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}


# ----------------------------------------------------------------------------
# algorithmic FLOPs (distinct products the method must compute; recompute and
# window duplication are not credited)
# ----------------------------------------------------------------------------
def pairs_of(wl):
    """Unmasked (query, key) pairs of one head, summed over the batch: every query
    with the keys before its batch's key length (and not after it when causal); with a
    Transformer-XL memory of M keys, query i sees the M cached keys and i + 1 of the
    segment's."""
    if wl.mem_len:
        return wl.B * (wl.L * wl.mem_len + wl.L * (wl.L + 1) // 2)
    lens = wl.seqlens_k if wl.seqlens_k is not None else (wl.L,) * wl.B
    tot = 0
    for lk in lens:
        lk = max(0, min(wl.L, lk))
        tot += lk * (lk + 1) // 2 + (wl.L - lk) * lk if wl.causal else wl.L * lk
    return tot


def algo_flops(wl):
    U = 2.0 * wl.H * wl.d * pairs_of(wl)

    def R(rows):
        return 2.0 * wl.B * wl.H * wl.L * rows * wl.d

    if wl.mech in (T5, ALIBI):
        return 2 * U, 5 * U
    if wl.mech == SHAW:
        r = R(2 * wl.shaw_clip + 1)
        if wl.shaw_value:  # value side: Pe aV forward; dO aV^T and Pe^T dO backward
            return 2 * U + 2 * r, 5 * U + 5 * r
        return 2 * U + r, 5 * U + 3 * r
    if wl.mech == TXL:
        return 3 * U, 8 * U
    r = R(2 * wl.deberta_span)
    return 2 * U + 2 * r, 5 * U + 6 * r


def fa_flops(wl):
    pairs = pairs_of(wl)
    return 4.0 * pairs * wl.d * wl.H, 10.0 * pairs * wl.d * wl.H


def kernel_launches(wl, path):
    """Kernels this library launches per forward and per backward call (the dispatch of csrc/api.cu)."""
    t5 = 1 if wl.mech in (T5, ALIBI) else 0  # per-call per-offset bias preparation
    # bf16 runs on the tensor cores except Shaw's value-side table with c > 64
    tc = path != "simt" and wl.dtype == torch.bfloat16 and not (wl.mech == SHAW and wl.shaw_value and wl.shaw_clip > 64)
    wide = tc and wl.mech == SHAW and wl.shaw_clip > 64  # the Transformer-XL kernels over the clip-expanded table
    if wide:  # table expansion, relation prep, the forward kernel
        fwd = 3
    elif tc:  # tensor-core forward: relation prep (TXL, DeBERTa) + the forward kernel
        fwd = 1 + t5 + (1 if wl.mech in (TXL, DEBERTA) else 0)
    else:
        fwd = 1 + t5
    if tc and (wl.mech == TXL or wide):
        nt = (wl.L + wl.mem_len + 127) // 128
        tiles = wl.B * wl.H * (nt * (nt + 1) // 2 if wl.causal else nt * nt)
        # stored P / dS tiles (up to 32 GiB): D, relation prep, query-tile, one launch of both
        # streaming roles, dr and u/v reductions; else key-tile, query-tile and diagonal kernels;
        # the wide Shaw route adds the table expansion and the collapse of its gradient
        bwd = (6 if tiles * 65536 <= 32 << 30 else 7) + (2 if wide else 0)
    elif tc and wl.mech == SHAW:  # D, per-row q.a products, key-tile, query-tile, da reduction; the value
        bwd = 7 if wl.shaw_value else 5  # side adds the dO.aV products and the daV reduction
    elif tc and wl.mech in (T5, ALIBI):  # bias vector, D, key-tile, query-tile, bucket / slope reduction
        bwd = 5
    elif tc and wl.mech == DEBERTA:  # D, relation products, key-tile, query-tile, rows GEMM, table GEMM, reduction
        bwd = 7
    else:  # D, key-tile, query-tile, then the table-gradient reductions (Shaw's value side: one more)
        bwd = 3 + t5 + {T5: 1, SHAW: 1, TXL: 3, DEBERTA: 2, ALIBI: 1}[wl.mech] + (1 if wl.shaw_value else 0)
    # Transformer-XL memory: the backward fills the placeholder rows' LSE (+inf)
    return fwd, bwd + (1 if wl.mem_len > 0 else 0)


def median_iqr(xs):
    """(median, interquartile range) of a list of timings (linear interpolation)."""
    ys = sorted(xs)

    def q(f):
        x = f * (len(ys) - 1)
        lo = int(math.floor(x))
        hi = min(lo + 1, len(ys) - 1)
        return ys[lo] + (ys[hi] - ys[lo]) * (x - lo)
    return q(0.5), q(0.75) - q(0.25)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


# ----------------------------------------------------------------------------
# clocks sampled during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    """SM clock, its maximum, power and the clock-event reasons of one GPU, read every
    5 ms by an in-process NVML thread (nvidia-smi every 100 ms if NVML is unavailable);
    only samples taken inside the timed region (``mark``) are summarised."""
    PERIOD_S = 0.005
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))
    SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                  "clocks_event_reasons.sw_power_cap")

    def __init__(self, device: torch.device):
        self.device = device
        self.samples = []  # (time, sm_mhz, sm_max_mhz, power_w, reasons)
        self.stop_flag = threading.Event()
        self.thread = None
        self.proc = None
        self.source = None
        self.t0, self.t1 = 0.0, float("inf")

    def _nvml_handle(self):
        """NVML handle of this process's CUDA device (CUDA_VISIBLE_DEVICES honoured)."""
        import pynvml
        pynvml.nvmlInit()
        try:
            idx = torch.cuda._get_nvml_device_index(self.device)
        except Exception:
            idx = self.device.index or 0
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(idx)

    def start(self):
        try:
            nv, h = self._nvml_handle()
            smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            masks = [(name, getattr(nv, attr)) for name, attr in self.REASONS]
        except Exception:
            return self._start_smi()
        self.source = "nvml, 5 ms"

        def run():
            while not self.stop_flag.is_set():
                t = time.time()
                try:
                    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((t, float(sm), float(smax), pw, [n for n, m in masks if rs & m]))
                except Exception:
                    pass
                self.stop_flag.wait(self.PERIOD_S)

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()

    def _start_smi(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.device.index or 0}", f"--query-gpu={self.SMI_FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.source = "nvidia-smi, 100 ms"

        def read():
            names = [n for n, _ in self.REASONS]
            for line in self.proc.stdout:
                f = [x.strip() for x in line.split(",")]
                try:
                    self.samples.append((time.time(), float(f[1]), float(f[2]), float(f[3]),
                                         [n for n, v in zip(names, f[5:9]) if v.lower().startswith("active")]))
                except (ValueError, IndexError):
                    continue

        self.thread = threading.Thread(target=read, daemon=True)
        self.thread.start()
        t_end = time.time() + 5.0  # let the sampler produce its first line before the timed region
        while not self.samples and time.time() < t_end and self.proc.poll() is None:
            time.sleep(0.02)

    def mark(self, t0, t1):
        """Wall-clock bounds of the timed region: only samples taken in it count."""
        self.t0, self.t1 = t0, t1

    def stop(self):
        self.stop_flag.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        if self.source is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source (NVML and nvidia-smi unavailable)"],
                    "samples": 0}
        inside = [x for x in self.samples if self.t0 <= x[0] <= self.t1]
        sm = [x[1] for x in inside]
        reasons = sorted({r for x in inside for r in x[4]})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(x[2] for x in inside) if inside else None,
                "power_w_max": max(x[3] for x in inside) if inside else None, "reasons": reasons, "samples": len(sm),
                "source": self.source}


# ----------------------------------------------------------------------------
# the CPU oracle on a bounded sample (baseline only)
# ----------------------------------------------------------------------------
def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 0) for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_sample(wl, rows_fraction=None):
    """Time the fp64 oracle on one (batch 0, head 0) slice of the workload.
    rows_fraction: only that fraction of query rows (forward rows + their dQ),
    else the whole head forward + backward.  Returns (seconds, flops, sample)."""
    import numpy as np

    import oracle as orc
    from attention_fwd_bwd_flashattention_b200.inputs import to_f64

    lk = None if wl.seqlens_k is None else (wl.seqlens_k[0],)
    one = wl.with_(B=1, H=1, seqlens_k=lk)
    inp = make_inputs(one, 0)
    q, k, v, do = (to_f64(inp[n]) for n in ("q", "k", "v", "do"))
    rel = [to_f64(r) for r in inp["rel"]]
    cfg = orc.RelCfg(t5_num_buckets=wl.t5_num_buckets, t5_max_distance=wl.t5_max_distance,
                     t5_bidirectional=wl.t5_bidirectional, shaw_clip=wl.shaw_clip, deberta_span=wl.deberta_span,
                     shaw_value=wl.shaw_value)
    f_fwd, f_bwd = algo_flops(one)
    t0 = time.perf_counter()
    if wl.mem_len:  # the memory formula on the whole slice (no row sampling)
        orc.txl_memory_forward(q, k, v, rel, wl.scale, cfg)
        orc.txl_memory_backward(q, k, v, rel, do, wl.scale, cfg)
        return (time.perf_counter() - t0, f_fwd + f_bwd,
                f"1 of {wl.B * wl.H} (batch, head) slices, memory {wl.mem_len} + segment {wl.L}, forward + backward")
    if rows_fraction is None:
        orc.forward(wl.mech, q, k, v, rel, wl.causal, wl.scale, cfg, seqlens_k=lk)
        orc.backward(wl.mech, q, k, v, rel, wl.causal, do, wl.scale, cfg, seqlens_k=lk)
        flops = f_fwd + f_bwd
        sample = f"1 of {wl.B * wl.H} (batch, head) slices at full L={wl.L}, forward + backward"
    else:
        step = max(1, int(round(1 / rows_fraction)))
        rows = np.arange(0, wl.L, step)
        orc.forward(wl.mech, q, k, v, rel, wl.causal, wl.scale, cfg, rows=rows, seqlens_k=lk)
        orc.backward_rows(wl.mech, q, k, v, rel, wl.causal, do, rows, wl.scale, cfg, seqlens_k=lk)
        flops = (f_fwd + f_bwd) * len(rows) / wl.L
        sample = f"{len(rows)} of {wl.L} query rows of 1 of {wl.B * wl.H} (batch, head) slices: O, LSE and dQ"
    return time.perf_counter() - t0, flops, sample


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    frac = (1 / 64) * min(1.0, 20 / max(1, args.steps))  # bounded total CPU time for any --steps
    for _ in range(args.warmup):
        oracle_sample(wl, rows_fraction=frac)
    secs, flops = 0.0, 0.0
    for _ in range(args.steps):
        s, f, sample = oracle_sample(wl, rows_fraction=frac)
        secs += s
        flops += f
    value = flops / secs / 1e12
    cores = cpu_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "mech": wl.name.split("_")[0], "B": wl.B, "H": wl.H, "L": wl.L, "d": wl.d,
                   "causal": wl.causal, "l2": "n/a (host)",
                   "seqlens_k": list(wl.seqlens_k) if wl.seqlens_k is not None else None},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------
# Algorithmic FLOPs credited to one launch of a kernel (in units of U = 2 B H d #pairs),
# the distinct products of the method that the kernel computes (recomputed products are
# not credited): the Transformer-XL backward's 8U split over its kernels.
KERNEL_CREDIT_U = {
    (TXL, "tc_bwd_q_kernel"): 5,     # S = Q K^T, the relation products, dP, dS K and E r (dQ)
    (TXL, "tc_bwd_stream_kernel"): 3,  # dV = P^T dO, dK = dS^T Q and G = E^T Q (dr) from the stored tiles
    (TXL, "tc_bwd_kv_kernel"): 2,    # dV, dK (it recomputes S, P, dS: not credited)
    (TXL, "tc_bwd_diag_kernel"): 1,  # the same (recomputing)
}
# DRAM traffic per launch of a kernel (dram__bytes_read.sum + dram__bytes_write.sum) from
# one ncu capture of the same build and workload (profiles/tc_kernels_txl_causal_L8192.md);
# removed whenever that kernel changes.
KERNEL_TRAFFIC = {
    ("txl_causal_L8192_bf16", "tc_fwd_kernel"): 34.50e6,
    ("txl_causal_L8192_bf16", "tc_bwd_q_kernel"): 1137.51e6,
}
# Further workloads timed by the default run (one line, sub-record "workloads"): the other
# configuration quoted at L = 8192 (DeBERTa), the Shaw configuration, and one point of the
# non-causal Transformer-XL length sweep.
SIDE_WORKLOADS = ("deberta_L8192_bf16", "shaw_L2048_bf16", "txl_L16384_bf16")


def params_of(wl, path):
    P = bd.Params(mech=wl.mech, B=wl.B, H=wl.H, L=wl.L, d=wl.d,
                  dtype=bd.BF16 if wl.dtype == torch.bfloat16 else bd.F32, causal=wl.causal, scale=wl.scale,
                  kernel_path=path, t5_num_buckets=wl.t5_num_buckets, t5_max_distance=wl.t5_max_distance,
                  t5_bidirectional=wl.t5_bidirectional, shaw_clip=wl.shaw_clip, deberta_span=wl.deberta_span,
                  shaw_value=wl.shaw_value, mem_len=wl.mem_len)
    return P


class Case:
    """Device buffers of one workload: inputs drawn on the host (seeded), outputs,
    gradients and both workspaces."""

    def __init__(self, wl, dev, rank, path, inp=None, bwd_pass=1):
        self.wl = wl
        self.P = params_of(wl, path)
        if wl.seqlens_k is not None:
            self.P.seqlens_k = torch.tensor(wl.seqlens_k, dtype=torch.int32, device=dev)
        if inp is None:
            inp = make_inputs(wl, seed=rank)
            if rank != 0:  # the relative tables are shared by all ranks (one model)
                inp["rel"] = make_inputs(wl, seed=0)["rel"]
        self.inp = inp
        self.q, self.k, self.v, self.do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
        self.rel = [r.to(dev) for r in inp["rel"]]
        self.ws_f = bd.workspace(self.P, 0, dev)
        self.ws_b = bd.workspace(self.P, bwd_pass, dev)  # 2: the smallest backward workspace
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(self.q.shape[:3], dtype=torch.float32, device=dev)
        self.dq, self.dk, self.dv = torch.empty_like(self.q), torch.empty_like(self.k), torch.empty_like(self.v)
        self.drel = [torch.empty(r.shape, dtype=torch.float32, device=dev) for r in self.rel[: self.P.n_rel()]]

    def fwd(self, stream):
        bd.relpos_attn_fwd(self.P, self.q, self.k, self.v, self.rel, self.o, self.lse, self.ws_f, stream=stream)

    def bwd(self, stream):
        bd.relpos_attn_bwd(self.P, self.q, self.k, self.v, self.rel, self.o, self.lse, self.do, self.dq, self.dk, self.dv,
                           self.drel, self.ws_b, stream=stream)

    def step_bytes(self):
        bufs = [self.q, self.k, self.v, self.do, self.o, self.lse, self.dq, self.dk, self.dv, *self.rel, *self.drel,
                self.ws_f, self.ws_b]
        return sum(t.numel() * t.element_size() for t in bufs if t is not None)

    def paths(self):
        name = {bd.PATH_TC: "tcgen05", bd.PATH_SIMT: "cuda-core fp32"}
        return {"fwd": name[bd.relpos_attn_resolved_path(self.P, 0)], "bwd": name[bd.relpos_attn_resolved_path(self.P, 1)]}


def time_case(c, steps, warmup, flush, stream, reduce_grads, on_region=None):
    """W untimed steps, then `steps` steps each timed with CUDA events on the launching
    stream (fwd and bwd separately), L2 flushed before each (untimed).  The warm-up steps
    trace every kernel the library launches (bd.Trace: events around each launch) to
    find the one with the largest share; in the timed steps only that kernel is
    bracketed by its own events (two per launch, nothing between the other kernels).
    Returns (fwd_ms, bwd_ms, warm, dom) with warm = {name: [ms of each warm-up launch]}
    and dom = (name, [ms of each timed launch])."""
    warm_traces = [bd.Trace(32) for _ in range(warmup)]
    for w in range(warmup):
        flush.fill_(1.0)
        with warm_traces[w]:
            c.fwd(stream)
            c.bwd(stream)
        if reduce_grads:
            rdist.allreduce_table_grads(c.drel)
    torch.cuda.synchronize()
    warm = {}
    for t in warm_traces[1:] or warm_traces:  # the first warm-up step includes one-time set-up
        for name, ms in t.kernels():
            warm.setdefault(name, []).append(ms)
    dom_name = max(warm, key=lambda n: sum(warm[n])) if warm else None
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    traces = [bd.Trace(8, only=dom_name) for _ in range(steps)]
    torch.cuda.synchronize()
    rdist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for s in range(steps):
        flush.fill_(float(s))
        ev[s][0].record(stream)
        with traces[s]:
            c.fwd(stream)
            ev[s][1].record(stream)
            c.bwd(stream)
        if reduce_grads:
            rdist.allreduce_table_grads(c.drel)
        ev[s][2].record(stream)
    torch.cuda.synchronize()
    if on_region is not None:
        on_region(t_wall0, time.time())
    rdist.barrier()
    fwd_ms = [e[0].elapsed_time(e[1]) for e in ev]
    bwd_ms = [e[1].elapsed_time(e[2]) for e in ev]
    dom_ms = [ms for t in traces for _, ms in t.kernels()]
    return fwd_ms, bwd_ms, warm, (dom_name, dom_ms)


def kernel_table(kernels, steps, step_ms):
    """Per kernel: launches per step, mean ms per launch, share of the step."""
    return {n: {"launches_per_step": len(v) / steps, "ms_per_launch": statistics.mean(v),
                "share_of_step": sum(v) / steps / step_ms} for n, v in sorted(kernels.items(), key=lambda kv: -sum(kv[1]))}


def side_workload(name, dev, rank, world, flush, stream, peaks, steps):
    wl = WORKLOADS[name]
    c = Case(wl, dev, rank, bd.PATH_AUTO)
    fwd_ms, bwd_ms, warm, (dom, dom_ms) = time_case(c, steps, 3, flush, stream, False)
    f_fwd, f_bwd = algo_flops(wl)
    fm, bm = median_iqr(fwd_ms)[0], median_iqr(bwd_ms)[0]
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    ktab = kernel_table({dom: dom_ms}, steps, fm + bm) if dom else {}
    out = {"workload": name, "B": wl.B, "H": wl.H, "L": wl.L, "causal": wl.causal, "kernel_path": c.paths(),
           "steps": steps, "fwd_ms_median": fm, "bwd_ms_median": bm,
           "fwd_tflops": f_fwd / (fm * 1e-3) / 1e12, "bwd_tflops": f_bwd / (bm * 1e-3) / 1e12,
           "fwd_bwd_tflops": (f_fwd + f_bwd) / ((fm + bm) * 1e-3) / 1e12,
           "frac_of_measured_bf16_burst": (f_fwd + f_bwd) / ((fm + bm) * 1e-3) / 1e12 / burst,
           "tokens_per_s": wl.B * wl.L / ((fm + bm) * 1e-3),
           "peak_mem_bytes": int(c.step_bytes()),
           "workspace_bytes": {"fwd": bd.relpos_attn_workspace_size(c.P, 0), "bwd": bd.relpos_attn_workspace_size(c.P, 1)},
           "dominant_kernel": {"name": dom, **ktab[dom]} if dom else None}
    del c
    torch.cuda.empty_cache()
    return out


def lean_backward(wl, dev, flush, stream, peaks, steps):
    """The same step with the smallest backward workspace (relpos_attn_workspace_size pass
    2): no stored P / dS tiles, memory O(L); timed like the main step."""
    c = Case(wl, dev, 0, bd.PATH_AUTO, bwd_pass=2)
    fwd_ms, bwd_ms, warm, _ = time_case(c, steps, 3, flush, stream, False)
    f_fwd, f_bwd = algo_flops(wl)
    fm, bm = median_iqr(fwd_ms)[0], median_iqr(bwd_ms)[0]
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    out = {"workspace": "smallest (pass 2)", "steps": steps, "fwd_ms_median": fm, "bwd_ms_median": bm,
           "fwd_bwd_tflops": (f_fwd + f_bwd) / ((fm + bm) * 1e-3) / 1e12,
           "frac_of_measured_bf16_burst": (f_fwd + f_bwd) / ((fm + bm) * 1e-3) / 1e12 / burst,
           "bwd_tflops": f_bwd / (bm * 1e-3) / 1e12, "peak_mem_bytes": int(c.step_bytes()),
           "kernels_warmup": kernel_table(warm, 2, fm + bm)}
    del c
    torch.cuda.empty_cache()
    return out


def run_ours(args, wl):
    rank, world, local = rdist.init_from_env(backend="nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    path_name = "simt" if args.path == "simt" else "auto"
    path = bd.PATH_SIMT if args.path == "simt" else bd.PATH_AUTO
    # N > 1: each rank its own batch of the workload (weak scaling, table gradients
    # all-reduced) or its block of the workload's heads (strong scaling, no collective)
    mode = "single" if world == 1 else args.shard
    if mode == "heads":
        lo, hi = rdist.shard_range(wl.H, rank, world)
        c = Case(wl.with_(H=hi - lo), dev, rank, path, inp=rdist.shard_inputs(make_inputs(wl, seed=0), "heads", rank, world))
    else:
        c = Case(wl, dev, rank, path)
    P = c.P
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    torch.cuda.reset_peak_memory_stats(dev)
    base_mem = torch.cuda.memory_allocated(dev)
    clocks = ClockSampler(dev)
    clocks.start()
    fwd_ms, bwd_ms, warm, (dom, dom_ms) = time_case(c, args.steps, args.warmup, flush, stream, mode == "batch",
                                                    on_region=clocks.mark)
    clk = clocks.stop()
    tot_ms = sum(f + b for f, b in zip(fwd_ms, bwd_ms))
    tot_ms = rdist.max_over_ranks(tot_ms)
    alloc_in_steps = torch.cuda.max_memory_allocated(dev) - base_mem  # 0: the library allocates nothing
    # device memory of one fwd + bwd step: every buffer the two calls read or write
    step_mem = c.step_bytes()
    ws_sizes = {"fwd": bd.relpos_attn_workspace_size(P, 0), "bwd": bd.relpos_attn_workspace_size(P, 1),
                "bwd_smallest": bd.relpos_attn_workspace_size(P, 2)}

    f_fwd, f_bwd = algo_flops(c.wl)  # this rank's work
    fa_f, fa_b = fa_flops(wl)
    ms_step = tot_ms / args.steps
    # whole-job work per step: every rank's batch (weak), or the workload's heads once (strong)
    job = (1 if mode == "heads" else world)
    job_flops = sum(algo_flops(wl)) * job
    value = job_flops / (ms_step * 1e-3) / 1e12
    tokens = job * wl.B * wl.L / (ms_step * 1e-3)
    peaks, peak_src = load_peaks()
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    fwd_avg = statistics.mean(fwd_ms)
    bwd_avg = statistics.mean(bwd_ms)
    # every kernel's share from the traced warm-up steps; the dominant kernel's time from
    # its own events in the timed steps
    ktab_warm = kernel_table(warm, max(1, args.warmup - 1), statistics.mean(fwd_ms) + statistics.mean(bwd_ms))
    ktab = {dom: kernel_table({dom: dom_ms}, args.steps, ms_step)[dom]}
    U = 2.0 * wl.H * wl.d * pairs_of(wl)
    # each pass timed as one unit with events (its helper kernels included): a pass of about
    # a millisecond timed by itself, so the burst peak is the denominator
    passes = []
    for name, fl, ms in (("relpos_attn_fwd", f_fwd, fwd_avg), ("relpos_attn_bwd", f_bwd, bwd_avg)):
        ach = fl / (ms * 1e-3) / 1e12
        passes.append({"pass": name, "achieved": ach, "ms": ms, "frac_of_burst": ach / burst})
    pass_tc = [path_name == "auto" and wl.dtype == torch.bfloat16 and bd.tc_available(P, ps) for ps in (0, 1)]
    dom_tc = not dom.startswith("simt_")
    credit = None
    if dom_tc:
        # the dominant kernel: the one with the largest share of the step, timed with its own
        # events around every launch in the timed region; credited with the algorithmic FLOPs
        # of the products it computes (the forward kernel: the whole forward)
        credit = f_fwd if dom == "tc_fwd_kernel" else (KERNEL_CREDIT_U.get((wl.mech, dom), 0) * U or None)
    if credit is not None:
        per_launch = credit / ktab[dom]["launches_per_step"]
        ach = per_launch / (ktab[dom]["ms_per_launch"] * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": burst, "unit": "TFLOP/s", "frac": ach / burst,
                "traffic": KERNEL_TRAFFIC.get((wl.name, dom)), "kernel": dom, "flops_per_launch": per_launch,
                "ms_per_launch": ktab[dom]["ms_per_launch"], "share_of_step": ktab[dom]["share_of_step"],
                "peak_kind": f"bf16 burst ({peak_src}): kernel timed by itself with events"}
    else:  # no per-kernel credit: the dominant pass, against the peak of the kernel family it runs on
        di = 0 if fwd_avg > bwd_avg else 1
        dp = passes[di]
        if pass_tc[di]:
            roof = {"bound": "tensor", "achieved": dp["achieved"], "peak": burst, "unit": "TFLOP/s",
                    "frac": dp["frac_of_burst"], "traffic": None, "kernel": dp["pass"],
                    "peak_kind": f"bf16 burst ({peak_src}): pass timed as one unit"}
        else:
            # CUDA-core path: fp32 FFMA bound, peak = 148 SMs x 128 lanes x 2 flop x max SM clock
            peak = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
            roof = {"bound": "alu", "achieved": dp["achieved"], "peak": peak, "unit": "TFLOP/s",
                    "frac": dp["achieved"] / peak, "traffic": None, "kernel": dp["pass"],
                    "peak_kind": "fp32 FFMA, 148 SM x 128 lanes x 2 x max clock"}
    tensor_path = pass_tc[0] and pass_tc[1]

    # ---- end to end through the public API: pinned host in, host out ----
    e2e = run_e2e(args, wl, c, dev, stream, world, mode)

    lean = None
    if (world == 1 and path_name == "auto" and not args.no_side_workloads
            and bd.relpos_attn_workspace_size(P, 2) < bd.relpos_attn_workspace_size(P, 1)):
        lean = lean_backward(wl, dev, flush, stream, peaks, min(args.steps, 50))
    side = []
    if not args.no_side_workloads and world == 1 and path_name == "auto":
        for name in SIDE_WORKLOADS:
            if name != wl.name:
                side.append(side_workload(name, dev, rank, world, flush, stream, peaks, min(args.steps, 10)))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        secs, flops, sample = oracle_sample(wl)
        cpu = {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
               "sample": sample, "seconds": secs}

    fl, bl = kernel_launches(wl, path_name if not tensor_path else "tc")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if mode == "heads" else "weak",
        "vs_baseline": None, "dtype": "bf16" if wl.dtype == torch.bfloat16 else "f32", "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "H": wl.H, "L": wl.L, "d": wl.d, "causal": wl.causal,
                   "seqlens_k": list(wl.seqlens_k) if wl.seqlens_k is not None else None, "mem_len": wl.mem_len,
                   "kernel_path": c.paths(),
                   "l2": "flushed before every timed step (256 MB write, untimed)",
                   "parallelism": {"single": "single GPU", "batch": f"dp{world} (weak; table grads all-reduced)",
                                   "heads": f"heads split over {world} GPUs (strong; no collective)"}[mode]},
        "tokens_per_s": tokens,
        "fwd_ms": fwd_avg, "bwd_ms": bwd_avg,
        "fwd_tflops": f_fwd / (fwd_avg * 1e-3) / 1e12, "bwd_tflops": f_bwd / (bwd_avg * 1e-3) / 1e12,
        "fa_convention_tflops": job * (fa_f + fa_b) / (ms_step * 1e-3) / 1e12,
        "frac_of_dense_bf16_datasheet": value / world / 2250.0,  # per GPU
        "frac_of_measured_bf16": value / world / burst,
        "peak_mem_bytes": int(step_mem),
        "peak_mem_smallest_workspace_bytes": int(step_mem - ws_sizes["bwd"] + ws_sizes["bwd_smallest"]),
        "workspace_bytes": ws_sizes,
        "alloc_during_steps_bytes": int(alloc_in_steps),
        "timing_ms": {"fwd_median": median_iqr(fwd_ms)[0], "fwd_iqr": median_iqr(fwd_ms)[1],
                      "bwd_median": median_iqr(bwd_ms)[0], "bwd_iqr": median_iqr(bwd_ms)[1]},
        "roofline": roof,
        "roofline_passes": passes,
        "kernels_warmup": ktab_warm,
        "cpu_baseline": cpu,
        "e2e": e2e,
        # launches of this library's kernels in the timed steps: the traced warm-up steps'
        # count per step (the dispatch table of csrc/api.cu gives gpu_launches_expected)
        "gpu_launches": round(sum(len(v) for v in warm.values()) / max(1, args.warmup - 1) * args.steps),
        "gpu_launches_expected": (fl + bl) * args.steps,
        "clocks": clk,
        "workloads": side,
        "smallest_workspace": lean,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    rdist.shutdown()
    return 0


def run_e2e(args, wl, c, dev, stream, world, mode="single"):
    """Same metric through the public entry points, with every step's inputs copied
    from pinned host memory and its results (O, LSE, dQ, dK, dV, drel) copied back.  Steps are
    pipelined over two buffer sets: step k's host-to-device copies (one stream) and
    step k - 1's device-to-host copies (another) overlap step k - 1's / k's kernels (the
    compute stream); within a step dO's copy overlaps the forward and O / LSE go back
    under the backward; events order every reuse of a buffer.  The timed region runs from
    the first input copy to the last result copy."""
    P, inp = c.P, c.inp
    host_in = {n: inp[n].pin_memory() for n in ("q", "k", "v", "do")}
    host_rel = [r.pin_memory() for r in inp["rel"]]
    ws_f = bd.workspace(P, 0, dev)
    ws_b = bd.workspace(P, 1, dev)

    def buffers():
        b = {n: torch.empty_like(host_in[n], device=dev) for n in ("q", "k", "v", "do")}
        b["rel"] = [torch.empty_like(r, device=dev) for r in host_rel]
        b["o"] = torch.empty_like(b["q"])
        b["lse"] = torch.empty(b["q"].shape[:3], dtype=torch.float32, device=dev)
        b["dq"], b["dk"], b["dv"] = (torch.empty_like(b["q"]) for _ in range(3))
        b["drel"] = [torch.empty(r.shape, dtype=torch.float32, device=dev) for r in b["rel"][: P.n_rel()]]
        b["out"] = [torch.empty_like(t, device="cpu").pin_memory() for t in results(b)]
        return b

    def results(b):  # everything the step returns: O, LSE, dQ, dK, dV and the table gradients
        return [b["o"], b["lse"], b["dq"], b["dk"], b["dv"]] + b["drel"]

    bufs = [buffers(), buffers()]
    h2d = sum(t.numel() * t.element_size() for t in list(host_in.values()) + host_rel)
    d2h = sum(t.numel() * t.element_size() for t in bufs[0]["out"])
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]     # q, k, v and the tables landed
    ev_in_do = [torch.cuda.Event() for _ in range(2)]  # dO landed (the backward's only extra input)
    ev_fwd = [torch.cuda.Event() for _ in range(2)]    # O, LSE written
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def step(kk):
        i = kk & 1
        B = bufs[i]
        res = results(B)
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_done[i])  # the kernels of step kk - 2 are done with these inputs
            for n in ("q", "k", "v"):
                B[n].copy_(host_in[n], non_blocking=True)
            for dst, src in zip(B["rel"], host_rel):
                dst.copy_(src, non_blocking=True)
            ev_in[i].record(s_in)
            B["do"].copy_(host_in["do"], non_blocking=True)  # under the forward
            ev_in_do[i].record(s_in)
        with torch.cuda.stream(stream):
            stream.wait_event(ev_in[i])
            stream.wait_event(ev_out[i])  # step kk - 2's results have left these buffers
            bd.relpos_attn_fwd(P, B["q"], B["k"], B["v"], B["rel"], B["o"], B["lse"], ws_f, stream=stream)
            ev_fwd[i].record(stream)
            stream.wait_event(ev_in_do[i])
            bd.relpos_attn_bwd(P, B["q"], B["k"], B["v"], B["rel"], B["o"], B["lse"], B["do"], B["dq"], B["dk"], B["dv"],
                               B["drel"], ws_b, stream=stream)
            if mode == "batch":
                rdist.allreduce_table_grads(B["drel"])
            ev_done[i].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_fwd[i])  # O and LSE go out under the backward (which only reads them)
            for dst, src in zip(B["out"][:2], res[:2]):
                dst.copy_(src, non_blocking=True)
            s_out.wait_event(ev_done[i])
            for dst, src in zip(B["out"][2:], res[2:]):
                dst.copy_(src, non_blocking=True)
            ev_out[i].record(s_out)

    for kk in range(max(1, args.warmup)):
        step(kk)
    torch.cuda.synchronize()
    rdist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for kk in range(args.steps):
        step(kk)
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = rdist.max_over_ranks(e0.elapsed_time(e1)) / args.steps
    job_flops = sum(algo_flops(wl)) * (1 if mode == "heads" else world)
    return {"value": job_flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipeline": "two buffer sets; host-to-device, kernels and device-to-host on three streams"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)  # about half a second of timed work at the default workload
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--path", default="auto", choices=["auto", "simt"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-side-workloads", action="store_true", help="time only the main workload")
    ap.add_argument("--shard", default="batch", choices=["batch", "heads"],
                    help="N > 1: each rank its own batch (weak scaling) or a block of the heads (strong scaling)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least three untimed warm-up steps
    wl = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_ours(args, wl)


if __name__ == "__main__":
    sys.exit(main())
