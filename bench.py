#!/usr/bin/env python
"""Benchmark of the varlen attention hot path on B200.

One step = the whole path on one batch: work-list preparation, forward
(out, logsumexp), then backward (preprocess, dQ/dK/dV, dQ conversion), on the
fwd+bwd workload: 16384 packed tokens, lengths U{512..8192} (seed 5, last
clipped), 16 heads, head_dim 128, causal, bf16 inputs ~N(0,1).

FLOPs: F_fwd = 4 * sum_b lq_b * lk_b * heads * head_dim, halved for causal;
backward = 2.5 * F_fwd; the headline fwd+bwd figure uses 3.5 * F_fwd (the
literal 2.5 * F_fwd / step time is reported beside it, labelled).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs the same workload shape on its own
seeded data (weak scaling, no collective on the data path); timing is the
max over ranks. Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import random
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from varlen_flashattention_02_b200 import synth  # noqa: E402

METRIC = "attention TFLOP/s (fwd, fwd+bwd) at 1 B200 and % of dense BF16 peak"
UNIT = "TFLOP/s"
WORKLOAD = ("varlen fwd+bwd: 16384 total tokens, lengths uniform int [512,8192] from seed 5 (last clipped), "
            "16 heads, head_dim 128, bf16 Q/K/V/dO ~N(0,1), causal, LSE saved fwd, outputs dQ/dK/dV")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLUSH_BYTES = 256 << 20


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process
    group). Works with NCCL (CUDA tensor) and gloo (CPU tensor)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def head_range(heads: int, world: int, rank: int) -> tuple[int, int]:
    """Heads [h0, h1) of rank ``rank`` when the heads of one problem are split
    across ``world`` GPUs: contiguous, balanced (the first heads % world ranks
    take one extra head). Every (sequence, head) unit is independent in both
    directions, so the ranks exchange nothing; cu_seqlens is replicated."""
    if world < 1 or not 0 <= rank < world or heads < world:
        raise ValueError(f"cannot split {heads} heads over {world} ranks (rank {rank})")
    base, extra = divmod(heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def shard_heads(tensors: dict, h0: int, h1: int, kv_group: int = 1) -> dict:
    """This rank's slice of packed [tokens, heads, d] arrays (bf16 bits):
    query-side arrays (q, dout) take heads [h0, h1); key/value arrays take the
    key/value heads those query heads read (h / kv_group). Contiguous copies,
    so each slice is again a packed [tokens, h1 - h0, d] problem."""
    if h0 % kv_group or h1 % kv_group:
        raise ValueError("a rank's heads must cover whole key/value groups")
    out = {}
    for n, a in tensors.items():
        lo, hi = (h0, h1) if n in ("q", "dout") else (h0 // kv_group, h1 // kv_group)
        out[n] = np.ascontiguousarray(a[:, lo:hi, :])
    return out


def sequence_split(cu_q, cu_k, world: int) -> list:
    """Sequences of each rank when the sequences of one problem are split
    across ``world`` GPUs, balanced by attention work: sequence b costs
    lq_b * lk_b (a causal mask halves every cost alike), and the sequences,
    largest first, go one by one to the rank with the least work so far (ties
    to the lower rank, then to the lower sequence index). Each rank's list is
    in sequence order. Every (sequence, head) unit is independent in both
    directions, so the ranks exchange nothing."""
    lq = np.diff(np.asarray(cu_q, dtype=np.int64))
    lk = np.diff(np.asarray(cu_k, dtype=np.int64))
    if world < 1 or len(lq) < world:
        raise ValueError(f"cannot split {len(lq)} sequences over {world} ranks")
    cost = lq * lk
    load = [0] * world
    parts = [[] for _ in range(world)]
    for b in sorted(range(len(cost)), key=lambda i: (-int(cost[i]), i)):
        r = min(range(world), key=lambda i: (load[i], i))
        parts[r].append(b)
        load[r] += int(cost[b])
    return [sorted(x) for x in parts]


def shard_sequences(tensors: dict, cu_q, cu_k, seqs) -> tuple:
    """This rank's problem: the rows of sequences ``seqs`` (in that order)
    packed back to back, query-side arrays (q, dout) from cu_q and key/value
    arrays from cu_k, with their own cumulative offsets."""
    cu_q = np.asarray(cu_q, dtype=np.int64)
    cu_k = np.asarray(cu_k, dtype=np.int64)

    def rows(cu):
        return np.concatenate([np.arange(cu[b], cu[b + 1]) for b in seqs]).astype(np.int64)

    def offsets(cu):
        return np.concatenate([[0], np.cumsum([cu[b + 1] - cu[b] for b in seqs])]).astype(np.int32)

    rq, rk = rows(cu_q), rows(cu_k)
    out = {n: np.ascontiguousarray(a[rq if n in ("q", "dout") else rk]) for n, a in tensors.items()}
    return out, offsets(cu_q), offsets(cu_k)


def weak_scaling_value(world: int, flops_per_rank: float, max_ms_per_step: float) -> float:
    """Whole-job TFLOP/s: every rank did ``flops_per_rank`` per step; the job's
    step time is the slowest rank's."""
    return world * flops_per_rank / (max_ms_per_step * 1e-3) / 1e12


def fwd_flops(cu_q, cu_k, heads, head_dim, causal, units=None):
    lq = np.diff(np.asarray(cu_q, dtype=np.int64))
    lk = np.diff(np.asarray(cu_k, dtype=np.int64))
    if units is None:
        total = float(np.sum(lq * lk)) * heads
    else:
        total = float(sum(lq[b] * lk[b] for b, _ in units))
    f = 4.0 * total * head_dim
    return f / 2 if causal else f


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples the SM clock and the clock-event reasons of one GPU through NVML
    every 5 ms on a background thread while the timed region runs (read-only;
    no setting of the GPU is touched)."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown", 0x8),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap", 0x4),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80))

    def __init__(self, uuid: str | None):
        self.samples = []
        self.handle = None
        self.thread = None
        self.stop_flag = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(uuid) if uuid else pynvml.nvmlDeviceGetHandleByIndex(0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.handle = None

    def _run(self):
        nv = self.nvml
        while not self.stop_flag:
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((sm, rs))
            except Exception:
                pass
            time.sleep(0.005)

    def start(self):
        if self.handle is None:
            return
        import threading

        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def stop(self):
        if self.handle is None or self.thread is None:
            return None
        self.stop_flag = True
        self.thread.join()
        if not self.samples:
            return None
        reasons = set()
        for _, rs in self.samples:
            for name, attr, default in self.REASONS:
                if rs & getattr(self.nvml, attr, default):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s for s, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples), "source": "NVML, 5 ms period"}


# ----------------------------------------------------------------- our arm
def kernel_traffic(kernel_file: str):
    """Per-launch DRAM bytes of the dominant kernel from the committed ncu
    summary, if it was taken on the current source of that kernel."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    src = os.path.join(ROOT, "varlen_flashattention_02_b200", "csrc", kernel_file)
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    ent = d.get(kernel_file)
    if not ent or ent.get("source_sha256_16") != h:
        return None
    return ent.get("dram_bytes_per_launch")


def bench_workload(tokens: int):
    """The fwd+bwd workload; ``tokens`` < 16384 gives the same recipe on fewer
    tokens (used only for small profiling captures)."""
    if tokens == synth.TOTAL_TOKENS:
        return synth.standard_workload(5)
    lens = synth.lengths_uniform(5, tokens, 512, 8192)
    return synth.make_workload(f"varlen-{tokens}-U512..8192-h16-d128-causal", lens, heads=16, head_dim=128,
                               causal=True, seed=5, with_grad=True)


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from varlen_flashattention_02_b200 import fa_varlen

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = bench_workload(args.tokens)
    split_heads = args.split in ("heads", "sequences") and world > 1  # one problem over the ranks
    heads_job, batch_job, tokens_job = w.heads, w.batch, w.total_q
    if split_heads:
        F_job = fwd_flops(w.cu_q, w.cu_k, w.heads, w.head_dim, w.causal)
    if split_heads and args.split == "heads":
        # One problem, its heads split across the ranks: every rank draws the
        # same seeded batch and keeps its contiguous slice of heads.
        h0, h1 = head_range(w.heads, world, rank)
        t = shard_heads(w.tensors(), h0, h1)
        w.heads = h1 - h0
    elif split_heads:
        # One problem, its sequences split across the ranks by work: every
        # rank draws the same seeded batch and keeps its sequences, repacked.
        seqs = sequence_split(w.cu_q, w.cu_k, world)[rank]
        t, w.cu_q, w.cu_k = shard_sequences(w.tensors(), w.cu_q, w.cu_k, seqs)
    else:
        w.seed = w.seed + 1000 * rank  # same shape, own data per rank
        t = w.tensors()
    H, D = w.heads, w.head_dim

    def dev_bf16(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    q, k, v, do = (dev_bf16(t[n]) for n in ("q", "k", "v", "dout"))
    cu_q = torch.from_numpy(w.cu_q).to(dev)
    cu_k = torch.from_numpy(w.cu_k).to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((H, w.total_q), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_f = fa_varlen.new_workspace(fa_varlen.fwd_workspace_size(w.batch, w.total_q, H, D), dev)
    ws_b = fa_varlen.new_workspace(fa_varlen.bwd_workspace_size(w.batch, w.total_q, w.total_k, H, D), dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    lib = fa_varlen.lib

    def fwd():
        fa_varlen.fa_varlen_fwd(q, k, v, cu_q, cu_k, w.max_seqlen_q, w.max_seqlen_k, w.scale, w.causal,
                                out=out, softmax_lse=lse, workspace=ws_f, stream=stream)

    def bwd():
        fa_varlen.fa_varlen_bwd(do, q, k, v, out, lse, cu_q, cu_k, w.max_seqlen_q, w.max_seqlen_k, w.scale,
                                w.causal, dq=dq, dk=dk, dv=dv, workspace=ws_b, stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        fwd()
        bwd()
    torch.cuda.synchronize(dev)
    if fa_varlen.device_status(ws_f) != 0 or fa_varlen.device_status(ws_b) != 0:
        raise RuntimeError("device status not OK after warm-up")

    def mk():
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)  # materialise the handle
        return e

    K = args.steps
    step_ev = [(mk(), mk()) for _ in range(K)]
    fwd_ev = [[mk() for _ in range(4)] for _ in range(K)]   # prep, attention
    bwd_ev = [[mk() for _ in range(8)] for _ in range(K)]   # prep, preprocess, main, convert
    import ctypes

    fwd_arr = [(ctypes.c_void_p * 4)(*[e.cuda_event for e in evs]) for evs in fwd_ev]
    bwd_arr = [(ctypes.c_void_p * 8)(*[e.cuda_event for e in evs]) for evs in bwd_ev]
    torch.cuda.synchronize(dev)

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    wall0 = time.perf_counter()
    for i in range(K):
        flush.zero_()
        step_ev[i][0].record(stream)
        lib.fa_set_kernel_events(fwd_arr[i], 2)
        fwd()
        lib.fa_set_kernel_events(bwd_arr[i], 4)
        bwd()
        lib.fa_set_kernel_events(None, 0)
        step_ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    wall1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    if fa_varlen.device_status(ws_f) != 0 or fa_varlen.device_status(ws_b) != 0:
        raise RuntimeError("device status not OK after the timed steps")

    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    fwd_call_ms = [evs[0].elapsed_time(evs[3]) for evs in fwd_ev]
    fwd_kern_ms = [evs[2].elapsed_time(evs[3]) for evs in fwd_ev]
    bwd_call_ms = [evs[0].elapsed_time(evs[7]) for evs in bwd_ev]
    bwd_main_ms = [evs[4].elapsed_time(evs[5]) for evs in bwd_ev]
    per_kernel = {
        "sched_prep_fwd": statistics.mean(evs[0].elapsed_time(evs[1]) for evs in fwd_ev),
        "fwd_attention": statistics.mean(fwd_kern_ms),
        "sched_prep_bwd": statistics.mean(evs[0].elapsed_time(evs[1]) for evs in bwd_ev),
        "bwd_preprocess": statistics.mean(evs[2].elapsed_time(evs[3]) for evs in bwd_ev),
        "bwd_attention": statistics.mean(bwd_main_ms),
        "bwd_dq_convert": statistics.mean(evs[6].elapsed_time(evs[7]) for evs in bwd_ev),
    }
    tot_ms = max_over_ranks(sum(step_ms), dev)
    F = fwd_flops(w.cu_q, w.cu_k, H, D, w.causal)  # this rank's share
    ms_step = tot_ms / K
    if split_heads:
        value = 3.5 * F_job / (ms_step * 1e-3) / 1e12  # the whole problem per slowest rank's step
    else:
        value = weak_scaling_value(world, 3.5 * F, ms_step)

    # ---- end to end through the public API with host buffers (pinned)
    host_in = {n: torch.from_numpy(t[n].view(np.int16)).view(torch.bfloat16).pin_memory()
               for n in ("q", "k", "v", "dout")}
    host_cu = (torch.from_numpy(w.cu_q).pin_memory(), torch.from_numpy(w.cu_k).pin_memory())
    host_out = [torch.empty(x.shape, dtype=torch.bfloat16).pin_memory() for x in (dq, dk, dv)]
    h2d = sum(x.numel() * x.element_size() for x in host_in.values()) + sum(x.numel() * 4 for x in host_cu)
    d2h = sum(x.numel() * x.element_size() for x in host_out)
    # Pipelined: while step i computes, the inputs of step i+1 travel to the
    # device on a copy stream and the gradients of step i-1 travel back on
    # another; every step still moves all of its inputs and outputs inside
    # the timed region. Two device copies of the inputs and gradients
    # alternate between steps.
    e2e_steps = 0 if args.no_e2e else max(6, min(2 * K, 20))
    sets = [dict(q=q, k=k, v=v, do=do, cu_q=cu_q, cu_k=cu_k, dq=dq, dk=dk, dv=dv)]
    sets.append({n: torch.empty_like(x) for n, x in sets[0].items()})
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)

    def e2e_step(i, ev_in, ev_comp, ev_out):
        b = sets[i % 2]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_comp[i - 2])  # set i%2's inputs no longer in use
            for n in ("q", "k", "v"):
                b[n].copy_(host_in[n], non_blocking=True)
            b["do"].copy_(host_in["dout"], non_blocking=True)
            b["cu_q"].copy_(host_cu[0], non_blocking=True)
            b["cu_k"].copy_(host_cu[1], non_blocking=True)
            ev_in[i].record(s_in)
        stream.wait_event(ev_in[i])
        if i >= 2:
            stream.wait_event(ev_out[i - 2])  # set i%2's gradients copied out
        fa_varlen.fa_varlen_fwd(b["q"], b["k"], b["v"], b["cu_q"], b["cu_k"], w.max_seqlen_q, w.max_seqlen_k,
                                w.scale, w.causal, out=out, softmax_lse=lse, workspace=ws_f, stream=stream)
        fa_varlen.fa_varlen_bwd(b["do"], b["q"], b["k"], b["v"], out, lse, b["cu_q"], b["cu_k"], w.max_seqlen_q,
                                w.max_seqlen_k, w.scale, w.causal, dq=b["dq"], dk=b["dk"], dv=b["dv"],
                                workspace=ws_b, stream=stream)
        ev_comp[i].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[i])
            host_out[0].copy_(b["dq"], non_blocking=True)
            host_out[1].copy_(b["dk"], non_blocking=True)
            host_out[2].copy_(b["dv"], non_blocking=True)
            ev_out[i].record(s_out)

    def run_e2e(n):
        ev_in, ev_comp, ev_out = ([torch.cuda.Event() for _ in range(n)] for _ in range(3))
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        for i in range(n):
            e2e_step(i, ev_in, ev_comp, ev_out)
        s_out.wait_event(ev_out[n - 1])
        t1.record(s_out)
        torch.cuda.synchronize(dev)
        return t0.elapsed_time(t1)

    if e2e_steps:
        run_e2e(2)  # untimed warm-up of the copy streams
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e2e_ms = run_e2e(e2e_steps) / e2e_steps if e2e_steps else float("nan")
    if e2e_steps and (fa_varlen.device_status(ws_f) != 0 or fa_varlen.device_status(ws_b) != 0):
        raise RuntimeError("device status not OK after the end-to-end steps")
    e2e_ms = max_over_ranks(e2e_ms, dev)
    if world > 1:
        dist.barrier()
    e2e_value = (3.5 * F_job / (e2e_ms * 1e-3) / 1e12) if split_heads else weak_scaling_value(world, 3.5 * F, e2e_ms)
    e2e = None if not e2e_steps else {
        "value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
        "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps,
        "pipelining": "step i+1's inputs copied in while step i computes; step i's gradients copied out "
                      "while step i+1 computes (copy streams, two device buffer sets)"}

    peaks, peak_src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    bwd_main = statistics.mean(bwd_main_ms)
    achieved = 2.5 * F / (bwd_main * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": "bwd_attention (fa_bwd_sm100.cu, bwd_kernel<128,causal>)",
                "achieved": achieved, "peak": peak, "peak_source": f"{peak_src} bf16_tflops (burst)",
                "unit": UNIT, "frac": achieved / peak,
                "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained", peak)),
                "traffic": kernel_traffic("fa_bwd_sm100.cu"),
                "algorithmic": "2.5 * F_fwd FLOPs per launch (5 bf16 matmuls over visible tiles, causal halved)"}
    fwd_k = statistics.mean(fwd_kern_ms)
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "strong" if split_heads else "weak",
        "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded bf16 N(0,1); lengths from numpy default_rng)",
        "config": {"workload": WORKLOAD, "total_tokens": tokens_job, "batch": batch_job, "heads": heads_job,
                   "head_dim": D, "causal": True, "max_seqlen": w.max_seqlen_q,
                   "flops_fwd": F, "flop_convention": "fwd+bwd = 3.5 * F_fwd (bwd = 2.5 * F_fwd); causal halved",
                   "l2": "256 MiB buffer written between steps (and step inputs exceed L2)",
                   "parallelism": (f"strong: heads split over {world} ranks (contiguous slices, cu_seqlens "
                                   f"replicated, no data-path collective)" if split_heads and args.split == "heads"
                                   else f"strong: sequences split over {world} ranks, balanced by lq*lk (each "
                                   f"rank's sequences repacked, no data-path collective)" if split_heads else
                                   f"weak: {world} independent replicas of the workload, no data-path collective")},
        "fwd_tflops": F / (statistics.mean(fwd_call_ms) * 1e-3) / 1e12,
        "bwd_tflops": 2.5 * F / (statistics.mean(bwd_call_ms) * 1e-3) / 1e12,
        "fwd_bwd_tflops_literal_2p5": weak_scaling_value(world, 2.5 * F, ms_step),
        "fwd_kernel_tflops": F / (fwd_k * 1e-3) / 1e12,
        "pct_of_peak": {"fwd_bwd": 100 * value / world / peak,
                        "fwd": 100 * F / (statistics.mean(fwd_call_ms) * 1e-3) / 1e12 / peak,
                        "bwd": 100 * 2.5 * F / (statistics.mean(bwd_call_ms) * 1e-3) / 1e12 / peak,
                        "denominator": f"{peak} TFLOP/s ({peak_src} bf16 burst)"},
        "kernel_ms": per_kernel,
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": 6 * K,
        "clocks": clocks,
        "wall_s_timed_region": wall1 - wall0,
    }
    if rank == 0 and not args.no_aux:
        result["fwd_by_workload"] = fwd_only_workloads(dev, stream, flush, peak)
        result["bwd_by_workload"] = bwd_workloads(dev, stream, flush, peak)
        result["decode_by_workload"] = decode_workloads(dev, stream, float(peaks["hbm_gbs"]))
    return result, w


def fwd_only_workloads(dev, stream, flush, peak, iters=10):
    """Forward TFLOP/s of the other standard workloads (same launch path)."""
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    res = {}
    gqa = lambda: synth.make_workload("gqa", synth.lengths_uniform(5, synth.TOTAL_TOKENS, 512, 8192), heads=32,
                                      head_dim=128, causal=True, seed=5, heads_k=8)
    d256 = lambda: synth.make_workload("d256", synth.lengths_uniform(5, synth.TOTAL_TOKENS, 512, 8192), heads=16,
                                       head_dim=256, causal=True, seed=5)
    specs = [("varlen-2seq-h12-d64 (cu_q=[0,200,1024], cu_k=[0,300,1024])", 1, {}),
             ("fixed-8x2048-h16-d128 non-causal", 2, {"causal": False}),
             ("fixed-8x2048-h16-d128 causal", 2, {"causal": True}),
             ("packed-16k-U128..4096-h32-d128 causal", 3, {}),
             ("long-1x16384-h16-d64 causal", 4, {"head_dim": 64}),
             ("long-1x16384-h16-d128 causal", 4, {"head_dim": 128}),
             ("grouped-query varlen-16k-U512..8192 (seed 5) h32 kv8 d128 causal", gqa, {}),
             ("varlen-16k-U512..8192 (seed 5) h16 d256 causal", d256, {})]
    for name, n, kw in specs:
        w = n() if callable(n) else synth.standard_workload(n, **kw)
        fwd_fn = fa_varlen.fa_varlen_fwd_gqa if w.kv_heads != w.heads else fa_varlen.fa_varlen_fwd
        t = w.tensors()
        mk = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(dev)
        q, k, v = mk(t["q"]), mk(t["k"]), mk(t["v"])
        cq, ck = torch.from_numpy(w.cu_q).to(dev), torch.from_numpy(w.cu_k).to(dev)
        out = torch.empty_like(q)
        lse = torch.empty((w.heads, w.total_q), dtype=torch.float32, device=dev)
        ws = fa_varlen.new_workspace(fa_varlen.fwd_workspace_size(w.batch, w.total_q, w.heads, w.head_dim), dev)
        call = lambda: fwd_fn(q, k, v, cq, ck, w.max_seqlen_q, w.max_seqlen_k, w.scale, w.causal, out=out,
                              softmax_lse=lse, workspace=ws, stream=stream)
        for _ in range(3):
            call()
        evs = []
        for _ in range(iters):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            call()
            b.record(stream)
            evs.append((a, b))
        torch.cuda.synchronize(dev)
        ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
        F = fwd_flops(w.cu_q, w.cu_k, w.heads, w.head_dim, w.causal)
        res[name] = {"ms": ms, "tflops": F / (ms * 1e-3) / 1e12, "pct_of_peak": 100 * F / (ms * 1e-3) / 1e12 / peak}
        del q, k, v, out, lse, ws
    return res


def bwd_workloads(dev, stream, flush, peak, iters=10):
    """Backward (and fwd+bwd) TFLOP/s of the fwd+bwd workload's lengths at the
    other head dimensions and with grouped heads (same launch path as the
    headline: the whole fa_varlen_bwd call, work list included)."""
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    lens = synth.lengths_uniform(5, synth.TOTAL_TOKENS, 512, 8192)
    specs = [("varlen-16k-U512..8192 (seed 5) h16 d64 causal",
              lambda: synth.make_workload("d64", lens, heads=16, head_dim=64, causal=True, seed=5)),
             ("grouped-query varlen-16k-U512..8192 (seed 5) h32 kv8 d128 causal",
              lambda: synth.make_workload("gqa", lens, heads=32, head_dim=128, causal=True, seed=5, heads_k=8)),
             ("varlen-16k-U512..8192 (seed 5) h16 d256 causal",
              lambda: synth.make_workload("d256", lens, heads=16, head_dim=256, causal=True, seed=5))]
    res = {}
    for name, make in specs:
        w = make()
        t = w.tensors()
        mk = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(dev)
        q, k, v, do = mk(t["q"]), mk(t["k"]), mk(t["v"]), mk(t["dout"])
        cq, ck = torch.from_numpy(w.cu_q).to(dev), torch.from_numpy(w.cu_k).to(dev)
        out = torch.empty_like(q)
        lse = torch.empty((w.heads, w.total_q), dtype=torch.float32, device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        wsf = fa_varlen.new_workspace(fa_varlen.fwd_workspace_size(w.batch, w.total_q, w.heads, w.head_dim), dev)
        wsb = fa_varlen.new_workspace(
            fa_varlen.bwd_workspace_size(w.batch, w.total_q, w.total_k, w.heads, w.head_dim), dev)
        fwd_fn = fa_varlen.fa_varlen_fwd_gqa if w.kv_heads != w.heads else fa_varlen.fa_varlen_fwd
        bwd_fn = fa_varlen.fa_varlen_bwd_gqa if w.kv_heads != w.heads else fa_varlen.fa_varlen_bwd
        fwd = lambda: fwd_fn(q, k, v, cq, ck, w.max_seqlen_q, w.max_seqlen_k, w.scale, True, out=out,
                             softmax_lse=lse, workspace=wsf, stream=stream)
        bwd = lambda: bwd_fn(do, q, k, v, out, lse, cq, ck, w.max_seqlen_q, w.max_seqlen_k, w.scale, True, dq=dq,
                             dk=dk, dv=dv, workspace=wsb, stream=stream)
        for _ in range(3):
            fwd()
            bwd()
        tf, tb = [], []
        for _ in range(iters):
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            flush.zero_()
            evs[0].record(stream)
            fwd()
            evs[1].record(stream)
            bwd()
            evs[2].record(stream)
            torch.cuda.synchronize(dev)
            tf.append(evs[0].elapsed_time(evs[1]))
            tb.append(evs[1].elapsed_time(evs[2]))
        if fa_varlen.device_status(wsf) != 0 or fa_varlen.device_status(wsb) != 0:
            raise RuntimeError(f"device status not OK in {name}")
        F = fwd_flops(w.cu_q, w.cu_k, w.heads, w.head_dim, True)
        ms_f, ms_b = statistics.mean(tf), statistics.mean(tb)
        res[name] = {"fwd_ms": ms_f, "bwd_ms": ms_b, "bwd_tflops": 2.5 * F / (ms_b * 1e-3) / 1e12,
                     "bwd_pct_of_peak": 100 * 2.5 * F / (ms_b * 1e-3) / 1e12 / peak,
                     "fwd_bwd_tflops": 3.5 * F / ((ms_f + ms_b) * 1e-3) / 1e12}
        del q, k, v, do, out, lse, dq, dk, dv, wsf, wsb
    return res


def decode_workloads(dev, stream, hbm_peak_gbs, iters=20):
    """Split-KV decoding: one query token per sequence against a long key/value
    cache, 32 query heads over 8 key/value heads, d=128. The bound is HBM: the
    figure is the K/V bytes the call must read over its time, against the
    measured copy bandwidth. The key/value cache is 4x to 17x the L2, so no
    flush runs between calls (a write flush would leave L2 full of dirty lines
    whose write-back this DRAM-bound call would then pay for); the calls are
    queued back to back and timed together, so that host-side launch work
    never leaves the device idle inside the timed region."""
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    res = {}
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    for batch, lk in ((64, 8192), (4, 32768)):
        # The same seeded inputs as the split-KV parity test at these shapes.
        w = synth.decode_workload(batch, lk)
        H, Hk, D = w.heads, w.kv_heads, w.head_dim
        t = w.tensors()
        q, k, v = (torch.from_numpy(t[n].view(np.int16)).view(torch.bfloat16).to(dev) for n in ("q", "k", "v"))
        cu_q = torch.from_numpy(w.cu_q).to(dev)
        cu_k = torch.from_numpy(w.cu_k).to(dev)
        splits = fa_varlen.fa_varlen_splitkv_num_splits(batch, 1, H, Hk, lk, sms)
        out = torch.empty_like(q)
        lse = torch.empty((H, batch), dtype=torch.float32, device=dev)
        ws = fa_varlen.new_workspace(int(fa_varlen.lib.fa_varlen_fwd_splitkv_workspace_size(batch, batch, H, Hk, D,
                                                                                           splits)), dev)
        call = lambda: fa_varlen.fa_varlen_fwd_splitkv(q, k, v, cu_q, 1, lk, w.scale, True, splits, cu_seqlens_k=cu_k,
                                                       out=out, softmax_lse=lse, workspace=ws, stream=stream)
        for _ in range(3):
            call()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(iters):
            call()
        b.record(stream)
        torch.cuda.synchronize(dev)
        if fa_varlen.device_status(ws) != 0:
            raise RuntimeError("device status not OK after the decode calls")
        ms = a.elapsed_time(b) / iters
        kv_bytes = 2 * batch * lk * Hk * D * 2
        gbs = kv_bytes / (ms * 1e-3) / 1e9
        res[f"decode {batch} seqs x {lk} keys, h32 kv8 d128, 1 query token, {splits} splits"] = {
            "ms": ms, "kv_gbytes": kv_bytes / 1e9, "gbs": gbs, "pct_of_hbm_peak": 100 * gbs / hbm_peak_gbs,
            "timing": f"{iters} calls back to back, no L2 flush (K/V {kv_bytes / 2**20:.0f} MiB > 126 MB L2)"}
        del q, k, v, out, lse, ws
    return res


def fwd_only(args):
    """--fwd-only N[:D]: the forward of standard workload N alone, for
    profiling captures (the same seeded inputs as the forward lines of the
    full run)."""
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    n, _, d = args.fwd_only.partition(":")
    w = synth.standard_workload(int(n), head_dim=int(d) if d else None)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    t = w.tensors()
    q, k, v = (torch.from_numpy(t[x].view(np.int16)).view(torch.bfloat16).to(dev) for x in ("q", "k", "v"))
    cq, ck = torch.from_numpy(w.cu_q).to(dev), torch.from_numpy(w.cu_k).to(dev)
    call = lambda: fa_varlen.fa_varlen_fwd(q, k, v, cq, ck, w.max_seqlen_q, w.max_seqlen_k, w.scale, w.causal,
                                           stream=stream)
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        call()
    b.record(stream)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b) / args.steps
    return {"mode": "fwd-only", "workload": w.name, "calls": args.steps, "ms_per_call": ms,
            "tflops": fwd_flops(w.cu_q, w.cu_k, w.heads, w.head_dim, w.causal) / (ms * 1e-3) / 1e12}


def decode_only(args):
    """--decode BATCHxKEYS: the split-KV decode call of that shape alone, for
    profiling captures (the same seeded inputs and split count as the decode
    lines of the full run)."""
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    batch, lk = (int(x) for x in args.decode.lower().split("x"))
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    w = synth.decode_workload(batch, lk)
    H, Hk, D = w.heads, w.kv_heads, w.head_dim
    t = w.tensors()
    q, k, v = (torch.from_numpy(t[n].view(np.int16)).view(torch.bfloat16).to(dev) for n in ("q", "k", "v"))
    cu_q = torch.from_numpy(w.cu_q).to(dev)
    cu_k = torch.from_numpy(w.cu_k).to(dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    splits = fa_varlen.fa_varlen_splitkv_num_splits(batch, 1, H, Hk, lk, sms)
    out = torch.empty_like(q)
    lse = torch.empty((H, batch), dtype=torch.float32, device=dev)
    ws = fa_varlen.new_workspace(int(fa_varlen.lib.fa_varlen_fwd_splitkv_workspace_size(batch, batch, H, Hk, D, splits)),
                                 dev)
    call = lambda: fa_varlen.fa_varlen_fwd_splitkv(q, k, v, cu_q, 1, lk, w.scale, True, splits, cu_seqlens_k=cu_k,
                                                   out=out, softmax_lse=lse, workspace=ws, stream=stream)
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        call()
    b.record(stream)
    torch.cuda.synchronize(dev)
    if fa_varlen.device_status(ws) != 0:
        raise RuntimeError("device status not OK after the decode calls")
    ms = a.elapsed_time(b) / args.steps
    kv_bytes = 2 * batch * lk * Hk * D * 2
    return {"mode": "decode", "workload": f"{batch} seqs x {lk} keys, h32 kv8 d128, 1 query token", "splits": splits,
            "calls": args.steps, "ms_per_call": ms, "kv_gbs": kv_bytes / (ms * 1e-3) / 1e9}


# ------------------------------------------------------------- oracle (CPU)
def oracle_sample(w, budget_s: float, seed: int = 0):
    """Pick (sequence, head) units of ``w`` whose oracle fwd+bwd takes about
    ``budget_s`` on this host. The oracle runs one unit per thread, so the
    estimate is max(total work / cores, largest unit) at the single-thread
    rate measured on a first batch of one unit per core."""
    import oracle

    t = w.tensors()
    cores = oracle.num_threads()
    lens = np.diff(w.cu_q)
    shortest = int(np.argmin(lens))
    calib = [(shortest, h % w.heads) for h in range(max(cores, 1))]
    t0 = time.perf_counter()
    oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, w.causal, units=calib)
    oracle.bwd(t["q"], t["k"], t["v"], t["dout"], w.cu_q, w.cu_k, w.scale, w.causal, units=calib)
    dt = time.perf_counter() - t0
    unit_f = lambda u: 3.5 * fwd_flops(w.cu_q, w.cu_k, w.heads, w.head_dim, w.causal, [u])
    r1 = unit_f(calib[0]) / max(dt, 1e-6)  # one thread's rate
    units = [(b, h) for b in range(w.batch) for h in range(w.heads)]
    random.Random(seed).shuffle(units)
    pick, total, biggest = [], 0.0, 0.0
    for u in units:
        f = unit_f(u)
        est = max((total + f) / (cores * r1), max(biggest, f) / r1)
        if est > budget_s:
            continue
        pick.append(u)
        total += f
        biggest = max(biggest, f)
    if not pick:
        pick = calib
    return pick, cores


def time_oracle(w, units):
    import oracle

    t = w.tensors()
    t0 = time.perf_counter()
    oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, w.causal, units=units)
    oracle.bwd(t["q"], t["k"], t["v"], t["dout"], w.cu_q, w.cu_k, w.scale, w.causal, units=units)
    dt = time.perf_counter() - t0
    fl = 3.5 * fwd_flops(w.cu_q, w.cu_k, w.heads, w.head_dim, w.causal, units)
    return fl / dt / 1e12, dt, fl


def describe_sample(w, units):
    seqs = sorted({b for b, _ in units})
    return (f"{len(units)} (sequence, head) units of the workload (sequences {seqs[:8]}{'...' if len(seqs) > 8 else ''}, "
            f"lengths {[int(np.diff(w.cu_q)[b]) for b in seqs[:8]]}), fp64 fwd+bwd, value scaled by the sample's "
            f"3.5*F_fwd FLOPs")


def cpu_baseline(w, budget_s=15.0):
    units, cores = oracle_sample(w, budget_s)
    tf, dt, _ = time_oracle(w, units)
    return {"value": tf, "unit": UNIT, "cores": cores, "kind": "oracle", "seconds": dt,
            "sample": describe_sample(w, units)}


def run_reference(args):
    """The oracle as it stands, on bounded samples of the same workload."""
    w = synth.standard_workload(5)
    per_step = max(1.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    units, cores = oracle_sample(w, per_step)
    for _ in range(args.warmup):
        time_oracle(w, units)
    times, flops = [], 0.0
    for _ in range(args.steps):
        _, dt, fl = time_oracle(w, units)
        times.append(dt)
        flops = fl
    ms = 1e3 * statistics.mean(times)
    value = flops / (ms * 1e-3) / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded bf16 N(0,1) inputs, widened exactly)",
        "config": {"workload": WORKLOAD, "total_tokens": w.total_q, "heads": w.heads, "head_dim": w.head_dim,
                   "causal": True},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": describe_sample(w, units)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def summary(r):
    """The line's key figures again, compact, at its end: headline, forward
    and backward of the headline workload, each other workload's % of peak."""
    pct = lambda x: round(x, 1)
    out = {"fwd_bwd_tflops": round(r["value"], 1), "pct_of_peak": {k: pct(v) for k, v in r["pct_of_peak"].items()
                                                                   if k != "denominator"},
           "kernel_ms": {k: round(v, 4) for k, v in r["kernel_ms"].items()},
           "bwd_kernel_frac": round(r["roofline"]["frac"], 4)}
    if "fwd_by_workload" in r:
        out["fwd_pct_by_workload"] = {k: pct(v["pct_of_peak"]) for k, v in r["fwd_by_workload"].items()}
    if "bwd_by_workload" in r:
        out["bwd_pct_by_workload"] = {k: pct(v["bwd_pct_of_peak"]) for k, v in r["bwd_by_workload"].items()}
    if "decode_by_workload" in r:
        out["decode_pct_of_hbm"] = {k: pct(v["pct_of_hbm_peak"]) for k, v in r["decode_by_workload"].items()}
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-aux", action="store_true", help="skip the forward-only workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--split", choices=("replicas", "heads", "sequences"), default="replicas",
                    help="N > 1: replicas = every rank runs the whole workload on its own data (weak scaling); "
                         "heads = one workload, its heads split across the ranks; sequences = one workload, its "
                         "sequences split across the ranks balanced by lq*lk (strong scaling)")
    ap.add_argument("--tokens", type=int, default=synth.TOTAL_TOKENS,
                    help="total tokens of the workload (default 16384; smaller only for profiling captures)")
    ap.add_argument("--fwd-only", metavar="N[:D]",
                    help="profiling mode, one GPU: only the forward of standard workload N (1-5) at head_dim D, "
                         "--warmup untimed and --steps timed calls")
    ap.add_argument("--decode", metavar="BATCHxKEYS",
                    help="profiling mode, one GPU: only the split-KV decode call of that shape (one query token, "
                         "32 query heads over 8 key/value heads, d=128), --warmup untimed and --steps timed calls")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            sys.exit("--gpus N > 1 must be launched with torchrun (one process per GPU)")

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if args.decode:
        if world != 1:
            sys.exit("--decode runs on one GPU")
        print(json.dumps(decode_only(args)), flush=True)
        return
    if args.fwd_only:
        if world != 1:
            sys.exit("--fwd-only runs on one GPU")
        print(json.dumps(fwd_only(args)), flush=True)
        return

    import torch

    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        result, w = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                result["cpu_baseline"] = cpu_baseline(w)
            result["summary"] = summary(result)
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
