#!/usr/bin/env python
"""Decode-step benchmark of the B200 quantized KV cache.

One step = one pass of the whole decode hot path for one layer: quantize and
append the new token's K and V for every sequence, split-K decode attention
over the quantized cache (dequantized in registers), and the log-sum-exp
combine.  After each step the cache is rolled back one token (host
bookkeeping), so every timed step decodes at the same context length.

Default workload: GQA 8 KV / 32 query heads, head_dim 128, batch 8, 32K
context, NVFP4 KV (K with per-channel lognormal scales and 2 % outlier
channels), one layer timed.  Inputs are seeded and synthetic (no model or
dataset), generated on the host and resident in HBM before timing starts.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

Prints one JSON line (rank 0).  Under torchrun each rank runs its own copy of
the workload (its own batch of sequences; no collective on the data path)
and the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_kv_cache_13_b200 import workloads as W  # noqa: E402

FMT_NAMES = {W.NVFP4: "nvfp4", W.INT4: "int4", W.FP8: "fp8", W.INT8: "int8", W.INT2: "int2"}
DTYPE = {W.NVFP4: "e2m1+e4m3 codes, f16 mma, f32 accumulate",
         W.INT4: "u4 affine codes, f16 mma, f32 accumulate",
         W.INT8: "u8 affine codes, f16 mma, f32 accumulate",
         W.INT2: "u2 affine codes, f16 mma, f32 accumulate",
         W.FP8: "e4m3 codes, f16 mma, f32 accumulate"}


def token_bytes(w: W.Workload) -> int:
    """Cache bytes one token of one KV head occupies, K plus V."""
    if w.fmt == W.NVFP4:
        return 2 * (w.head_dim // 2 + w.head_dim // 16)
    if w.fmt == W.INT4:
        if w.compact_meta:   # {f16 S0, f16 S1, i8 Z0, i8 Z1, 2 zero bytes} per token
            return 2 * (w.head_dim // 2 + 8)
        return 2 * (w.head_dim // 2 + 8 * (w.head_dim // w.group_size))
    if w.fmt == W.INT8:
        return 2 * (w.head_dim + 8 * (w.head_dim // w.group_size))
    if w.fmt == W.INT2:
        return 2 * (w.head_dim // 4 + 8 * (w.head_dim // w.group_size))
    return 2 * w.head_dim


def decode_bytes(w: W.Workload, L_main: int, L_ring: int) -> int:
    """Algorithmic HBM bytes of one decode-attention call: the quantized cache
    (codes + scales), the BF16 ring tokens, Q (bf16) and O (f32)."""
    return (w.units * (L_main * token_bytes(w) + L_ring * 2 * w.head_dim * 2)
            + w.batch * w.q_heads * w.head_dim * (2 + 4))


def append_bytes(w: W.Workload, n: int) -> int:
    """BF16 in + codes/scales out for appending n tokens per sequence."""
    return w.units * n * (2 * w.head_dim * 2 + token_bytes(w))


def step_bytes(w: W.Workload, L_main: int, L_ring: int) -> int:
    """Algorithmic HBM bytes of one fused decode step: the attention over the
    cache that already holds the new token, plus reading the new token's K/V
    (bf16) and writing it (quantized into the cache, or bf16 into the ring)."""
    write = 2 * w.head_dim * 2 if w.residual_length else token_bytes(w)
    return decode_bytes(w, L_main, L_ring) + w.units * (2 * w.head_dim * 2 + write)


# --------------------------------------------------------------------------
# DRAM traffic of the attention kernel from the committed ncu capture
# --------------------------------------------------------------------------

KERNEL_SOURCES = ["quantized_kv_cache_13_b200/csrc/kvq_attn.cu",
                  "quantized_kv_cache_13_b200/csrc/kvq_device.cuh",
                  "quantized_kv_cache_13_b200/csrc/kvq_encode.cuh",
                  "quantized_kv_cache_13_b200/csrc/kvq_internal.h"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_attn_traffic.json")


def kernel_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic(workload: str):
    """dram read+write bytes per launch measured by ncu for this workload, or
    None when there is no capture or the kernel source changed since."""
    try:
        rec = json.load(open(TRAFFIC_FILE))
    except Exception:
        return None
    entry = rec.get("workloads", {}).get(workload)
    if not entry or rec.get("kernel_sha256") != kernel_source_hash():
        return None
    return entry.get("dram_bytes_per_launch")


def traffic_note(workload: str) -> str:
    """Where roofline.traffic comes from, or why it is null."""
    try:
        rec = json.load(open(TRAFFIC_FILE))
    except Exception:
        return "no ncu capture committed"
    if workload not in rec.get("workloads", {}):
        return "no ncu capture of this workload"
    if rec.get("kernel_sha256") != kernel_source_hash():
        return ("null: the kernel sources changed after the committed ncu capture "
                "(profiles/decode_attn_traffic.json)")
    return "ncu capture of the current kernel sources (profiles/decode_attn_traffic.json)"


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.samples = []
        self.proc = None
        self.dev = device_index
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)

    def summary(self, t0: float, t1: float):
        rows = []
        for t, line in self.samples:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            rows.append((t, parts))
        inside = [p for t, p in rows if t0 <= t <= t1]
        note = None
        if not inside and rows:
            # timed window shorter than the sampling interval: nearest samples
            rows.sort(key=lambda x: min(abs(x[0] - t0), abs(x[0] - t1)))
            inside = [p for _, p in rows[:3]]
            note = "timed window shorter than the 50 ms sampling interval; nearest samples"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(p[1]) for p in inside if num(p[1]) is not None]
        smax = [num(p[2]) for p in inside if num(p[2]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for p in inside:
            for name, v in zip(names, p[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        out = {"sm_mhz": float(np.median(sm)) if sm else None,
               "sm_max_mhz": max(smax) if smax else None,
               "reasons": sorted(reasons), "samples": len(inside)}
        if note:
            out["note"] = note
        return out


# --------------------------------------------------------------------------
# distributed plumbing (one process per GPU; timing only, no data exchange)
# --------------------------------------------------------------------------

def dist_init(backend: str = "nccl"):
    """One process per GPU, ranks from the torchrun environment."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300), **kw)
    return world, rank, local


def dist_max(x: float, world: int) -> float:
    """Max of a per-rank scalar over all ranks (timing only)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def weak_scaling_value(ms_step_local: float, batch: int, world: int):
    """Whole-job decode tokens/s: every rank decodes `batch` sequences per
    step (replicas, no exchange); the step time is the slowest rank's."""
    ms = dist_max(ms_step_local, world)
    return ms, batch * world / (ms * 1e-3)


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------

def staged_inputs(tensors, pinned: bool):
    """One flat host buffer holding `tensors` (same dtype) back to back, and
    the element offset of each.  Every piece starts on a 16-byte boundary
    (the library's alignment rule for its inputs)."""
    import torch
    offs, n = [], 0
    for t in tensors:
        assert (n * t.element_size()) % 16 == 0, "staged piece not 16-byte aligned"
        offs.append(n)
        n += t.numel()
    buf = torch.empty(n, dtype=tensors[0].dtype)
    if pinned:
        buf = buf.pin_memory()
    for t, o in zip(tensors, offs):
        buf[o:o + t.numel()].copy_(t.reshape(-1).cpu())
    return buf, offs


def staged_views(buf, tensors):
    """Views of a staging buffer laid out by staged_inputs, shaped like `tensors`."""
    views, o = [], 0
    for t in tensors:
        views.append(buf[o:o + t.numel()].view(t.shape))
        o += t.numel()
    return views


def upload_prefill(w: W.Workload, which: str, torch):
    """[B, Hkv, context, D] bf16 on the GPU, generated slice by slice on the host."""
    t = torch.empty((w.batch, w.kv_heads, w.context, w.head_dim), dtype=torch.bfloat16, device="cuda")
    for b in range(w.batch):
        for h in range(w.kv_heads):
            x = W.kv_slice(w, which, b, h, 0, w.context)
            t[b, h].copy_(torch.from_numpy(x).to(torch.bfloat16))
    return t


def run_ours(args, world, rank, local):
    import torch
    import quantized_kv_cache_13_b200 as kvq

    kvq.load_library()
    w = W.WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    n_new = 1 + max(args.steps, args.warmup) + 4
    max_len = w.context + max(n_new, 2 * w.residual_length)
    grp = w.group_size if w.fmt in (W.INT4, W.INT8, W.INT2) else 0
    cache = kvq.KVCache(w.fmt, 1, w.batch, w.kv_heads, max_len, w.head_dim, grp, w.residual_length,
                        scale_renewal=w.scale_renewal, compact_meta=w.compact_meta)

    k_pre = upload_prefill(w, "k", torch)
    v_pre = upload_prefill(w, "v", torch)
    stream = torch.cuda.current_stream()

    # ---- prefill (bulk quantize-append with amax calibration), timed ----
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    cache.append(0, k_pre, v_pre)
    e1.record(stream)
    torch.cuda.synchronize()
    prefill_ms = e0.elapsed_time(e1)
    del k_pre, v_pre
    L0 = sum(cache.lengths(0))

    # ---- decode-step inputs, resident in HBM ----
    knew = torch.from_numpy(W.kv_tensor(w, "k", w.context, 1)).to(torch.bfloat16).cuda()
    vnew = torch.from_numpy(W.kv_tensor(w, "v", w.context, 1)).to(torch.bfloat16).cuda()
    q = torch.from_numpy(W.q_tensor(w)).to(torch.bfloat16).cuda()
    out = torch.empty((w.batch, w.q_heads, w.head_dim), dtype=torch.float32, device="cuda")
    ws = cache.workspace(w.q_heads)
    h = cache.handle

    L_main, L_ring = cache.lengths(0)
    if w.residual_length:
        # the decode token goes to the ring (no flush: context is a multiple of R)
        L_ring_step, L_main_step = L_ring + 1, L_main
    else:
        L_ring_step, L_main_step = 0, L_main + 1

    # one step = kvq_decode_step: append the new token and attend, one launch
    def step():
        kvq.kvq_decode_step(h, 0, knew, vnew, q, out, ws, 0.0, stream)
        kvq.kvq_truncate(h, 0, L0)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # The timed region launches exactly one kernel per step (kvq_truncate
    # only moves the host-side length back), so the events around it give
    # that kernel's mean launch duration, inter-launch gaps included.
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    dist_barrier(world)
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    wall0 = time.time()
    t_start.record(stream)
    for i in range(args.steps):
        kvq.kvq_decode_step(h, 0, knew, vnew, q, out, ws, 0.0, stream)
        kvq.kvq_truncate(h, 0, L0)
    t_end.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    dist_barrier(world)
    elapsed_ms = t_start.elapsed_time(t_end)
    att_ms = elapsed_ms / args.steps
    time.sleep(0.1)
    sampler.stop()
    clocks = sampler.summary(wall0, wall1)
    ms_step, value = weak_scaling_value(elapsed_ms / args.steps, w.batch, world)
    att_ms = dist_max(att_ms, world)
    status = cache.device_status()

    # the same attention as a separate call (cache already holding the token)
    kvq.kvq_append(h, 0, knew, vnew, stream)
    for _ in range(args.warmup):
        kvq.kvq_decode_attention(h, 0, q, out, ws, 0.0, stream)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_sep = min(args.steps, 500)
    a0.record(stream)
    for _ in range(n_sep):
        kvq.kvq_decode_attention(h, 0, q, out, ws, 0.0, stream)
    a1.record(stream)
    torch.cuda.synchronize()
    attn_only_ms = a0.elapsed_time(a1) / n_sep
    kvq.kvq_truncate(h, 0, L0)

    # the separate single-token append (launch-latency bound; the fused step
    # does this inside the attention launch)
    for _ in range(args.warmup):
        kvq.kvq_append(h, 0, knew, vnew, stream)
        kvq.kvq_truncate(h, 0, L0)
    a0.record(stream)
    for _ in range(n_sep):
        kvq.kvq_append(h, 0, knew, vnew, stream)
        kvq.kvq_truncate(h, 0, L0)
    a1.record(stream)
    torch.cuda.synchronize()
    append1_ms = a0.elapsed_time(a1) / n_sep

    # ---- end to end through the public API with host buffers ----
    # The step's inputs (the new token's K and V, and q) sit back to back in
    # one pinned host buffer, so a step makes one host-to-device copy and one
    # device-to-host copy of the output.
    stage_h, _ = staged_inputs([knew, vnew, q], pinned=True)
    stage_d = torch.empty(stage_h.shape, dtype=stage_h.dtype, device=dev)
    kd, vd, qd = staged_views(stage_d, [knew, vnew, q])
    out_h = torch.empty(out.shape, dtype=torch.float32).pin_memory()

    def e2e_step():
        stage_d.copy_(stage_h, non_blocking=True)
        kvq.kvq_decode_step(h, 0, kd, vd, qd, out, ws, 0.0, stream)
        out_h.copy_(out, non_blocking=True)
        kvq.kvq_truncate(h, 0, L0)

    for _ in range(args.warmup):
        e2e_step()
    dist_barrier(world)
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    s1.record(stream)
    torch.cuda.synchronize()
    dist_barrier(world)
    e2e_ms = dist_max(s0.elapsed_time(s1) / args.steps, world)
    h2d = knew.numel() * 2 + vnew.numel() * 2 + q.numel() * 2
    d2h = out.numel() * 4

    # ---- residual ring (INT formats): attention at ring occupancy 1, 64, R-1, and the flush ----
    ring_extra = None
    if w.residual_length:
        R = w.residual_length
        kr = torch.from_numpy(W.kv_tensor(w, "k", w.context, R - 1)).to(torch.bfloat16).cuda()
        vr = torch.from_numpy(W.kv_tensor(w, "v", w.context, R - 1)).to(torch.bfloat16).cuda()

        def loop_ms(fn, n):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(n):
                fn()
            b.record(stream)
            torch.cuda.synchronize()
            return a.elapsed_time(b) / n

        occ = {}
        for r in sorted({1, min(64, R - 1), R - 1}):
            kvq.kvq_truncate(h, 0, L0)
            kvq.kvq_append(h, 0, kr[:, :, :r].contiguous(), vr[:, :, :r].contiguous(), stream)
            occ[str(r)] = round(1e3 * loop_ms(lambda: kvq.kvq_decode_attention(h, 0, q, out, ws, 0.0, stream), 200), 2)
        kvq.kvq_truncate(h, 0, L0)

        def fill():
            kvq.kvq_append(h, 0, kr, vr, stream)
            kvq.kvq_truncate(h, 0, L0)

        def fill_flush():
            kvq.kvq_append(h, 0, kr, vr, stream)
            kvq.kvq_flush_residual(h, 0, stream)
            kvq.kvq_truncate(h, 0, L0)

        t_fill = loop_ms(fill, 100)
        t_flush = loop_ms(fill_flush, 100) - t_fill
        ring_extra = {"attention_us_at_ring_occupancy": occ,
                      "flush_us_%d_tokens" % (R - 1): round(1e3 * t_flush, 2),
                      "flush_note": "quantize of the ring into the main cache, timed as (ring append + flush) minus (ring append)"}
        status = status or cache.device_status()

    # ---- roofline of the decode-attention call ----
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        pass
    peak = peaks.get("hbm_gbs")
    peak_note = "of measured"
    if not peak:
        peak, peak_note = 6650.0, "of fallback"
    bytes_call = step_bytes(w, L_main_step, L_ring_step)
    achieved = bytes_call / (att_ms * 1e-3) / 1e9

    tokens_per_step = w.batch * world
    res = {
        "metric": "decode-attention tokens/s (one layer, B sequences per step) and achieved HBM GB/s per cache format",
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": DTYPE[w.fmt],
        "data": "synthetic (seeded numpy, BF16), no model or dataset",
        "config": {"workload": w.name, "format": FMT_NAMES[w.fmt], "batch": w.batch,
                   "kv_heads": w.kv_heads, "q_heads": w.q_heads, "head_dim": w.head_dim,
                   "context": L_main_step + L_ring_step, "group_size": w.group_size,
                   "residual_length": w.residual_length, "layers_timed": 1,
                   "parallelism": "replicas (dp%d), no collective on the data path" % world,
                   "l2": "inputs larger than L2 (cache %.0f MB > 126 MB)" % (bytes_call / 1e6)},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": recorded_traffic(w.name),
                     "traffic_source": traffic_note(w.name),
                     "kernel": "decode step: fused append + split-K attention + combine (one kvq_decode_step launch)",
                     "bytes_per_launch": bytes_call, "launch_ms": round(att_ms, 5),
                     "peak_source": peak_note},
        "e2e": {"value": round(tokens_per_step / (e2e_ms * 1e-3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps,   # one fused kernel per step
        "clocks": clocks,
        "extra": {"model_tokens_per_s_32_layers": round(value / 32, 1),
                  "attention_only_ms": round(attn_only_ms, 5),
                  "append_1_token_us": round(1e3 * append1_ms, 2),
                  "attention_only_gbs": round(decode_bytes(w, L_main_step, L_ring_step) / (attn_only_ms * 1e-3) / 1e9, 1),
                  "kv_tokens_per_s": round(value * (L_main_step + L_ring_step), 1),
                  "prefill_append_ms": round(prefill_ms, 3),
                  "prefill_append_tokens_per_s": round(w.batch * w.context / (prefill_ms * 1e-3), 1),
                  "prefill_append_gbs": round(append_bytes(w, w.context) / (prefill_ms * 1e-3) / 1e9, 1),
                  "device_status": status},
    }
    if ring_extra:
        res["extra"]["residual_ring"] = ring_extra
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = cpu_baseline(w, args.cpu_units, L_main_step + L_ring_step)
    return res


# --------------------------------------------------------------------------
# the oracle, timed on the host cores (CPU baseline / reference arm)
# --------------------------------------------------------------------------

def oracle_decode_sample(w: W.Workload, units, ctx: int):
    """Oracle decode step for the given (b, kvh) units at context `ctx`:
    quantize the unit's tokens, then decode attention for its G query heads.
    Returns seconds spent in the timed part (the decode step: quantize the
    new token + dequantize + attention)."""
    import oracle
    q_all = W.q_tensor(w)
    G = w.G
    t_total = 0.0
    for (b, h) in units:
        k = W.kv_slice(w, "k", b, h, 0, ctx)
        v = W.kv_slice(w, "v", b, h, 0, ctx)
        if w.compact_meta or w.scale_renewal or (w.residual_length and w.fmt in (W.NVFP4, W.FP8)):
            # cache options: the oracle's cache of this unit (prefill untimed;
            # the step = append the new token, dequantize, attend)
            oc = oracle.OracleCache(w.fmt, 1, 1, 1, w.head_dim, ctx,
                                    w.group_size if w.fmt in (W.INT4, W.INT8, W.INT2) else 0,
                                    w.residual_length, recalibrate_every=w.scale_renewal,
                                    compact=w.compact_meta)
            oc.append(0, k[None, None, :-1], v[None, None, :-1])
            t0 = time.perf_counter()
            oc.append(0, k[None, None, -1:], v[None, None, -1:])
            oc.decode_attention(0, q_all[b, h * G:(h + 1) * G][None])
            t_total += time.perf_counter() - t0
            continue
        if w.fmt in (W.INT4, W.INT8, W.INT2):
            gk = gv = None
        else:
            gk = oracle.global_scale(w.fmt, oracle.amax(k[:w.context]))
            gv = oracle.global_scale(w.fmt, oracle.amax(v[:w.context]))
        # prefill codes (not timed: the cache already holds them on the GPU side too)
        if w.fmt == W.NVFP4:
            ck, cv = oracle.nvfp4_quantize(k[:-1], gk), oracle.nvfp4_quantize(v[:-1], gv)
        elif w.fmt == W.FP8:
            ck, cv = (oracle.fp8_quantize(k[:-1], gk),), (oracle.fp8_quantize(v[:-1], gv),)
        elif w.fmt == W.INT8:
            ck, cv = oracle.int8_quantize(k[:-1], w.group_size), oracle.int8_quantize(v[:-1], w.group_size)
        elif w.fmt == W.INT2:
            ck, cv = oracle.int2_quantize(k[:-1], w.group_size), oracle.int2_quantize(v[:-1], w.group_size)
        else:
            ck, cv = oracle.int4_quantize(k[:-1], w.group_size), oracle.int4_quantize(v[:-1], w.group_size)
        t0 = time.perf_counter()
        # the step: quantize-append the new token, dequantize, attend
        if w.fmt in (W.INT4, W.INT8, W.INT2) and w.residual_length:
            K = np.concatenate([oracle.dequantize_arrays(w.fmt, ck, None, w.group_size), k[-1:]], 0)
            V = np.concatenate([oracle.dequantize_arrays(w.fmt, cv, None, w.group_size), v[-1:]], 0)
        else:
            if w.fmt == W.NVFP4:
                nk, nv = oracle.nvfp4_quantize(k[-1:], gk), oracle.nvfp4_quantize(v[-1:], gv)
            elif w.fmt == W.FP8:
                nk, nv = (oracle.fp8_quantize(k[-1:], gk),), (oracle.fp8_quantize(v[-1:], gv),)
            elif w.fmt == W.INT8:
                nk, nv = oracle.int8_quantize(k[-1:], w.group_size), oracle.int8_quantize(v[-1:], w.group_size)
            elif w.fmt == W.INT2:
                nk, nv = oracle.int2_quantize(k[-1:], w.group_size), oracle.int2_quantize(v[-1:], w.group_size)
            else:
                nk, nv = oracle.int4_quantize(k[-1:], w.group_size), oracle.int4_quantize(v[-1:], w.group_size)
            ck = tuple(np.concatenate([a, b_], 0) for a, b_ in zip(ck, nk))
            cv = tuple(np.concatenate([a, b_], 0) for a, b_ in zip(cv, nv))
            K = oracle.dequantize_arrays(w.fmt, ck, gk, w.group_size)
            V = oracle.dequantize_arrays(w.fmt, cv, gv, w.group_size)
        oracle.attention(q_all[b, h * G:(h + 1) * G], K, V)
        t_total += time.perf_counter() - t0
    return t_total


def _oracle_unit_worker(job):
    """One (batch, kv-head) unit's oracle decode step in a worker process."""
    name, unit, ctx = job
    return oracle_decode_sample(W.WORKLOADS[name], [unit], ctx)


def cpu_baseline(w: W.Workload, n_units: int, ctx: int):
    units = [(u // w.kv_heads, u % w.kv_heads) for u in range(min(n_units, w.units))]
    secs = oracle_decode_sample(w, units, ctx)
    per_step = secs / len(units) * w.units
    res = {"value": round(w.batch / per_step, 4), "unit": "tokens/s", "cores": 1, "kind": "oracle",
           "sample": "%d of %d (batch, kv-head) units at context %d, one decode step each "
                     "(quantize new token, dequantize cache, fp64 attention), scaled to the full "
                     "batch; single-threaded C oracle" % (len(units), w.units, ctx),
           "seconds": round(secs, 3)}
    # The same oracle on the host cores: one unit per worker process (spawned,
    # so no CUDA state is inherited), all workers at once; at most 16 workers
    # (each imports numpy and torch).
    try:
        import multiprocessing as mp
        cores = len(os.sched_getaffinity(0))
        n = min(cores, w.units, 16)
        if n > 1:
            every = [(u // w.kv_heads, u % w.kv_heads) for u in range(n)]
            with mp.get_context("spawn").Pool(n) as pool:
                per_unit = pool.map(_oracle_unit_worker, [(w.name, u, ctx) for u in every], chunksize=1)
            wall = max(per_unit)   # the units ran concurrently, one per core
            res["all_cores"] = {"value": round(w.batch / (wall * w.units / n), 4), "cores": n,
                                "sample": "%d units at once, one per process; value = the full batch at "
                                          "the slowest unit's time x %d/%d" % (n, w.units, n)}
    except Exception as e:   # report, do not fail the bench line
        res["all_cores"] = {"error": str(e)[:200]}
    return res


def run_reference(args, world, rank):
    """Reference arm: the oracle, timed as it stands, on this workload."""
    if rank != 0:
        return None
    w = W.WORKLOADS[args.workload]
    ctx = w.context + 1
    units = [(0, 0)]
    for _ in range(args.warmup):
        pass   # the oracle has no warm-up state; warm-up steps are not timed
    per_steps = []
    for i in range(args.steps):
        u = [((i // w.kv_heads) % w.batch, i % w.kv_heads)]
        per_steps.append(oracle_decode_sample(w, u, ctx) * w.units)
    ms_step = 1e3 * float(np.mean(per_steps))
    value = w.batch / (ms_step * 1e-3)
    return {
        "impl": "reference",
        "metric": "decode-attention tokens/s (one layer, B sequences per step) and achieved HBM GB/s per cache format",
        "value": round(value, 4), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32 encode, f64 attention",
        "data": "synthetic (seeded numpy, BF16), no model or dataset",
        "config": {"workload": w.name, "format": FMT_NAMES[w.fmt], "batch": w.batch,
                   "kv_heads": w.kv_heads, "q_heads": w.q_heads, "head_dim": w.head_dim,
                   "context": ctx},
        "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": "each step: one (batch, kv-head) unit of %d at context %d, "
                                   "scaled to the full batch" % (w.units, ctx)},
        "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="gqa_nvfp4_32k", choices=sorted(W.WORKLOADS))
    ap.add_argument("--cpu-units", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    args.steps = max(args.steps, 1)

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
        res = run_reference(args, world, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    world, rank, local = dist_init()
    res = run_ours(args, world, rank, local)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
