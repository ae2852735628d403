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


METRIC = ("decode-attention tokens/s (one layer, B sequences per step) and achieved HBM GB/s "
          "per cache format")


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

    # NVML clocks-event reason bits reported as the recipe's reason names
    NVML_REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
                    ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))

    def __init__(self, device_index: int):
        self.samples = []
        self.fast = []            # (time, sm MHz, max sm MHz, reason bits) read through NVML
        self.proc = None
        self.dev = device_index
        self.thread = None
        self.fast_thread = None
        self.fast_stop = threading.Event()

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
        # a timed window of a millisecond or two falls between nvidia-smi's
        # 50 ms samples: NVML is read every 0.5 ms as well (reads only)
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.dev)
            self.fast_thread = threading.Thread(target=self._read_nvml, args=(pynvml, h), daemon=True)
            self.fast_thread.start()
        except Exception:
            self.fast_thread = None

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def _read_nvml(self, nv, h):
        reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        try:
            smax = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            while not self.fast_stop.is_set():
                t = time.time()
                self.fast.append((t, float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)), smax,
                                  int(reasons(h))))
                time.sleep(0.0005)
        except Exception:
            pass
        finally:
            try:
                nv.nvmlShutdown()
            except Exception:
                pass

    def stop(self):
        self.fast_stop.set()
        if self.fast_thread:
            self.fast_thread.join(timeout=2)
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
        fast = [f for f in self.fast if t0 <= f[0] <= t1]
        note = None
        if fast:
            reasons = set(name for f in fast for name, bit in self.NVML_REASONS if f[3] & bit)
            for p in inside:
                for name, v in zip([n for n, _ in self.NVML_REASONS], p[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(name)
            return {"sm_mhz": float(np.median([f[1] for f in fast])),
                    "sm_max_mhz": max(f[2] for f in fast), "reasons": sorted(reasons),
                    "samples": len(fast) + len(inside),
                    "source": "NVML every 0.5 ms and nvidia-smi every 50 ms, inside the timed window"}
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
    """[B, Hkv, context, D] bf16 on the GPU, generated slice by slice on the
    host (every slice has its own seeded generator, so the slices are drawn
    on several threads at once; the values do not depend on the order)."""
    from concurrent.futures import ThreadPoolExecutor
    t = torch.empty((w.batch, w.kv_heads, w.context, w.head_dim), dtype=torch.bfloat16, device="cuda")
    jobs = [(b, h) for b in range(w.batch) for h in range(w.kv_heads)]

    def one(bh):
        b, h = bh
        return bh, torch.from_numpy(W.kv_slice(w, which, b, h, 0, w.context)).to(torch.bfloat16)

    workers = max(1, min(16, len(os.sched_getaffinity(0))))
    with ThreadPoolExecutor(workers) as ex:
        for (b, h), x in ex.map(one, jobs):
            t[b, h].copy_(x)
    return t


# Workloads timed besides the headline one on a 1-GPU run, one per cache
# format and shape the metric covers (the headline itself is gqa_nvfp4_32k).
PER_WORKLOAD = ["long_nvfp4_128k", "gqa_fp8_32k", "gqa_nvfp4_32k_b16", "mha_int4_16k",
                "mha_int8_16k", "mha_int2_16k"]


def hbm_peak():
    """(GB/s, note): the measured copy bandwidth of this machine's B200s, else
    the fallback figure."""
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        if peaks.get("hbm_gbs"):
            return float(peaks["hbm_gbs"]), "of measured"
    except Exception:
        pass
    return 6650.0, "of fallback"


def step_lengths(w: W.Workload):
    """(main, ring) token counts a timed decode step attends over: the prefill
    plus the step's own token, which goes to the ring when there is one (the
    prefill length is a multiple of the ring, so nothing is flushed)."""
    if w.residual_length:
        return (w.context // w.residual_length) * w.residual_length, w.context % w.residual_length + 1
    return w.context + 1, 0


def config_dict(w: W.Workload, world: int):
    """The `config` of a bench line (both arms print the same one)."""
    L_main, L_ring = step_lengths(w)
    nbytes = step_bytes(w, L_main, L_ring)
    return {"workload": w.name, "format": FMT_NAMES[w.fmt], "batch": w.batch,
            "kv_heads": w.kv_heads, "q_heads": w.q_heads, "head_dim": w.head_dim,
            "context": L_main + L_ring, "group_size": w.group_size,
            "residual_length": w.residual_length, "layers_timed": 1,
            "parallelism": "replicas (dp%d), no collective on the data path" % world,
            "l2": ("inputs larger than L2 (cache %.0f MB > 126 MB)" % (nbytes / 1e6)
                   if nbytes > 126e6 else
                   "cache of %.2f MB fits in L2 (no flush between steps)" % (nbytes / 1e6))}


class DecodeBench:
    """One workload's cache after its timed prefill, with the decode-step
    inputs resident in HBM."""

    def __init__(self, w: W.Workload, n_new: int, local: int):
        import torch
        import quantized_kv_cache_13_b200 as kvq
        self.w, self.kvq, self.torch = w, kvq, torch
        self.dev = torch.device("cuda", local)
        max_len = w.context + max(n_new, 2 * w.residual_length)
        grp = w.group_size if w.fmt in (W.INT4, W.INT8, W.INT2) else 0
        self.cache = kvq.KVCache(w.fmt, 1, w.batch, w.kv_heads, max_len, w.head_dim, grp,
                                 w.residual_length, scale_renewal=w.scale_renewal,
                                 compact_meta=w.compact_meta)
        k_pre = upload_prefill(w, "k", torch)
        v_pre = upload_prefill(w, "v", torch)
        self.stream = torch.cuda.current_stream()
        # prefill: bulk quantize-append with amax calibration, timed on a
        # second pass (the first one includes the kernels' first launches)
        self.cache.append(0, k_pre, v_pre)
        self.cache.reset()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        self.cache.append(0, k_pre, v_pre)
        e1.record(self.stream)
        torch.cuda.synchronize()
        self.prefill_ms = e0.elapsed_time(e1)
        # the same prefill into a cache created with the calibrated scales
        # given (the pages' *_cast form: a constant per-tensor scale, no amax
        # pass), timed the same way
        self.cast_ms = None
        if w.fmt in (W.NVFP4, W.FP8) and not w.scale_renewal:
            gs = [[float(self.cache.raw(0, 0)["scale"][0]), float(self.cache.raw(0, 1)["scale"][0])]]
            cast = kvq.KVCache(w.fmt, 1, w.batch, w.kv_heads, max_len, w.head_dim, 0,
                               w.residual_length, gs)
            cast.append(0, k_pre, v_pre)
            cast.reset()
            torch.cuda.synchronize()
            e0.record(self.stream)
            cast.append(0, k_pre, v_pre)
            e1.record(self.stream)
            torch.cuda.synchronize()
            self.cast_ms = e0.elapsed_time(e1)
            del cast
        del k_pre, v_pre
        self.L0 = sum(self.cache.lengths(0))
        self.knew = torch.from_numpy(W.kv_tensor(w, "k", w.context, 1)).to(torch.bfloat16).cuda()
        self.vnew = torch.from_numpy(W.kv_tensor(w, "v", w.context, 1)).to(torch.bfloat16).cuda()
        self.q = torch.from_numpy(W.q_tensor(w)).to(torch.bfloat16).cuda()
        self.out = torch.empty((w.batch, w.q_heads, w.head_dim), dtype=torch.float32, device="cuda")
        self.ws = self.cache.workspace(w.q_heads)
        self.h = self.cache.handle
        L_main, L_ring = self.cache.lengths(0)
        if w.residual_length:
            # the decode token goes to the ring (no flush: context is a multiple of R)
            self.L_main_step, self.L_ring_step = L_main, L_ring + 1
        else:
            self.L_main_step, self.L_ring_step = L_main + 1, 0
        assert (self.L_main_step, self.L_ring_step) == step_lengths(w)

    def step(self):
        """One decode step = kvq_decode_step (append the new token and
        attend, one launch); the host then rolls the length back."""
        kvq = self.kvq
        kvq.kvq_decode_step(self.h, 0, self.knew, self.vnew, self.q, self.out, self.ws, 0.0, self.stream)
        kvq.kvq_truncate(self.h, 0, self.L0)

    def warm_up(self, steps: int) -> int:
        """`steps` untimed steps, run right before a timed region."""
        for _ in range(steps):
            self.step()
        self.torch.cuda.synchronize()
        return steps

    def time_steps(self, steps: int, world: int, sampler=None):
        """Mean device time of `steps` back-to-back steps (CUDA events on the
        launching stream, barrier + synchronize on both sides) and the wall
        window of the timed region."""
        torch = self.torch
        dist_barrier(world)
        torch.cuda.synchronize()
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        wall0 = time.time()
        t_start.record(self.stream)
        for _ in range(steps):
            self.step()
        t_end.record(self.stream)
        torch.cuda.synchronize()
        wall1 = time.time()
        dist_barrier(world)
        return t_start.elapsed_time(t_end) / steps, (wall0, wall1)

    def loop_ms(self, fn, n: int, warmup: int = 3) -> float:
        torch = self.torch
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(self.stream)
        for _ in range(n):
            fn()
        b.record(self.stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    def attention_only_ms(self, n: int) -> float:
        """The attention as a separate call over the cache that holds the token."""
        kvq = self.kvq
        kvq.kvq_append(self.h, 0, self.knew, self.vnew, self.stream)
        ms = self.loop_ms(lambda: kvq.kvq_decode_attention(self.h, 0, self.q, self.out, self.ws, 0.0,
                                                           self.stream), n)
        kvq.kvq_truncate(self.h, 0, self.L0)
        return ms

    def roofline(self, launch_ms: float):
        w = self.w
        peak, note = hbm_peak()
        nbytes = step_bytes(w, self.L_main_step, self.L_ring_step)
        achieved = nbytes / (launch_ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": recorded_traffic(w.name),
                "traffic_source": traffic_note(w.name),
                "kernel": "decode step: fused append + split-K attention + combine (one kvq_decode_step launch)",
                "bytes_per_launch": nbytes, "launch_ms": round(launch_ms, 5), "peak_source": note}

    def config(self, world: int):
        return config_dict(self.w, world)

    def prefill(self):
        w = self.w
        out = {"prefill_append_ms": round(self.prefill_ms, 3),
               "prefill_append_tokens_per_s": round(w.batch * w.context / (self.prefill_ms * 1e-3), 1),
               "prefill_append_gbs": round(append_bytes(w, w.context) / (self.prefill_ms * 1e-3) / 1e9, 1)}
        if w.fmt in (W.NVFP4, W.FP8) and not w.scale_renewal:
            # the calibrating prefill cannot form a code before the
            # per-tensor amax is known, so it must read its input twice
            # (amax pass, then the encode): the bytes it has to move
            moved = append_bytes(w, w.context) + w.units * w.context * 2 * w.head_dim * 2
            out["prefill_append_moved_gbs"] = round(moved / (self.prefill_ms * 1e-3) / 1e9, 1)
            out["prefill_append_moved_note"] = ("calibrating prefill: BF16 K and V read twice (amax, "
                                                "then encode) plus the codes and scales written")
        return {**out,
                **({} if self.cast_ms is None else {
                    "prefill_append_cast_ms": round(self.cast_ms, 3),
                    "prefill_append_cast_gbs": round(append_bytes(w, w.context) / (self.cast_ms * 1e-3) / 1e9, 1)})}


def per_workload_line(name: str, args, local: int):
    """ms per step, tokens/s, roofline and clocks of one more workload, timed
    like the headline (fused decode steps, CUDA events).  The timed loop runs
    at least `args.pw_min_ms` of device time so the clock samples cover it."""
    import torch
    w = W.WORKLOADS[name]
    n_new = 1 + max(args.steps, args.warmup) + 4
    bm = DecodeBench(w, n_new, local)
    for _ in range(args.warmup):
        bm.step()
    torch.cuda.synchronize()
    est, _ = bm.time_steps(max(3, args.warmup), 1)
    steps = max(args.steps, int(args.pw_min_ms / max(est, 1e-3)) + 1)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    bm.warm_up(args.warmup)
    ms, (w0, w1) = bm.time_steps(steps, 1)
    time.sleep(0.1)
    sampler.stop()
    attn_ms = bm.attention_only_ms(min(steps, 500))
    line = {"value": round(w.batch / (ms * 1e-3), 1), "unit": "tokens/s", "steps": steps,
            "ms_per_step": round(ms, 5), "roofline": bm.roofline(ms), "clocks": sampler.summary(w0, w1),
            "config": bm.config(1),
            "attention_only_ms": round(attn_ms, 5),
            "attention_only_gbs": round(decode_bytes(w, bm.L_main_step, bm.L_ring_step) / (attn_ms * 1e-3) / 1e9, 1),
            "device_status": bm.cache.device_status()}
    line.update(bm.prefill())
    del bm
    torch.cuda.empty_cache()
    return line


def selected_workload(args) -> W.Workload:
    """The workload to time; --context overrides its prefill length (small
    cases for profiling captures)."""
    import dataclasses
    w = W.WORKLOADS[args.workload]
    if args.context:
        w = dataclasses.replace(w, context=args.context)
    return w


def run_ours(args, world, rank, local):
    import torch
    import quantized_kv_cache_13_b200 as kvq

    kvq.load_library()
    w = selected_workload(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    n_new = 1 + max(args.steps, args.warmup) + 4
    bm = DecodeBench(w, n_new, local)
    h, stream = bm.h, bm.stream
    knew, vnew, q, out, ws, L0 = bm.knew, bm.vnew, bm.q, bm.out, bm.ws, bm.L0

    # The timed region launches exactly one kernel per step (kvq_truncate
    # only moves the host-side length back), so the events around it give
    # that kernel's mean launch duration, inter-launch gaps included.  The
    # W warm-up steps run right before it (after the clock sampler has
    # started), so the timed steps do not start on a GPU that has just been
    # idle.
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    bm.warm_up(args.warmup)
    step_ms, (wall0, wall1) = bm.time_steps(args.steps, world)
    time.sleep(0.1)
    sampler.stop()
    clocks = sampler.summary(wall0, wall1)
    ms_step, value = weak_scaling_value(step_ms, w.batch, world)
    att_ms = dist_max(step_ms, world)
    status = bm.cache.device_status()

    n_sep = min(args.steps, 500)
    attn_only_ms = bm.attention_only_ms(n_sep)

    # the separate single-token append (launch-latency bound; the fused step
    # does this inside the attention launch)
    def append1():
        kvq.kvq_append(h, 0, knew, vnew, stream)
        kvq.kvq_truncate(h, 0, L0)
    append1_ms = bm.loop_ms(append1, n_sep, args.warmup)

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
        occ = {}
        for r in sorted({1, min(64, R - 1), R - 1}):
            kvq.kvq_truncate(h, 0, L0)
            kvq.kvq_append(h, 0, kr[:, :, :r].contiguous(), vr[:, :, :r].contiguous(), stream)
            occ[str(r)] = round(1e3 * bm.loop_ms(lambda: kvq.kvq_decode_attention(h, 0, q, out, ws, 0.0, stream), 200), 2)
        kvq.kvq_truncate(h, 0, L0)

        def fill():
            kvq.kvq_append(h, 0, kr, vr, stream)
            kvq.kvq_truncate(h, 0, L0)

        def fill_flush():
            kvq.kvq_append(h, 0, kr, vr, stream)
            kvq.kvq_flush_residual(h, 0, stream)
            kvq.kvq_truncate(h, 0, L0)

        t_fill = bm.loop_ms(fill, 100)
        t_flush = bm.loop_ms(fill_flush, 100) - t_fill
        ring_extra = {"attention_us_at_ring_occupancy": occ,
                      "flush_us_%d_tokens" % (R - 1): round(1e3 * t_flush, 2),
                      "flush_note": "quantize of the ring into the main cache, timed as (ring append + flush) minus (ring append)"}
        status = status or bm.cache.device_status()

    tokens_per_step = w.batch * world
    res = {
        "metric": METRIC,
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
        "config": bm.config(world),
        "roofline": bm.roofline(att_ms),
        "e2e": {"value": round(tokens_per_step / (e2e_ms * 1e-3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps,   # one fused kernel per step
        "clocks": clocks,
        "extra": {"model_tokens_per_s_32_layers": round(value / 32, 1),
                  "attention_only_ms": round(attn_only_ms, 5),
                  "append_1_token_us": round(1e3 * append1_ms, 2),
                  "attention_only_gbs": round(decode_bytes(w, bm.L_main_step, bm.L_ring_step) / (attn_only_ms * 1e-3) / 1e9, 1),
                  "kv_tokens_per_s": round(value * (bm.L_main_step + bm.L_ring_step), 1),
                  "device_status": status},
    }
    res["extra"].update(bm.prefill())
    if ring_extra:
        res["extra"]["residual_ring"] = ring_extra
    L_step = bm.L_main_step + bm.L_ring_step
    del bm, stage_d
    torch.cuda.empty_cache()
    if world == 1 and not args.no_per_workload:
        per = {}
        for name in PER_WORKLOAD:
            if name != w.name:
                per[name] = per_workload_line(name, args, local)
        res["extra"]["per_workload"] = per
        res["extra"]["per_workload_note"] = (
            "each workload timed like the headline: fused decode steps, CUDA events on the "
            "launching stream, at least %d steps and %.0f ms of device time" % (args.steps, args.pw_min_ms))
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = cpu_baseline(w, args.cpu_units, L_step)
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
    """Reference arm: the oracle, timed as it stands on the host cores.  Each
    step is a bounded sample of the workload's decode step -- the oracle's
    step for one (batch, kv-head) unit, i.e. 1/kv_heads of one sequence's
    token -- and ms_per_step is the measured time of that sample."""
    if rank != 0:
        return None
    w = selected_workload(args)
    ctx = sum(step_lengths(w))
    units_per_step = 1
    for i in range(args.warmup):
        if i == 0:   # one untimed sample: imports and first-touch allocations
            oracle_decode_sample(w, [(0, 0)], min(ctx, 64))
    per_steps = []
    for i in range(args.steps):
        u = [((i // w.kv_heads) % w.batch, i % w.kv_heads)]
        per_steps.append(oracle_decode_sample(w, u, ctx))
    ms_step = 1e3 * float(np.mean(per_steps))
    tokens_per_step = units_per_step / w.kv_heads
    value = tokens_per_step / (ms_step * 1e-3)
    sample = ("each step: the oracle's decode step (quantize the new token, dequantize the cache, "
              "fp64 attention) for %d of the %d (batch, kv-head) units at context %d, i.e. %.4g "
              "sequence tokens; ms_per_step is that sample's measured time"
              % (units_per_step, w.units, ctx, tokens_per_step))
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 5), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32 encode, f64 attention",
        "data": "synthetic (seeded numpy, BF16), no model or dataset",
        "config": config_dict(w, world),
        "tokens_per_step": tokens_per_step,
        "cpu_baseline": {"value": round(value, 5), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 5), "unit": "tokens/s", "h2d_bytes_per_step": 0,
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
    ap.add_argument("--no-per-workload", action="store_true",
                    help="time only the headline workload")
    ap.add_argument("--context", type=int, default=0,
                    help="override the workload's prefill length (profiling a smaller case)")
    ap.add_argument("--pw-min-ms", type=float, default=100.0,
                    help="least device time of each per-workload timed loop")
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
