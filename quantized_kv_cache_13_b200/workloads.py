"""Seeded synthetic inputs shaped like the pages' decode workloads.

This module generates numbers only: it holds none of the quantization or
attention arithmetic, so both the CUDA path and the CPU oracle can be fed
from it.  No model, checkpoint or dataset is used; the distributions below
stand in for the Qwen3-480B / Llama-2-7B / Llama-3-70B KV tensors the pages
talk about.

Every (config, tensor, batch index, head) slice has its own generator,
seeded by ``numpy.random.SeedSequence([seed, tensor_id, b, h, chunk])``, so
any slice (or any token range of it, in whole chunks) can be regenerated on
the host without generating the rest.  Values are drawn in float32 and
rounded to BF16 (round-to-nearest-even, via torch on the CPU); the returned
float32 arrays hold exactly those BF16 values.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

NVFP4, INT4, FP8, INT8, INT2 = 1, 2, 3, 4, 5

# tensor ids inside a config's seed sequence
T_K, T_V, T_Q, T_KNEW, T_VNEW, T_CHAN = 0, 1, 2, 3, 4, 5

CHUNK = 4096   # tokens per independently seeded chunk


@dataclass(frozen=True)
class Workload:
    name: str
    fmt: int
    batch: int
    kv_heads: int
    q_heads: int
    head_dim: int
    context: int            # tokens quantized at prefill
    decode_steps: int       # decode steps after the prefill
    group_size: int
    residual_length: int
    k_dist: str             # "normal" | "lognormal_outlier" | "offset_uniform"
    v_dist: str
    seed: int
    compact_meta: bool = False  # INT4 g64: f16 S + i8 Z group metadata
    scale_renewal: int = 0      # NVFP4 / FP8: renew the per-tensor scales every this many tokens

    @property
    def G(self) -> int:
        return self.q_heads // self.kv_heads

    @property
    def units(self) -> int:
        return self.batch * self.kv_heads


WORKLOADS = {
    # Tiny NVFP4 case: 1 layer, B1, 2 KV heads, 8 query heads, L 512.
    "tiny_nvfp4": Workload("tiny_nvfp4", NVFP4, 1, 2, 8, 128, 512, 1, 16, 0,
                           "normal", "normal", 1001),
    # GQA 8/32, B8, 32K context, NVFP4, K with per-channel lognormal scales
    # and 2 % outlier channels.
    "gqa_nvfp4_32k": Workload("gqa_nvfp4_32k", NVFP4, 8, 8, 32, 128, 32768, 1, 16, 0,
                              "lognormal_outlier", "normal", 1002),
    # Llama-2-7B attention shape (MHA 32 heads), B4, 16K, INT4 g64 + ring 128.
    "mha_int4_16k": Workload("mha_int4_16k", INT4, 4, 32, 32, 128, 16384, 1, 64, 128,
                             "offset_uniform", "offset_uniform", 1003),
    # FP8-E4M3 per-tensor, GQA 8/32, B16, 32K.
    "gqa_fp8_32k": Workload("gqa_fp8_32k", FP8, 16, 8, 32, 128, 32768, 1, 0, 0,
                            "normal", "normal", 1004),
    # Same shape and seed in NVFP4 (the comparison the pages draw).
    "gqa_nvfp4_32k_b16": Workload("gqa_nvfp4_32k_b16", NVFP4, 16, 8, 32, 128, 32768, 1, 16, 0,
                                  "normal", "normal", 1004),
    # 70B-style attention: GQA 8/64, B8, 128K context, 64 decode steps.
    "long_nvfp4_128k": Workload("long_nvfp4_128k", NVFP4, 8, 8, 64, 128, 131072, 64, 16, 0,
                                "normal", "normal", 1005),
    # The INT4 workload's shape in INT8 g64 + ring 128 (the 8-bit setting of
    # the same affine residual-cache quantizer).
    "mha_int8_16k": Workload("mha_int8_16k", INT8, 4, 32, 32, 128, 16384, 1, 64, 128,
                             "offset_uniform", "offset_uniform", 1006),
    # The same shape in INT2 g64 + ring 128 (the INT2 row of the Llama-2 table).
    "mha_int2_16k": Workload("mha_int2_16k", INT2, 4, 32, 32, 128, 16384, 1, 64, 128,
                             "offset_uniform", "offset_uniform", 1007),
    # Cache options on the headline shapes, for timing against the plain ones
    # (same seeds, so the same data):
    # INT4 g64 with compact group metadata (72 instead of 80 bytes per token and head).
    "mha_int4_16k_compact": Workload("mha_int4_16k_compact", INT4, 4, 32, 32, 128, 16384, 1, 64, 128,
                                     "offset_uniform", "offset_uniform", 1003, compact_meta=True),
    # NVFP4 with the scale renewed every 512 tokens; the context leaves the
    # decode token inside a segment, so the step is the fused one.
    "gqa_nvfp4_32k_renew512": Workload("gqa_nvfp4_32k_renew512", NVFP4, 8, 8, 32, 128, 32868, 1, 16, 0,
                                       "lognormal_outlier", "normal", 1002, scale_renewal=512),
    # NVFP4 with a 128-token BF16 ring in front of the main cache.
    "gqa_nvfp4_32k_ring128": Workload("gqa_nvfp4_32k_ring128", NVFP4, 8, 8, 32, 128, 32768, 1, 16, 128,
                                      "lognormal_outlier", "normal", 1002),
}


def _rng(seed: int, tensor: int, b: int, h: int, chunk: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor, b, h, chunk])))


def to_bf16_values(x: np.ndarray) -> np.ndarray:
    """Round float32 to BF16 (RNE) and return the exact values as float32."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def _channel_scale(w: Workload, kind: str, h: int) -> Optional[np.ndarray]:
    """Per-(kv head, channel) multiplier or offset, shared across the batch."""
    D = w.head_dim
    rng = _rng(w.seed, T_CHAN, 0, h, 0)
    if kind == "lognormal_outlier":
        c = rng.lognormal(0.0, 0.5, size=D).astype(np.float32)
        n_out = int(round(0.02 * D))                 # 2 % of the channels
        idx = rng.permutation(D)[:n_out]
        c[idx] *= 8.0
        return c
    if kind == "offset_uniform":
        return rng.uniform(-1.0, 1.0, size=D).astype(np.float32)
    return None


def _draw(w: Workload, dist: str, tensor: int, b: int, h: int, t0: int, n: int) -> np.ndarray:
    """float32 [n, D] for tokens [t0, t0 + n) of slice (b, h), before BF16."""
    D = w.head_dim
    out = np.empty((n, D), np.float32)
    pos = 0
    c0 = t0 // CHUNK
    c1 = (t0 + n - 1) // CHUNK if n > 0 else c0 - 1
    for c in range(c0, c1 + 1):
        chunk = _rng(w.seed, tensor, b, h, c).standard_normal((CHUNK, D), dtype=np.float32)
        lo = max(t0, c * CHUNK) - c * CHUNK
        hi = min(t0 + n, (c + 1) * CHUNK) - c * CHUNK
        out[pos:pos + hi - lo] = chunk[lo:hi]
        pos += hi - lo
    ch = _channel_scale(w, dist, h)
    if dist == "lognormal_outlier":
        out *= ch[None, :]
    elif dist == "offset_uniform":
        out += ch[None, :]
    return out


def kv_slice(w: Workload, which: str, b: int, h: int, t0: int, n: int) -> np.ndarray:
    """BF16 values (as float32 [n, D]) of K or V tokens [t0, t0+n) of (b, h).

    Prefill tokens are positions [0, context); decode step s appends the token
    at position context + s, drawn from the same per-slice stream.
    """
    tensor = T_K if which == "k" else T_V
    dist = w.k_dist if which == "k" else w.v_dist
    return to_bf16_values(_draw(w, dist, tensor, b, h, t0, n))


def kv_tensor(w: Workload, which: str, t0: int, n: int) -> np.ndarray:
    """BF16 values as float32 [B, Hkv, n, D] for tokens [t0, t0+n)."""
    out = np.empty((w.batch, w.kv_heads, n, w.head_dim), np.float32)
    for b in range(w.batch):
        for h in range(w.kv_heads):
            out[b, h] = kv_slice(w, which, b, h, t0, n)
    return out


def q_tensor(w: Workload, step: int = 0) -> np.ndarray:
    """Query BF16 values as float32 [B, Hq, D]; Q ~ N(0, 1) for every config."""
    out = np.empty((w.batch, w.q_heads, w.head_dim), np.float32)
    for b in range(w.batch):
        rng = _rng(w.seed, T_Q, b, step, 0)
        out[b] = rng.standard_normal((w.q_heads, w.head_dim), dtype=np.float32)
    return to_bf16_values(out)


def custom(fmt: int, batch: int, kv_heads: int, q_heads: int, context: int, seed: int,
           head_dim: int = 128, group_size: int = 0, residual_length: int = 0,
           k_dist: str = "normal", v_dist: str = "normal") -> Workload:
    """A small ad-hoc workload for tests (odd shapes, ragged lengths)."""
    if group_size == 0:
        group_size = 16 if fmt == NVFP4 else 64 if fmt in (INT4, INT8, INT2) else 0
    return Workload("custom", fmt, batch, kv_heads, q_heads, head_dim, context, 1,
                    group_size, residual_length, k_dist, v_dist, seed)
