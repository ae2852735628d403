"""Shared helpers for the parity tests: feed the same seeded inputs to the
CUDA library and to the oracle, read the CUDA cache's raw planes back and
compare."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import quantized_kv_cache_13_b200 as kvq
from quantized_kv_cache_13_b200 import workloads as W

ATOL = 1e-2      # attention: max-abs error
RTOL_L2 = 2e-3   # attention: relative L2 error


def to_dev(x: np.ndarray) -> torch.Tensor:
    """float32 array holding BF16 values -> contiguous bf16 CUDA tensor."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).cuda()


def gpu_arrays(cache: kvq.KVCache, layer: int, kv: int, n: int):
    """Main-cache arrays of the CUDA cache, shaped like the oracle's (codes in
    token-major packing, see KVCache.canonical_codes)."""
    raw = cache.raw(layer, kv)
    codes = cache.canonical_codes(layer, kv, 0, n).cpu().numpy()
    if cache.fmt == kvq.NVFP4:
        return (codes, raw["meta"][:, :, :n].cpu().numpy())
    if cache.fmt == kvq.FP8:
        return (codes,)
    meta = raw["meta"][:, :, :n].cpu()
    S = meta[..., 0].contiguous().view(torch.float32).numpy()
    Z = meta[..., 1].contiguous().numpy()
    return (codes, S, Z)


def gpu_unit_arrays(cache: kvq.KVCache, layer: int, kv: int, b: int, h: int, n: int):
    """Main-cache arrays of one (batch, kv-head) unit, tokens [0, n)."""
    raw = cache.raw(layer, kv)
    codes = cache.canonical_codes(layer, kv, 0, n)[b, h].cpu().numpy()
    if cache.fmt == kvq.NVFP4:
        return (codes, raw["meta"][b, h, :n].cpu().numpy())
    if cache.fmt == kvq.FP8:
        return (codes,)
    meta = raw["meta"][b, h, :n].cpu()
    return (codes, meta[..., 0].contiguous().view(torch.float32).numpy(), meta[..., 1].contiguous().numpy())


def gpu_scale(cache: kvq.KVCache, layer: int, kv: int):
    raw = cache.raw(layer, kv)
    return float(raw["scale"].cpu().numpy()[0]) if "scale" in raw else None


def gpu_ring(cache: kvq.KVCache, layer: int, kv: int, r: int) -> np.ndarray:
    raw = cache.raw(layer, kv)
    return raw["ring"][:, :, :r].float().cpu().numpy()


def assert_cache_bit_exact(cache: kvq.KVCache, oc: oracle.OracleCache, layer: int = 0):
    torch.cuda.synchronize()
    assert cache.lengths(layer) == oc.lengths(layer)
    n, r = oc.lengths(layer)
    for kv in (0, 1):
        if cache.fmt not in kvq.INT_AFFINE:
            g = gpu_scale(cache, layer, kv)
            assert np.float32(g).view(np.uint32) == np.float32(oc.scale(layer, kv)).view(np.uint32), \
                "per-tensor scale differs: %r vs %r" % (g, oc.scale(layer, kv))
        if n:
            ours = gpu_arrays(cache, layer, kv, n)
            ref = oc.main_arrays(layer, kv)
            for name, a, b in zip(("codes", "meta", "zero"), ours, ref):
                if a.dtype == np.float32:
                    a, b = a.view(np.uint32), np.asarray(b, np.float32).view(np.uint32)
                bad = np.argwhere(a != b)
                assert bad.size == 0, "%s differ at %d places, first %s: %r vs %r" % (
                    name, len(bad), bad[0].tolist(), a[tuple(bad[0])], b[tuple(bad[0])])
        if r:
            assert np.array_equal(gpu_ring(cache, layer, kv, r), oc.ring_tokens(layer, kv))


def reference_attention(cache: kvq.KVCache, q: np.ndarray, layer: int = 0, scale=None,
                        units=None) -> np.ndarray:
    """Oracle attention over the oracle's dequantization of the CUDA cache's
    own (bit-checked) codes plus its ring tokens.  units: optional list of
    (b, kvh) to compute (others left 0)."""
    n, r = cache.lengths(layer)
    B, Hkv, D = cache.batch, cache.kv_heads, cache.head_dim
    Hq = q.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    Ks = [None, None]
    for kv in (0, 1):
        parts = []
        if n:
            arrs = gpu_arrays(cache, layer, kv, n)
            parts.append(oracle.dequantize_arrays(cache.fmt, arrs, gpu_scale(cache, layer, kv),
                                                  cache.group_size or 16))
        if r:
            parts.append(gpu_ring(cache, layer, kv, r))
        Ks[kv] = np.concatenate(parts, axis=2)
    out = np.zeros((B, Hq, D), np.float64)
    todo = units if units is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    for b, h in todo:
        out[b, h * G:(h + 1) * G] = oracle.attention(q[b, h * G:(h + 1) * G], Ks[0][b, h],
                                                     Ks[1][b, h], scale)
    return out


def assert_attention_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    got = got.astype(np.float64)
    err = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert np.all(np.isfinite(got)), what + ": non-finite output"
    assert err.max() <= ATOL, "%s: max-abs error %.3e > %.0e" % (what, err.max(), ATOL)
    assert rel <= RTOL_L2, "%s: rel-L2 error %.3e > %.0e" % (what, rel, RTOL_L2)


def make_pair(w: W.Workload, max_len: int = None, global_scales=None):
    """A CUDA cache and an oracle cache for workload w (one layer)."""
    max_len = max_len or (w.context + w.decode_steps)
    grp = w.group_size if w.fmt in kvq.INT_AFFINE else 0
    cache = kvq.KVCache(w.fmt, 1, w.batch, w.kv_heads, max_len, w.head_dim, grp,
                        w.residual_length, global_scales)
    oc = oracle.OracleCache(w.fmt, 1, w.batch, w.kv_heads, w.head_dim, max_len, grp,
                            w.residual_length, global_scales)
    return cache, oc
