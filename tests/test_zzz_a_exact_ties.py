"""Quantized codes at exact rounding ties, against the oracle.

The bulk append kernels take each code from the correctly rounded
quotient of the value by the block / tensor / group scale, formed from a
reciprocal product with one FMA correction; the per-token kernels and the
fused decode step's encoder use a bracketed reciprocal and divide exactly
only when the bracket straddles a decision boundary.  These inputs put the
quotient exactly on a boundary -- E2M1 midpoints for NVFP4, E4M3 midpoints
for FP8, half-integers for the affine formats -- so every code here is a
tie that must round half to even like the oracle, and every bracket takes
its exact path.  Random values are mixed in, and the same inputs go
through the fused decode step's encoder."""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_13_b200 as kvq
from quantized_kv_cache_13_b200 import workloads as W

from _support import assert_cache_bit_exact, make_pair, to_dev

pytestmark = pytest.mark.gpu

E2M1_TIES = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]


def _nvfp4_tie_tokens(rng, B, H, n):
    """Blocks whose amax is 6 * 2^k (so with a per-tensor scale of 1 the
    block scale is 2^k exactly) and whose other values are E2M1 midpoints
    times 2^k, with random signs."""
    x = np.empty((B, H, n, 128), np.float32)
    for blk in range(8):
        k = rng.integers(-6, 5, size=(B, H, n, 1)).astype(np.float32)
        vals = rng.choice(E2M1_TIES + [0.5, 1.0, 3.0], size=(B, H, n, 16)).astype(np.float32)
        vals[..., 0] = 6.0
        sign = rng.choice([-1.0, 1.0], size=vals.shape).astype(np.float32)
        x[..., 16 * blk:16 * blk + 16] = vals * sign * np.exp2(k)
    return W.to_bf16_values(x)


def _nvfp4_scale_tie_tokens(rng, B, H, n):
    """Blocks whose amax / 6 is a midpoint between two E4M3 values (with a
    per-tensor scale of 1), so the block scale itself rounds a tie."""
    vals = np.abs(oracle.e4m3_decode(np.arange(8, 120, dtype=np.uint8)).astype(np.float64))
    mids = (vals[1:] + vals[:-1]) / 2
    mids = mids[(W.to_bf16_values((6 * mids).astype(np.float32)) == (6 * mids).astype(np.float32))]
    x = rng.standard_normal((B, H, n, 128)).astype(np.float32)
    for blk in range(8):
        m = rng.choice(mids, size=(B, H, n)).astype(np.float32)
        x[..., 16 * blk:16 * blk + 16] *= (m / 4)[..., None]
        x[..., 16 * blk] = 6 * m * rng.choice([-1.0, 1.0], size=(B, H, n))
    return W.to_bf16_values(x)


def _affine_tie_tokens(rng, B, H, n, qmax):
    """Groups spanning exactly qmax * 2^k (so S = 2^k) from min = -z * 2^k,
    other values at half-integers times 2^k inside the range."""
    x = np.empty((B, H, n, 128), np.float32)
    for g in range(2):
        k = rng.integers(-8, 3, size=(B, H, n, 1)).astype(np.float32)
        z = rng.integers(0, qmax + 1, size=(B, H, n, 1)).astype(np.float32)
        half = rng.integers(0, qmax, size=(B, H, n, 64)).astype(np.float32) + 0.5
        half[..., 0] = 0.0
        half[..., 1] = qmax
        x[..., 64 * g:64 * g + 64] = (half - z) * np.exp2(k)
    return W.to_bf16_values(x)


def _fp8_tie_tokens(rng, B, H, n):
    """Midpoints between neighbouring E4M3 values that BF16 holds exactly."""
    vals = np.abs(oracle.e4m3_decode(np.arange(0, 127, dtype=np.uint8)).astype(np.float64))
    vals = np.unique(vals[np.isfinite(vals)])
    mids = (vals[1:] + vals[:-1]) / 2
    mids = mids[W.to_bf16_values(mids.astype(np.float32)) == mids.astype(np.float32)]
    x = rng.choice(mids, size=(B, H, n, 128)) * rng.choice([-1.0, 1.0], size=(B, H, n, 128))
    return W.to_bf16_values(x.astype(np.float32))


@pytest.mark.parametrize("fmt", [kvq.NVFP4, kvq.FP8, kvq.INT4, kvq.INT8, kvq.INT2, "nvfp4_scale"])
def test_codes_at_exact_ties(fmt):
    B, H, n = 2, 2, 150
    rng = np.random.default_rng(12000 + (99 if fmt == "nvfp4_scale" else fmt))
    if fmt == "nvfp4_scale":
        fmt = kvq.NVFP4
        k, v = _nvfp4_scale_tie_tokens(rng, B, H, n), _nvfp4_scale_tie_tokens(rng, B, H, n)
    elif fmt == kvq.NVFP4:
        k, v = _nvfp4_tie_tokens(rng, B, H, n), _nvfp4_tie_tokens(rng, B, H, n)
    elif fmt == kvq.FP8:
        k, v = _fp8_tie_tokens(rng, B, H, n), _fp8_tie_tokens(rng, B, H, n)
    else:
        qmax = {kvq.INT4: 15, kvq.INT8: 255, kvq.INT2: 3}[fmt]
        k, v = _affine_tie_tokens(rng, B, H, n, qmax), _affine_tie_tokens(rng, B, H, n, qmax)
    # a few random tokens as well
    k[:, :, -20:] = W.to_bf16_values(rng.standard_normal((B, H, 20, 128)).astype(np.float32))
    gs = None if fmt in kvq.INT_AFFINE else [[1.0, 1.0]]
    w = W.custom(fmt, B, H, H, n, seed=1)
    cache, oc = make_pair(w, max_len=n + 8, global_scales=gs)
    # appends of odd length, so later ones start at odd destinations
    for lo, hi in ((0, 37), (37, 38), (38, 101), (101, n - 4)):
        cache.append(0, to_dev(k[:, :, lo:hi]), to_dev(v[:, :, lo:hi]))
        oc.append(0, k[:, :, lo:hi], v[:, :, lo:hi])
    assert_cache_bit_exact(cache, oc)
    # the fused decode step's encoder on tie tokens too
    q = to_dev(W.to_bf16_values(rng.standard_normal((B, H, 128)).astype(np.float32)))
    for t in range(n - 4, n):
        cache.decode_step(0, to_dev(k[:, :, t:t + 1]), to_dev(v[:, :, t:t + 1]), q)
        oc.append(0, k[:, :, t:t + 1], v[:, :, t:t + 1])
    assert_cache_bit_exact(cache, oc)
    assert cache.device_status() == 0
