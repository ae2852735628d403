"""Scale renewal on the GPU (NVFP4 / FP8 caches created with the
scale_renewal option) against the oracle's OracleCache(recalibrate_every=P).

Segment 0 of each layer keeps the scale calibrated from the first append;
segment s >= 1 takes the scale of segment s-1's amax; tokens are never
re-encoded.  The inputs grow 2x every 128 tokens (exact in BF16), so a
frozen scale would saturate and every renewed scale differs.  Checked: the
per-segment scales and all codes bit-exact after a prefill spanning several
segments, ragged chunked appends and fused decode steps across segment
boundaries (a step that starts a segment runs as an append plus an
attention launch); attention within tolerance of the oracle's attention over
its own cache (the same codes).
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_13_b200 as kvq
from quantized_kv_cache_13_b200 import workloads as W

from _support import ATOL, RTOL_L2, assert_attention_close, gpu_arrays, to_dev

pytestmark = pytest.mark.gpu

P = 64


def _growing(w, which, n, e0=-3):
    """N(0,1) * 2^e0 growing 2x every 128 tokens (exact in BF16): |v| stays
    below about 10 with e0 = -3 and reaches about 64 with e0 = 0."""
    x = W.kv_tensor(w, which, 0, n)
    g = np.exp2(np.arange(n) // 128 + e0).astype(np.float32)
    return (x * g[None, None, :, None]).astype(np.float32)


def _check(cache, oc):
    torch.cuda.synchronize()
    assert cache.lengths(0) == oc.lengths(0)
    n = oc.lengths(0)[0]
    for kv in (0, 1):
        segs = oc.segment_scales(0, kv)
        got = cache.raw(0, kv)["scale"].cpu().numpy()
        for i, (t, sc) in enumerate(segs):
            assert t == i * P
            assert np.float32(got[i]).view(np.uint32) == np.float32(sc).view(np.uint32), (kv, i)
        for a, b in zip(gpu_arrays(cache, 0, kv, n), oc.main_arrays(0, kv)):
            assert np.array_equal(a, b), kv


@pytest.mark.parametrize("e0", [-3, 0])
@pytest.mark.parametrize("fmt", [kvq.NVFP4, kvq.FP8])
def test_renewed_scales_codes_and_attention(fmt, e0):
    B, H, G, n, steps = 2, 2, 4, 520, 70
    w = W.custom(fmt, B, H, H * G, n + steps, seed=9700 + fmt)
    k = _growing(w, "k", n + steps, e0)
    v = _growing(w, "v", n + steps, e0)
    cache = kvq.KVCache(fmt, 1, B, H, n + steps + 8, 128, 0, 0, scale_renewal=P)
    oc = oracle.OracleCache(fmt, 1, B, H, 128, n + steps + 8, recalibrate_every=P)
    pos = 0
    for step in [200, 1, 63, 64, 65, 1, 126]:       # a prefill over 4 segments, then ragged pieces
        cache.append(0, to_dev(k[:, :, pos:pos + step]), to_dev(v[:, :, pos:pos + step]))
        oc.append(0, k[:, :, pos:pos + step], v[:, :, pos:pos + step])
        pos += step
    assert pos == n
    _check(cache, oc)
    for s in range(steps):                          # fused steps; 576 and 640 start segments
        q = W.q_tensor(w, s)
        out = cache.decode_step(0, to_dev(k[:, :, pos:pos + 1]), to_dev(v[:, :, pos:pos + 1]),
                                to_dev(q)).cpu().numpy()
        oc.append(0, k[:, :, pos:pos + 1], v[:, :, pos:pos + 1])
        pos += 1
        ref = oc.decode_attention(0, q)
        if e0 < 0:
            assert_attention_close(out, ref, "renewal step %d" % s)
        else:
            # the original magnitudes: the bound stated in kvq.h,
            # 2^-10 max|v - out| over the dequantized values (the required
            # max-abs as a floor), and the required rel-L2
            vd = oc.dequantize_main(0, 1).astype(np.float64)          # [B, H, n, D]
            G = q.shape[1] // H
            spread = max(float(np.abs(vd[b, hq // G] - ref[b, hq][None, :]).max())
                         for b in range(B) for hq in range(q.shape[1]))
            err = np.abs(out.astype(np.float64) - ref).max()
            rel = np.linalg.norm(out - ref) / np.linalg.norm(ref)
            assert err <= max(ATOL, 2.0 ** -10 * spread), (s, err, spread)
            assert rel <= RTOL_L2, (s, rel)
    _check(cache, oc)
    for kv in (0, 1):                               # the dequantization uses each token's segment
        got = cache.dequantize(0, kv, 0, pos).cpu().numpy()
        assert np.array_equal(got.view(np.uint32), oc.dequantize_main(0, kv).view(np.uint32))
    assert cache.device_status() == 0


def test_renewal_with_given_scales_and_reset():
    fmt, B, H, n = kvq.NVFP4, 1, 2, 300
    w = W.custom(fmt, B, H, H, n, seed=9800)
    k = _growing(w, "k", n)
    v = _growing(w, "v", n)
    gs = [[0.01, 0.02]]
    cache = kvq.KVCache(fmt, 1, B, H, n + 8, 128, 0, 0, gs, scale_renewal=P)
    oc = oracle.OracleCache(fmt, 1, B, H, 128, n + 8, global_scales=gs, recalibrate_every=P)
    cache.append(0, to_dev(k), to_dev(v))
    oc.append(0, k, v)
    _check(cache, oc)
    cache.reset()
    oc.reset()
    cache.append(0, to_dev(k[:, :, :100]), to_dev(v[:, :, :100]))
    oc.append(0, k[:, :, :100], v[:, :, :100])
    _check(cache, oc)
