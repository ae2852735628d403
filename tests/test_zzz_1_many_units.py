"""A cache with more (batch, kv head) units than a grid's y dimension holds.

The quantize kernels put units on gridDim.y, capped at 65,535 blocks; past
that cap each block walks units in steps of gridDim.y.  With 516 x 128 =
66,048 units, the units on both sides of the cap are checked against the
oracle: codes and scales bit for bit, the dequantization, decode attention,
and one fused decode step.  The cache holds about 8 GB.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_13_b200 as kvq

from _support import assert_attention_close, gpu_scale, gpu_unit_arrays, reference_attention, to_dev

pytestmark = pytest.mark.gpu

B, H, N = 516, 128, 5                      # 66,048 units, 5 prefill tokens each
UNITS = [0, 1, 4097, 65534, 65535, 65536, 65537, 66046, 66047]


def _bf16(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(a.astype(np.float32)).bfloat16().float().numpy()


def _oracle_unit(fmt, x, g):
    """Oracle encoding of one unit's tokens x [n, 128]."""
    if fmt == kvq.NVFP4:
        return oracle.nvfp4_quantize(x, g)
    return oracle.int4_quantize(x, 64)


def _check_codes(cache, fmt, k, v, n, gs):
    for kv, x in ((0, k), (1, v)):
        if fmt == kvq.NVFP4:
            assert np.float32(gpu_scale(cache, 0, kv)).view(np.uint32) == np.float32(gs[kv]).view(np.uint32)
        for u in UNITS:
            b, h = divmod(u, H)
            ours = gpu_unit_arrays(cache, 0, kv, b, h, n)
            ref = _oracle_unit(fmt, x[b, h, :n], gs[kv])
            for a, r in zip(ours, ref):
                a, r = np.asarray(a), np.asarray(r)
                if a.dtype == np.float32:
                    a, r = a.view(np.uint32), r.astype(np.float32).view(np.uint32)
                assert np.array_equal(a, r), "unit %d (b %d, h %d), kv %d" % (u, b, h, kv)


def _check_attention(cache, q, what):
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    units = [divmod(u, H) for u in UNITS]
    ref = reference_attention(cache, q, units=units)
    for b, h in units:                     # G = 1: query head h reads kv head h
        assert_attention_close(out[b, h:h + 1], ref[b, h:h + 1], "%s unit (%d, %d)" % (what, b, h))


@pytest.mark.parametrize("fmt", [kvq.NVFP4, kvq.INT4])
def test_units_beyond_one_grid_row(fmt):
    rng = np.random.default_rng(66048 + fmt)
    k = _bf16(rng.standard_normal((B, H, N + 1, 128)))
    v = _bf16(rng.standard_normal((B, H, N + 1, 128)))
    q = _bf16(rng.standard_normal((B, H, 128)))
    grp = 64 if fmt == kvq.INT4 else 0
    cache = kvq.KVCache(fmt, 1, B, H, N + 1, 128, grp, 0, None)
    gs = [None, None]
    if fmt == kvq.NVFP4:                   # calibrated from the first append's amax
        gs = [oracle.global_scale(fmt, oracle.amax(k[:, :, :N])),
              oracle.global_scale(fmt, oracle.amax(v[:, :, :N]))]

    cache.append(0, to_dev(k[:, :, :N]), to_dev(v[:, :, :N]))
    torch.cuda.synchronize()
    assert cache.lengths(0) == (N, 0)
    _check_codes(cache, fmt, k, v, N, gs)
    for kv, x in ((0, k), (1, v)):
        got = cache.dequantize(0, kv, 0, N).cpu().numpy()
        for u in UNITS:
            b, h = divmod(u, H)
            arrs = _oracle_unit(fmt, x[b, h, :N], gs[kv])
            ref = oracle.dequantize_arrays(fmt, arrs, gs[kv], grp or 16)
            assert np.array_equal(got[b, h].view(np.uint32), ref.view(np.uint32)), "dequantize unit %d" % u
    _check_attention(cache, q, "append")

    # one fused step: the new token is written by the attention launch
    out = cache.decode_step(0, to_dev(k[:, :, N:N + 1]), to_dev(v[:, :, N:N + 1]), to_dev(q))
    torch.cuda.synchronize()
    assert cache.lengths(0) == (N + 1, 0)
    _check_codes(cache, fmt, k, v, N + 1, gs)
    units = [divmod(u, H) for u in UNITS]
    ref = reference_attention(cache, q, units=units)
    out = out.cpu().numpy()
    for b, h in units:
        assert_attention_close(out[b, h:h + 1], ref[b, h:h + 1], "step unit (%d, %d)" % (b, h))
    assert cache.device_status() == 0
