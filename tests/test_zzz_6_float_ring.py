"""NVFP4 and FP8 caches with a BF16 residual ring (the ring of the INT
formats put in front of the per-tensor-scaled formats), against the oracle.

The per-tensor scales are calibrated from the first append even when all of
its tokens go to the ring; the ring's tokens are encoded with them when it
fills (or on flush).  Attention reads the quantized main cache with the
scales folded out and the ring's exact BF16 values scaled by 1 / g_V, and
the output multiplies g_V back.  Checked: codes, block scales, per-tensor
scales and ring bit-exact; attention within tolerance, including ring-only
caches; bulk = chunked appends; the fused step including the ring-fill
fallback.
"""
import pytest

import quantized_kv_cache_13_b200 as kvq
from quantized_kv_cache_13_b200 import workloads as W

from _support import (assert_attention_close, assert_cache_bit_exact, make_pair,
                      reference_attention, to_dev)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt,R,L,dist", [
    (kvq.NVFP4, 128, 700, "lognormal_outlier"),
    (kvq.NVFP4, 128, 100, "normal"),          # ring only: nothing quantized yet
    (kvq.FP8, 48, 333, "normal"),
    (kvq.FP8, 16, 1029, "offset_uniform"),
])
def test_float_format_ring_parity(fmt, R, L, dist):
    w = W.custom(fmt, 2, 2, 8, L, seed=9500 + L + R, residual_length=R, k_dist=dist, v_dist=dist)
    cache, oc = make_pair(w, max_len=L + 64)
    k = W.kv_tensor(w, "k", 0, L)
    v = W.kv_tensor(w, "v", 0, L)
    cache.append(0, to_dev(k), to_dev(v))
    oc.append(0, k, v)
    assert cache.lengths(0) == oc.lengths(0) == ((L // R) * R, L % R)
    assert_cache_bit_exact(cache, oc)
    q = W.q_tensor(w)
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert_attention_close(out, reference_attention(cache, q), "fmt %d R%d L%d" % (fmt, R, L))
    assert_attention_close(out, oc.decode_attention(0, q), "vs the oracle's cache")
    cache.flush_residual(0)
    oc.flush_residual(0)
    assert_cache_bit_exact(cache, oc)
    out2 = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert_attention_close(out2, reference_attention(cache, q), "after flush")
    assert cache.device_status() == 0


@pytest.mark.parametrize("fmt", [kvq.NVFP4, kvq.FP8])
def test_float_format_ring_chunked_equals_bulk(fmt):
    R, n = 64, 500
    w = W.custom(fmt, 2, 2, 4, n, seed=9600 + fmt, residual_length=R)
    k = W.kv_tensor(w, "k", 0, n)
    v = W.kv_tensor(w, "v", 0, n)
    # both caches calibrate on the same first append (its first 40 tokens)
    a, oa = make_pair(w, max_len=n + 16)
    a.append(0, to_dev(k[:, :, :40]), to_dev(v[:, :, :40]))
    oa.append(0, k[:, :, :40], v[:, :, :40])
    pos = 40
    for step in [1, 23, 64, 1, 130, 7, 234]:
        a.append(0, to_dev(k[:, :, pos:pos + step]), to_dev(v[:, :, pos:pos + step]))
        oa.append(0, k[:, :, pos:pos + step], v[:, :, pos:pos + step])
        pos += step
    assert pos == n
    gs = [[oa.scale(0, 0), oa.scale(0, 1)]]
    b, ob = make_pair(w, max_len=n + 16, global_scales=gs)
    b.append(0, to_dev(k), to_dev(v))
    ob.append(0, k, v)
    assert_cache_bit_exact(a, oa)
    assert_cache_bit_exact(b, ob)
    assert a.lengths(0) == b.lengths(0) == ((n // R) * R, n % R)
    # Only the live part of each plane is defined: ring slots at or past
    # len_ring hold whatever tokens an earlier ring fill left there, and those
    # differ between a chunked and a bulk history.
    import torch
    n_main, n_ring = a.lengths(0)
    for kv in (0, 1):
        ra, rb = a.raw(0, kv), b.raw(0, kv)
        assert torch.equal(ra["codes"][:, :, :n_main], rb["codes"][:, :, :n_main]), (kv, "codes")
        if "meta" in ra:
            assert torch.equal(ra["meta"][:, :, :n_main], rb["meta"][:, :, :n_main]), (kv, "meta")
        assert torch.equal(ra["ring"][:, :, :n_ring], rb["ring"][:, :, :n_ring]), (kv, "ring")
        assert torch.equal(ra["scale"], rb["scale"]), (kv, "scale")


@pytest.mark.parametrize("fmt,R,L,steps", [(kvq.NVFP4, 16, 40, 30), (kvq.FP8, 128, 1000, 6)])
def test_float_format_ring_decode_step(fmt, R, L, steps):
    from test_gpu_decode_step import test_decode_step_matches_separate_calls
    test_decode_step_matches_separate_calls(fmt, R, 2, L, steps)
