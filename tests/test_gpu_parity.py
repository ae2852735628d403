"""CUDA path vs the oracle on the same seeded inputs.

Codes, block scales, zero points, per-tensor scales and ring contents must
be bit-identical; decode attention must agree with the oracle's binary64
attention over the identically dequantized cache within max-abs 1e-2 and
relative L2 2e-3.  Sizes here finish in seconds on the oracle yet span many
128-token tiles, several splits and ragged tails.
"""

import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_13_b200 as kvq
from quantized_kv_cache_13_b200 import workloads as W

from _support import (assert_attention_close, assert_cache_bit_exact, make_pair,
                      reference_attention, to_dev)

pytestmark = pytest.mark.gpu


def _prefill(w, cache, oc, n=None):
    n = w.context if n is None else n
    k = W.kv_tensor(w, "k", 0, n)
    v = W.kv_tensor(w, "v", 0, n)
    cache.append(0, to_dev(k), to_dev(v))
    oc.append(0, k, v)
    return k, v


def test_tiny_nvfp4_config_end_to_end():
    """The tiny NVFP4 workload: quantize-append 512 tokens, one decode step."""
    w = W.WORKLOADS["tiny_nvfp4"]
    cache, oc = make_pair(w)
    _prefill(w, cache, oc)
    # the decode token, then attention
    k1 = W.kv_tensor(w, "k", w.context, 1)
    v1 = W.kv_tensor(w, "v", w.context, 1)
    cache.append(0, to_dev(k1), to_dev(v1))
    oc.append(0, k1, v1)
    assert_cache_bit_exact(cache, oc)
    q = W.q_tensor(w)
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert_attention_close(out, reference_attention(cache, q), "tiny nvfp4")
    # and the oracle's own cache gives the same reference (codes are identical)
    assert_attention_close(out, oc.decode_attention(0, q), "tiny nvfp4 vs oracle cache")


@pytest.mark.parametrize("fmt,grp,R,kd", [
    (kvq.NVFP4, 16, 0, "lognormal_outlier"),
    (kvq.FP8, 0, 0, "normal"),
    (kvq.INT4, 64, 128, "offset_uniform"),
    (kvq.INT4, 32, 0, "normal"),
    (kvq.INT4, 64, 48, "normal"),
    (kvq.INT8, 64, 128, "offset_uniform"),
    (kvq.INT8, 64, 0, "normal"),
])
@pytest.mark.parametrize("B,Hkv,G,L", [(2, 2, 4, 1000), (1, 3, 8, 129), (3, 1, 1, 777)])
def test_append_and_attention_parity(fmt, grp, R, kd, B, Hkv, G, L):
    w = W.custom(fmt, B, Hkv, Hkv * G, L, seed=7000 + L + 10 * G, group_size=grp,
                 residual_length=R, k_dist=kd, v_dist=kd)
    cache, oc = make_pair(w, max_len=L + 64)
    _prefill(w, cache, oc)
    assert_cache_bit_exact(cache, oc)
    q = W.q_tensor(w)
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert_attention_close(out, reference_attention(cache, q), "fmt %d B%d H%d G%d L%d" % (fmt, B, Hkv, G, L))


@pytest.mark.parametrize("fmt", [kvq.NVFP4, kvq.FP8, kvq.INT4, kvq.INT8])
@pytest.mark.parametrize("L", [1, 15, 16, 17, 127, 128, 129, 255, 256, 257, 383, 384, 385, 767, 768, 769])
def test_ragged_lengths(fmt, L):
    R = 128 if fmt in kvq.INT_AFFINE else 0
    w = W.custom(fmt, 2, 2, 8, L, seed=800 + L, residual_length=R)
    cache, oc = make_pair(w, max_len=max(300, L))
    _prefill(w, cache, oc)
    assert_cache_bit_exact(cache, oc)
    q = W.q_tensor(w)
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert_attention_close(out, reference_attention(cache, q), "ragged L=%d" % L)


@pytest.mark.parametrize("fmt", [kvq.NVFP4, kvq.FP8, kvq.INT4, kvq.INT8])
def test_incremental_equals_bulk_append(fmt):
    """Chunked appends (including single tokens) give the bulk result bit for bit."""
    R = 128 if fmt in kvq.INT_AFFINE else 0
    w = W.custom(fmt, 2, 2, 8, 700, seed=901, residual_length=R)
    k = W.kv_tensor(w, "k", 0, 700)
    v = W.kv_tensor(w, "v", 0, 700)
    gs = None
    if fmt not in kvq.INT_AFFINE:
        gs = [[oracle.global_scale(fmt, oracle.amax(k[:, :, :300])),
               oracle.global_scale(fmt, oracle.amax(v[:, :, :300]))]]
    cache, oc = make_pair(w, max_len=800)
    cache.append(0, to_dev(k[:, :, :300]), to_dev(v[:, :, :300]))
    oc.append(0, k[:, :, :300], v[:, :, :300])
    pos = 300
    for step in [1, 1, 5, 127, 1, 128, 129, 1, 7]:
        cache.append(0, to_dev(k[:, :, pos:pos + step]), to_dev(v[:, :, pos:pos + step]))
        oc.append(0, k[:, :, pos:pos + step], v[:, :, pos:pos + step])
        pos += step
    assert_cache_bit_exact(cache, oc)
    bulk = kvq.KVCache(fmt, 1, 2, 2, 800, 128, 64 if fmt in kvq.INT_AFFINE else 0, R, gs)
    ob = oracle.OracleCache(fmt, 1, 2, 2, 128, 800, 64 if fmt in kvq.INT_AFFINE else 0, R, gs)
    bulk.append(0, to_dev(k[:, :, :pos]), to_dev(v[:, :, :pos]))
    ob.append(0, k[:, :, :pos], v[:, :, :pos])
    assert_cache_bit_exact(bulk, ob)
    if fmt in kvq.INT_AFFINE:
        # token-by-token semantics: the two caches agree on every byte
        n, _ = cache.lengths(0)
        a = cache.raw(0, 0)["codes"][:, :, :n].cpu()
        b = bulk.raw(0, 0)["codes"][:, :, :n].cpu()
        assert torch.equal(a, b)
    q = W.q_tensor(w)
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert_attention_close(out, reference_attention(cache, q), "incremental")


@pytest.mark.parametrize("fmt", [kvq.INT4, kvq.INT8])
def test_flush_residual_and_ring_only_cache(fmt):
    w = W.custom(fmt, 2, 2, 4, 100, seed=33, residual_length=128)
    cache, oc = make_pair(w, max_len=400)
    _prefill(w, cache, oc)                  # 100 tokens: all in the ring
    assert cache.lengths(0) == (0, 100)
    q = W.q_tensor(w)
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert_attention_close(out, reference_attention(cache, q), "ring only")
    cache.flush_residual(0)
    oc.flush_residual(0)
    assert_cache_bit_exact(cache, oc)
    assert cache.lengths(0) == (100, 0)
    out2 = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert_attention_close(out2, reference_attention(cache, q), "after flush")


@pytest.mark.parametrize("fmt", [kvq.NVFP4, kvq.FP8, kvq.INT4, kvq.INT8])
def test_dequantize_matches_oracle_bit_exact(fmt):
    w = W.custom(fmt, 2, 3, 3, 300, seed=44)
    cache, oc = make_pair(w, max_len=300)
    _prefill(w, cache, oc)
    for kv in (0, 1):
        got = cache.dequantize(0, kv, 37, 200).cpu().numpy()
        ref = oc.dequantize_main(0, kv)[:, :, 37:237]
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("splits", ["1", "3", "7", "64", "1000"])
def test_split_count_invariance(splits, monkeypatch):
    monkeypatch.setenv("KVQ_CTAS", splits)
    w = W.custom(kvq.NVFP4, 2, 2, 8, 3000, seed=55)
    cache, oc = make_pair(w, max_len=3000)
    _prefill(w, cache, oc)
    q = W.q_tensor(w)
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert_attention_close(out, reference_attention(cache, q), "splits=" + splits)


def test_cast_scales_and_zero_tensor():
    """Given scales (the *_cast variants) are used as-is; an all-zero first
    append calibrates to scale 1."""
    w = W.custom(kvq.NVFP4, 1, 2, 8, 64, seed=66)
    k = W.kv_tensor(w, "k", 0, 64)
    v = W.kv_tensor(w, "v", 0, 64)
    cache, oc = make_pair(w, max_len=128, global_scales=[[1.0, 1.0]])
    cache.append(0, to_dev(k), to_dev(v))
    oc.append(0, k, v)
    assert_cache_bit_exact(cache, oc)
    for fmt in (kvq.NVFP4, kvq.FP8):
        z = np.zeros_like(k)
        c2 = kvq.KVCache(fmt, 1, 1, 2, 128)
        o2 = oracle.OracleCache(fmt, 1, 1, 2, 128, 128)
        c2.append(0, to_dev(z), to_dev(v))
        o2.append(0, z, v)
        assert_cache_bit_exact(c2, o2)


def test_sign_of_zero_codes():
    """Negative values that round to zero keep their sign bit (and a block
    whose scale is zero has only 0x0 codes)."""
    k = np.zeros((1, 1, 1, 128), np.float32)
    k[..., 0] = 6.0
    k[..., 1] = -0.1
    k[..., 2] = -0.0
    k[..., 16] = 448.0
    k[..., 17] = -1e-4
    k[..., 33] = -0.0                 # an all-zero block holding -0: NVFP4 codes stay 0x0
    k = W.to_bf16_values(k)           # both sides see the same BF16 inputs
    for fmt in (kvq.NVFP4, kvq.FP8):
        c = kvq.KVCache(fmt, 1, 1, 1, 16, global_scales=[[1.0, 1.0]])
        o = oracle.OracleCache(fmt, 1, 1, 1, 128, 16, global_scales=[[1.0, 1.0]])
        c.append(0, to_dev(k), to_dev(k))
        o.append(0, k, k)
        assert_cache_bit_exact(c, o)


def test_multi_layer_independent():
    w = W.custom(kvq.NVFP4, 1, 2, 8, 200, seed=77)
    k = W.kv_tensor(w, "k", 0, 200)
    v = W.kv_tensor(w, "v", 0, 200)
    cache = kvq.KVCache(kvq.NVFP4, 3, 1, 2, 256)
    oc = oracle.OracleCache(kvq.NVFP4, 3, 1, 2, 128, 256)
    for layer, s in enumerate((1.0, 3.0, 0.25)):
        ks = W.to_bf16_values(k * s)      # x3 is not exact in BF16: feed both sides the rounded input
        cache.append(layer, to_dev(ks), to_dev(v))
        oc.append(layer, ks, v)
    for layer in range(3):
        assert_cache_bit_exact(cache, oc, layer)
    q = W.q_tensor(w)
    for layer in range(3):
        out = cache.decode_attention(layer, to_dev(q)).cpu().numpy()
        assert_attention_close(out, reference_attention(cache, q, layer), "layer %d" % layer)


def test_reset_recalibrates():
    w = W.custom(kvq.FP8, 1, 2, 8, 64, seed=88)
    k = W.kv_tensor(w, "k", 0, 64)
    v = W.kv_tensor(w, "v", 0, 64)
    cache, oc = make_pair(w, max_len=64)
    cache.append(0, to_dev(k), to_dev(v))
    cache.reset()
    cache.append(0, to_dev(2 * k), to_dev(v))
    oc.append(0, 2 * k, v)
    assert_cache_bit_exact(cache, oc)


def test_error_paths_leave_cache_unchanged():
    w = W.custom(kvq.NVFP4, 1, 2, 8, 60, seed=99)
    k = W.kv_tensor(w, "k", 0, 60)
    v = W.kv_tensor(w, "v", 0, 60)
    cache, oc = make_pair(w, max_len=64)
    q = to_dev(W.q_tensor(w))
    with pytest.raises(kvq.KVQError) as e:
        cache.decode_attention(0, q)
    assert e.value.status == 7           # EMPTY
    cache.append(0, to_dev(k), to_dev(v))
    oc.append(0, k, v)
    with pytest.raises(kvq.KVQError) as e:
        cache.append(0, to_dev(k[:, :, :5]), to_dev(v[:, :, :5]))
    assert e.value.status == 2           # CAPACITY
    assert_cache_bit_exact(cache, oc)
    with pytest.raises(kvq.KVQError) as e:
        cache.append(1, to_dev(k[:, :, :1]), to_dev(v[:, :, :1]))
    assert e.value.status == 1           # layer out of range
    bad_q = torch.zeros((1, 6, 128), dtype=torch.bfloat16, device="cuda")   # 6 % 2 ok, G=3
    cache.decode_attention(0, bad_q)     # G = 3 is fine
    with pytest.raises(kvq.KVQError) as e:
        cache.decode_attention(0, torch.zeros((1, 5, 128), dtype=torch.bfloat16, device="cuda"))
    assert e.value.status == 1
    with pytest.raises(kvq.KVQError) as e:
        cache.decode_attention(0, torch.zeros((1, 18, 128), dtype=torch.bfloat16, device="cuda"))
    assert e.value.status == 6           # G = 9 unsupported
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_decode_attention(cache.handle, 0, q, torch.empty((1, 8, 128), device="cuda"), small)
    assert e.value.status == 3           # WORKSPACE
    assert cache.device_status() == 0
