"""The INT2 affine format on the GPU against the oracle.

INT2 is the 2-bit setting of the affine scheme: the INT2 row of the
long-text KV-cache article's section 3.1 table, and with a ring of one 8K
chunk, the age tiers of its section 4.2.  Quantize-append, ring, flush and
dequantize are checked bit for bit: codes, S, Z and ring contents.  Decode
attention (groups of 64 and of 32) is checked against the oracle's binary64
attention over the dequantized cache within the attention tolerance, as is
the fused decode step.  Groups of 32 with a 256-token ring are the debug
configuration of the article's section 4.3.
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


@pytest.mark.parametrize("grp,R,dist", [(64, 0, "normal"), (64, 128, "offset_uniform"),
                                        (32, 48, "lognormal_outlier"), (32, 0, "offset_uniform")])
def test_int2_append_ring_flush_dequantize(grp, R, dist):
    L = 700
    w = W.custom(kvq.INT2, 2, 3, 3, L, seed=5200 + grp + R, group_size=grp, residual_length=R,
                 k_dist=dist, v_dist=dist)
    k = W.kv_tensor(w, "k", 0, L)
    v = W.kv_tensor(w, "v", 0, L)
    cache, oc = make_pair(w, max_len=800)
    # a bulk prefill, then ragged pieces and single tokens
    pos = 0
    for step in [300, 1, 1, 5, 127, 129, 1, 7, 129]:
        cache.append(0, to_dev(k[:, :, pos:pos + step]), to_dev(v[:, :, pos:pos + step]))
        oc.append(0, k[:, :, pos:pos + step], v[:, :, pos:pos + step])
        pos += step
        assert cache.lengths(0) == oc.lengths(0)
    assert pos == L
    assert_cache_bit_exact(cache, oc)
    cache.flush_residual(0)
    oc.flush_residual(0)
    assert_cache_bit_exact(cache, oc)
    assert cache.lengths(0) == (L, 0)
    for kv in (0, 1):
        got = cache.dequantize(0, kv, 37, 600).cpu().numpy()
        ref = oc.dequantize_main(0, kv)[:, :, 37:637]
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_int2_age_tiers_chunk_ring():
    """INT2 with an 8192-token ring: the newest chunk stays BF16, a completed
    chunk is quantized in one flush."""
    R, n = 8192, 8192 + 300
    w = W.custom(kvq.INT2, 1, 2, 2, n, seed=5301, residual_length=R)
    k = W.kv_tensor(w, "k", 0, n)
    v = W.kv_tensor(w, "v", 0, n)
    cache, oc = make_pair(w, max_len=n + 16)
    cache.append(0, to_dev(k[:, :, :5000]), to_dev(v[:, :, :5000]))
    oc.append(0, k[:, :, :5000], v[:, :, :5000])
    assert cache.lengths(0) == (0, 5000)
    cache.append(0, to_dev(k[:, :, 5000:]), to_dev(v[:, :, 5000:]))
    oc.append(0, k[:, :, 5000:], v[:, :, 5000:])
    assert cache.lengths(0) == oc.lengths(0) == (8192, 300)
    assert_cache_bit_exact(cache, oc)
    q = W.q_tensor(w)
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert_attention_close(out, reference_attention(cache, q), "int2 + 8192-token ring")


@pytest.mark.parametrize("R,L,G", [(0, 40, 4), (0, 1153, 8), (256, 1100, 1), (256, 750, 4)])
def test_int2_g32_attention_and_decode_steps(R, L, G):
    """Groups of 32 (with the section-4.3 debug ring of 256 tokens): layout,
    codes bit-exact, attention and fused decode steps within tolerance."""
    w = W.custom(kvq.INT2, 2, 2, 2 * G, L + 40, seed=5302 + L, group_size=32, residual_length=R,
                 k_dist="offset_uniform", v_dist="lognormal_outlier")
    cache, oc = make_pair(w, max_len=L + 48)
    k = W.kv_tensor(w, "k", 0, L + 40)
    v = W.kv_tensor(w, "v", 0, L + 40)
    cache.append(0, to_dev(k[:, :, :L]), to_dev(v[:, :, :L]))
    oc.append(0, k[:, :, :L], v[:, :, :L])
    torch.cuda.synchronize()
    lay = cache.layout(0, 0)
    assert lay.code_bytes == 32 and lay.meta_bytes == 32 and not lay.global_scale
    assert_cache_bit_exact(cache, oc)
    q = W.q_tensor(w)
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert_attention_close(out, reference_attention(cache, q), "int2 g32")
    assert_attention_close(out, oc.decode_attention(0, q), "int2 g32 vs the oracle cache")
    for t in range(L, L + 40):
        qt = W.q_tensor(w, t)
        o = cache.decode_step(0, to_dev(k[:, :, t:t + 1]), to_dev(v[:, :, t:t + 1]), to_dev(qt))
        oc.append(0, k[:, :, t:t + 1], v[:, :, t:t + 1])
        if t % 13 == 0 or t == L + 39:
            assert_cache_bit_exact(cache, oc)
            assert_attention_close(o.cpu().numpy(), oc.decode_attention(0, qt), "int2 g32 step %d" % t)
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    kvq.kvq_decode_attention_noalloc(cache.handle, 0, to_dev(q), out)
    assert_attention_close(out.cpu().numpy(), reference_attention(cache, q), "int2 g32 no-alloc")
    assert cache.device_status() == 0


def _prefill(w, cache, oc, n):
    k = W.kv_tensor(w, "k", 0, n)
    v = W.kv_tensor(w, "v", 0, n)
    cache.append(0, to_dev(k), to_dev(v))
    oc.append(0, k, v)


@pytest.mark.parametrize("R,dist,B,Hkv,G,L", [
    (0, "normal", 2, 2, 4, 1000),
    (128, "offset_uniform", 1, 3, 8, 1029),
    (128, "lognormal_outlier", 3, 1, 1, 777),
    (0, "offset_uniform", 2, 2, 2, 129),
])
def test_int2_attention_parity(R, dist, B, Hkv, G, L):
    w = W.custom(kvq.INT2, B, Hkv, Hkv * G, L, seed=5400 + L + G, residual_length=R,
                 k_dist=dist, v_dist=dist)
    cache, oc = make_pair(w, max_len=L + 64)
    _prefill(w, cache, oc, L)
    assert_cache_bit_exact(cache, oc)
    q = W.q_tensor(w)
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert_attention_close(out, reference_attention(cache, q), "int2 R%d G%d L%d" % (R, G, L))
    assert_attention_close(out, oc.decode_attention(0, q), "int2 vs the oracle's cache")
    assert cache.device_status() == 0


@pytest.mark.parametrize("L", [1, 15, 16, 17, 383, 384, 385, 767, 768, 769])
def test_int2_ragged_lengths(L):
    w = W.custom(kvq.INT2, 2, 2, 8, L, seed=5500 + L)
    cache, oc = make_pair(w, max_len=max(300, L))
    _prefill(w, cache, oc, L)
    q = W.q_tensor(w)
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert_attention_close(out, reference_attention(cache, q), "int2 ragged L=%d" % L)


@pytest.mark.parametrize("R,L,steps", [(0, 380, 7), (16, 40, 30), (128, 1000, 6)])
def test_int2_decode_step(R, L, steps):
    B, H, G = 2, 3, 2
    w = W.custom(kvq.INT2, B, H, H * G, L + steps, seed=5600 + L, residual_length=R)
    k = W.kv_tensor(w, "k", 0, L + steps)
    v = W.kv_tensor(w, "v", 0, L + steps)
    a = kvq.KVCache(kvq.INT2, 1, B, H, L + steps + 4, 128, 64, R)
    b = kvq.KVCache(kvq.INT2, 1, B, H, L + steps + 4, 128, 64, R)
    o = oracle.OracleCache(oracle.INT2, 1, B, H, 128, L + steps + 4, 64, R)
    for c in (a, b):
        c.append(0, to_dev(k[:, :, :L]), to_dev(v[:, :, :L]))
    o.append(0, k[:, :, :L], v[:, :, :L])
    for s in range(steps):
        kn, vn = k[:, :, L + s:L + s + 1], v[:, :, L + s:L + s + 1]
        q = to_dev(W.q_tensor(w, s))
        out_a = a.decode_step(0, to_dev(kn), to_dev(vn), q)
        b.append(0, to_dev(kn), to_dev(vn))
        out_b = b.decode_attention(0, q)
        o.append(0, kn, vn)
        assert a.lengths(0) == b.lengths(0) == o.lengths(0)
        assert_attention_close(out_a.cpu().numpy(), out_b.double().cpu().numpy(), "int2 step %d" % s)
    assert_cache_bit_exact(a, o)
    assert_cache_bit_exact(b, o)
    assert a.device_status() == 0


def test_int2_full_size_workload():
    """The INT2 workload (B4, MHA 32 heads, 16K context, g64, ring 128) at
    full size, checked like the other workloads on sampled units."""
    from test_gpu_configs import test_full_size_workload
    test_full_size_workload("mha_int2_16k", 1)
