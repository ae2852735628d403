"""The INT2 affine format on the GPU against the oracle.

INT2 is the 2-bit setting of the affine scheme: the INT2 row of the
long-text KV-cache article's section 3.1 table, and with a ring of one 8K
chunk, the age tiers of its section 4.2.  Quantize-append, ring, flush and
dequantize are checked bit for bit: codes, S, Z and ring contents.  Decode
attention over an INT2 cache is refused with UNSUPPORTED until its kernel
exists.  (Kept after the main parity files.)
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_13_b200 as kvq
from quantized_kv_cache_13_b200 import workloads as W

from _support import assert_cache_bit_exact, make_pair, to_dev

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


def test_int2_layout_and_attention_refused():
    w = W.custom(kvq.INT2, 1, 2, 4, 40, seed=5302)
    cache, oc = make_pair(w, max_len=64)
    k = W.kv_tensor(w, "k", 0, 40)
    v = W.kv_tensor(w, "v", 0, 40)
    cache.append(0, to_dev(k), to_dev(v))
    torch.cuda.synchronize()
    lay = cache.layout(0, 0)
    assert lay.code_bytes == 32 and lay.meta_bytes == 16 and not lay.global_scale
    assert kvq.kvq_workspace_bytes(cache.handle, 4) == 0
    q = to_dev(W.q_tensor(w))
    with pytest.raises(kvq.KVQError) as e:
        cache.decode_attention(0, q)
    assert e.value.status == 6
    with pytest.raises(kvq.KVQError) as e:
        cache.decode_step(0, to_dev(k[:, :, :1]), to_dev(v[:, :, :1]), q)
    assert e.value.status == 6
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_decode_attention_noalloc(cache.handle, 0, q, torch.empty(q.shape, device="cuda"))
    assert e.value.status == 6
    assert cache.lengths(0) == (40, 0)
    assert cache.device_status() == 0
