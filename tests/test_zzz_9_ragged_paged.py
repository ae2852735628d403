"""Sequences of different lengths (a ragged batch) and paged main-cache
planes, against the oracle's ragged batch (B independent one-sequence
caches sharing each layer's per-tensor scale).

Checked per sequence: lengths, codes / scales / zero points and ring
bit-exact (gathered through the block table for a paged cache), attention
within the required tolerance against the oracle's attention over the
CUDA cache's own codes and against the oracle cache; empty sequences give
0; fused decode steps with per-sequence positions (and the ring-fill
fallback); per-sequence reset, truncate and dequantize; the page pool
(assignment, reuse after reset, exhaustion)."""
import math

import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_13_b200 as kvq
from quantized_kv_cache_13_b200 import workloads as W

from _support import assert_attention_close, to_dev

pytestmark = pytest.mark.gpu

D = 128


def _grp(fmt):
    return 64 if fmt in kvq.INT_AFFINE else 0


def _kv(seed, H, n, dist="normal"):
    w = W.custom(kvq.NVFP4, 1, H, H, max(n, 1), seed=seed, k_dist=dist, v_dist=dist)
    return W.kv_tensor(w, "k", 0, n)[0], W.kv_tensor(w, "v", 0, n)[0]   # [H, n, D]


def _q(seed, B, Hq):
    w = W.custom(kvq.NVFP4, B, 1, Hq, 1, seed=seed)
    return W.q_tensor(w)


def _seq_arrays(cache, layer, kv, seq, n):
    """Main-cache arrays of one sequence shaped like the oracle's [1, H, n, ...]."""
    codes = cache.seq_canonical_codes(layer, kv, seq, n).cpu().numpy()
    raw = cache.seq_raw(layer, kv, seq, n)
    if cache.fmt == kvq.NVFP4:
        return (codes, raw["meta"].cpu().numpy())
    if cache.fmt == kvq.FP8:
        return (codes,)
    meta = raw["meta"].cpu()
    return (codes, meta[..., 0].contiguous().view(torch.float32).numpy(), meta[..., 1].contiguous().numpy())


def _scale(cache, layer, kv):
    raw = cache.raw(layer, kv)
    return float(raw["scale"].cpu().numpy()[0]) if "scale" in raw else None


def assert_seq_bit_exact(cache, rc, layer=0):
    torch.cuda.synchronize()
    for b in range(cache.batch):
        assert cache.seq_lengths(layer, b) == rc.lengths(layer, b), b
        n, r = rc.lengths(layer, b)
        for kv in (0, 1):
            if cache.fmt not in kvq.INT_AFFINE and rc.scale(layer, kv) is not None:
                assert np.float32(_scale(cache, layer, kv)) == np.float32(rc.scale(layer, kv))
            if n:
                ours = _seq_arrays(cache, layer, kv, b, n)
                ref = rc.main_arrays(layer, kv, b)
                for name, a, e in zip(("codes", "meta", "zero"), ours, ref):
                    if a.dtype == np.float32:
                        a, e = a.view(np.uint32), np.asarray(e, np.float32).view(np.uint32)
                    assert np.array_equal(a, e), (b, kv, name)
            if r:
                ring = cache.raw(layer, kv)["ring"][b, :, :r].float().cpu().numpy()
                assert np.array_equal(ring, rc.ring_tokens(layer, kv, b)[0]), (b, kv)


def reference_ragged(cache, q, layer=0):
    """Oracle attention over the oracle's dequantization of the CUDA cache's
    own codes, per sequence (0 for an empty one)."""
    B, Hq = q.shape[0], q.shape[1]
    H = cache.kv_heads
    G = Hq // H
    out = np.zeros((B, Hq, D), np.float64)
    grp = cache.group_size or 16
    for b in range(B):
        n, r = cache.seq_lengths(layer, b)
        if n + r == 0:
            continue
        KV = []
        for kv in (0, 1):
            parts = []
            if n:
                parts.append(oracle.dequantize_arrays(cache.fmt, _seq_arrays(cache, layer, kv, b, n),
                                                      _scale(cache, layer, kv), grp)[0])
            if r:
                parts.append(cache.raw(layer, kv)["ring"][b, :, :r].float().cpu().numpy())
            KV.append(np.concatenate(parts, axis=1))
        for h in range(H):
            out[b, h * G:(h + 1) * G] = oracle.attention(q[b, h * G:(h + 1) * G], KV[0][h], KV[1][h],
                                                         1.0 / math.sqrt(D))
    return out


def _pair(fmt, B, H, max_len, R=0, paged=False, num_pages=0):
    kw = {}
    if paged:
        kw = dict(page_tokens=2 * kvq.kvq_page_granularity(fmt), num_pages=num_pages)
    cache = kvq.KVCache(fmt, 1, B, H, max_len, D, _grp(fmt), R, **kw)
    rc = oracle.RaggedOracleCache(fmt, 1, B, H, D, max_len, _grp(fmt), R)
    return cache, rc


CASES = [(kvq.NVFP4, 0), (kvq.FP8, 0), (kvq.INT4, 128), (kvq.INT8, 64), (kvq.INT2, 128),
         (kvq.NVFP4, 64)]


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("fmt,R", CASES)
def test_ragged_append_and_attention(fmt, R, paged):
    B, H, G = 5, 2, 4
    lens = [0, 1, 383, 1200, 770]          # empty, one token, tile and page edges
    cache, rc = _pair(fmt, B, H, 1400, R, paged, num_pages=64)
    for b, n in enumerate(lens):
        if n:
            k, v = _kv(7000 + 13 * b + fmt, H, n, "lognormal_outlier" if b % 2 else "offset_uniform")
            cache.append_seq(0, b, to_dev(k), to_dev(v))
            rc.append_seq(0, b, k, v)
    assert_seq_bit_exact(cache, rc)
    q = _q(7100 + fmt, B, H * G)
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert np.all(out[0] == 0.0)
    assert_attention_close(out, reference_ragged(cache, q), "ragged")
    assert_attention_close(out, rc.decode_attention(0, q), "ragged vs the oracle cache")
    o2, lse = cache.decode_attention_lse(0, to_dev(q))
    lse = lse.cpu().numpy()
    assert np.all(np.isneginf(lse[0])) and np.all(np.isfinite(lse[1:]))
    assert np.array_equal(o2.cpu().numpy(), out)
    if paged:
        P = cache.layout(0, 0).page_tokens
        used = []
        for b, n in enumerate(lens):
            m = cache.seq_lengths(0, b)[0]
            tab = cache.block_table(b)
            k = (m + P - 1) // P
            assert all(p >= 0 for p in tab[:k]) and all(p == -1 for p in tab[k:]), (b, tab)
            used += tab[:k]
        assert len(used) == len(set(used))
    # dequantize one sequence against the oracle's dequantization
    n = cache.seq_lengths(0, 3)[0]
    if n:
        deq = cache.dequantize_seq(0, 1, 3, 0, n).cpu().numpy()
        ref = oracle.dequantize_arrays(fmt, rc.main_arrays(0, 1, 3), rc.scale(0, 1), cache.group_size or 16)[0]
        assert np.array_equal(deq.view(np.uint32), ref.astype(np.float32).view(np.uint32))
    assert cache.device_status() == 0


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("fmt,R", CASES)
def test_ragged_decode_steps(fmt, R, paged):
    """Fused decode steps with every sequence at its own position, against
    the oracle appending the same token to each sequence."""
    B, H, G = 3, 2, 3
    lens = [5, 380, 129 if R else 766]
    cache, rc = _pair(fmt, B, H, 1200, R, paged, num_pages=40)
    for b, n in enumerate(lens):
        k, v = _kv(7200 + 7 * b + fmt, H, n)
        cache.append_seq(0, b, to_dev(k), to_dev(v))
        rc.append_seq(0, b, k, v)
    steps = 70
    kn, vn = _kv(7300 + fmt, B * H, steps)
    kn = kn.reshape(B, H, steps, D)
    vn = vn.reshape(B, H, steps, D)
    for t in range(steps):
        q = _q(7400 + t, B, H * G)
        ks, vs = kn[:, :, t:t + 1], vn[:, :, t:t + 1]
        out = cache.decode_step(0, to_dev(ks), to_dev(vs), to_dev(q)).cpu().numpy()
        rc.append(0, ks, vs)
        if t % 10 == 0 or t == steps - 1:
            assert_seq_bit_exact(cache, rc)
            assert_attention_close(out, reference_ragged(cache, q), "step %d" % t)
            assert_attention_close(out, rc.decode_attention(0, q), "step %d vs the oracle" % t)
    assert cache.device_status() == 0


def test_ragged_batch_append_flush_truncate_reset():
    fmt, R, B, H = kvq.INT4, 32, 3, 2
    cache, rc = _pair(fmt, B, H, 600, R)
    for b, n in enumerate([10, 40, 0]):
        if n:
            k, v = _kv(7500 + b, H, n)
            cache.append_seq(0, b, to_dev(k), to_dev(v))
            rc.append_seq(0, b, k, v)
    # a batch append: every sequence at its own end, its own ring phase
    k, v = _kv(7510, B * H, 45)
    k, v = k.reshape(B, H, 45, D), v.reshape(B, H, 45, D)
    cache.append(0, to_dev(k), to_dev(v))
    rc.append(0, k, v)
    assert_seq_bit_exact(cache, rc)
    cache.flush_residual(0)
    rc.flush_residual(0)
    assert_seq_bit_exact(cache, rc)
    q = _q(7520, B, H)
    assert_attention_close(cache.decode_attention(0, to_dev(q)).cpu().numpy(),
                           rc.decode_attention(0, q), "after flush")
    # truncate one sequence, then every sequence longer than 50
    cache.truncate_seq(0, 1, 60)
    assert cache.seq_lengths(0, 1) == (60, 0)
    cache.truncate(0, 50)
    assert [sum(cache.seq_lengths(0, b)) for b in range(B)] == [50, 50, 45]
    # reset one sequence: the others keep their tokens, it restarts empty
    cache.seq_reset(1)
    rc.reset_seq(1)
    assert cache.seq_lengths(0, 1) == (0, 0)
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert np.all(out[1] == 0.0)
    assert_attention_close(out, reference_ragged(cache, q), "after reset")
    assert cache.device_status() == 0


def test_paged_pool_reuse_and_exhaustion():
    fmt, B, H = kvq.NVFP4, 3, 2
    P = kvq.kvq_page_granularity(fmt)
    cache = kvq.KVCache(fmt, 2, B, H, 4 * P, D, 0, 0, page_tokens=P, num_pages=5)
    k, v = _kv(7600, H, 2 * P + 1)
    cache.append_seq(0, 0, to_dev(k), to_dev(v))           # 3 pages
    assert cache.block_table(0)[:3] == [0, 1, 2]
    cache.append_seq(1, 0, to_dev(k[:, :P]), to_dev(v[:, :P]))   # layer 1 uses the same pages
    assert cache.block_table(0)[:4] == [0, 1, 2, -1]
    k2, v2 = _kv(7601, H, P + 1)
    cache.append_seq(0, 1, to_dev(k2), to_dev(v2))          # 2 pages: the pool is full
    with pytest.raises(kvq.KVQError) as e:
        cache.append_seq(0, 2, to_dev(k2[:, :1]), to_dev(v2[:, :1]))
    assert e.value.status == 2 and cache.seq_lengths(0, 2) == (0, 0)
    cache.seq_reset(0)                                     # its pages go back
    cache.append_seq(0, 2, to_dev(k2[:, :1]), to_dev(v2[:, :1]))
    assert cache.block_table(2)[0] in (0, 1, 2)
    # the reused page holds sequence 2's token, not sequence 0's old ones
    rc = oracle.RaggedOracleCache(fmt, 1, B, H, D, 4 * P)
    rc.append_seq(0, 0, k, v)      # calibrates like the CUDA cache's first append
    rc.reset_seq(0)
    rc.append_seq(0, 1, k2, v2)
    rc.append_seq(0, 2, k2[:, :1], v2[:, :1])
    assert_seq_bit_exact(cache, rc)
    q = _q(7602, B, H)
    assert_attention_close(cache.decode_attention(0, to_dev(q)).cpu().numpy(),
                           rc.decode_attention(0, q), "after reuse")
    cache.reset()
    assert cache.block_table(1) == [-1] * 4
    assert cache.device_status() == 0


@pytest.mark.parametrize("fmt", [kvq.NVFP4, kvq.FP8, kvq.INT8])
def test_paged_uniform_equals_contiguous(fmt):
    """The same uniform batch in a paged and a contiguous cache: identical
    codes; attention from the ragged kernel and from the uniform kernel
    agree within the tolerance."""
    B, H, G, n = 4, 2, 4, 1537
    w = W.custom(fmt, B, H, H * G, n, seed=7700 + fmt)
    k, v = W.kv_tensor(w, "k", 0, n), W.kv_tensor(w, "v", 0, n)
    a = kvq.KVCache(fmt, 1, B, H, n + 8, D, _grp(fmt), 0)
    p = kvq.KVCache(fmt, 1, B, H, n + 8, D, _grp(fmt), 0,
                    page_tokens=kvq.kvq_page_granularity(fmt), num_pages=B * 20)
    a.append(0, to_dev(k), to_dev(v))
    p.append(0, to_dev(k), to_dev(v))
    torch.cuda.synchronize()
    for b in range(B):
        for kv in (0, 1):
            assert torch.equal(a.seq_canonical_codes(0, kv, b, n), p.seq_canonical_codes(0, kv, b, n))
    q = W.q_tensor(w)
    oa = a.decode_attention(0, to_dev(q)).cpu().numpy()
    op = p.decode_attention(0, to_dev(q)).cpu().numpy()
    assert_attention_close(op, oa.astype(np.float64), "paged vs contiguous")
    oc = oracle.OracleCache(fmt, 1, B, H, D, n + 8, _grp(fmt), 0)
    oc.append(0, k, v)
    assert_attention_close(op, oc.decode_attention(0, q), "paged vs the oracle")
    assert a.device_status() == 0 and p.device_status() == 0
