"""INT4, INT8 and INT2 g64 caches with compact group metadata (f16 S and an
i8 Z, or an i16 Z for INT8: 8 meta bytes per token and head instead of 16)
against the oracle's OracleCache(compact=True): codes, S and Z bit-exact,
the dequantization bit-exact, attention and the fused step within
tolerance.  Inputs include groups shifted away from zero (Z far from the
code range, still inside its integer type).
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_13_b200 as kvq
from quantized_kv_cache_13_b200 import workloads as W

from _support import assert_attention_close, to_dev

pytestmark = pytest.mark.gpu


def _inputs(rng, B, H, n):
    x = rng.standard_normal((B, H, n, 128)) * 0.5
    x = x + np.repeat(rng.choice([-1.5, 0.0, 1.5], size=(B, H, n, 2)), 64, axis=-1)
    return W.to_bf16_values(x.astype(np.float32))


def _unpack(fmt, c):
    """Canonical code bytes [B, H, n, bytes] -> one code per value [B, H, n, 128]."""
    if fmt == kvq.INT8:
        return c
    if fmt == kvq.INT4:
        return np.stack([c & 0xF, c >> 4], axis=-1).reshape(c.shape[:3] + (128,))
    return np.stack([(c >> s) & 3 for s in (0, 2, 4, 6)], axis=-1).reshape(c.shape[:3] + (128,))


def _check(cache, oc):
    torch.cuda.synchronize()
    assert cache.lengths(0) == oc.lengths(0)
    n, r = oc.lengths(0)
    for kv in (0, 1):
        codes, S16, Zc = oc.main_arrays(0, kv)
        c = cache.canonical_codes(0, kv, 0, n).cpu().numpy()
        assert np.array_equal(_unpack(cache.fmt, c), codes), kv
        raw = cache.raw(0, kv)
        assert np.array_equal(raw["meta_s16"][:, :, :n].cpu().numpy().view(np.uint16), S16.view(np.uint16))
        if cache.fmt == kvq.INT8:
            assert Zc.dtype == np.int16
            assert np.array_equal(raw["meta_z16"][:, :, :n].cpu().numpy(), Zc)
        else:
            assert np.array_equal(raw["meta_z8"][:, :, :n].cpu().numpy(), Zc)
            assert torch.count_nonzero(raw["meta"][:, :, :n, 6:]).item() == 0
        if r:
            assert np.array_equal(raw["ring"][:, :, :r].float().cpu().numpy(), oc.ring_tokens(0, kv))


@pytest.mark.parametrize("fmt", [kvq.INT4, kvq.INT8, kvq.INT2])
@pytest.mark.parametrize("R", [0, 128])
def test_compact_against_the_oracle(fmt, R):
    B, H, G, n, steps = 2, 2, 4, 700, 6
    rng = np.random.default_rng(9900 + R + 10 * fmt)
    k = _inputs(rng, B, H, n + steps)
    v = _inputs(rng, B, H, n + steps)
    cache = kvq.KVCache(fmt, 1, B, H, n + steps + 8, 128, 64, R, compact_meta=True)
    oc = oracle.OracleCache(fmt, 1, B, H, 128, n + steps + 8, 64, R, compact=True)
    pos = 0
    for step in [300, 1, 129, 7, 263]:
        cache.append(0, to_dev(k[:, :, pos:pos + step]), to_dev(v[:, :, pos:pos + step]))
        oc.append(0, k[:, :, pos:pos + step], v[:, :, pos:pos + step])
        pos += step
    _check(cache, oc)
    q = W.to_bf16_values(rng.standard_normal((B, H * G, 128)).astype(np.float32))
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert_attention_close(out, oc.decode_attention(0, q), "compact fmt %d R%d" % (fmt, R))
    for s in range(steps):
        out = cache.decode_step(0, to_dev(k[:, :, pos:pos + 1]), to_dev(v[:, :, pos:pos + 1]),
                                to_dev(q)).cpu().numpy()
        oc.append(0, k[:, :, pos:pos + 1], v[:, :, pos:pos + 1])
        pos += 1
        assert_attention_close(out, oc.decode_attention(0, q), "compact step %d" % s)
    _check(cache, oc)
    n_main = oc.lengths(0)[0]
    for kv in (0, 1):
        got = cache.dequantize(0, kv, 0, n_main).cpu().numpy()
        assert np.array_equal(got.view(np.uint32), oc.dequantize_main(0, kv).view(np.uint32))
    assert cache.device_status() == 0


@pytest.mark.parametrize("fmt", [kvq.INT8, kvq.INT2])
def test_compact_ragged_and_paged(fmt):
    """Compact metadata through the ragged / paged kernel: per-sequence
    appends of different lengths into a paged cache, against the oracle's
    one-sequence caches."""
    B, H, G = 3, 2, 2
    lens = [5, 800, 390]
    P = kvq.kvq_page_granularity(fmt)
    cache = kvq.KVCache(fmt, 1, B, H, 1600, 128, 64, 0, compact_meta=True, page_tokens=P, num_pages=12)
    rng = np.random.default_rng(9950 + fmt)
    q = W.to_bf16_values(rng.standard_normal((B, H * G, 128)).astype(np.float32))
    ref = np.zeros((B, H * G, 128))
    for b, n in enumerate(lens):
        k = _inputs(rng, 1, H, n)
        v = _inputs(rng, 1, H, n)
        cache.append_seq(0, b, to_dev(k[0]), to_dev(v[0]))
        one = oracle.OracleCache(fmt, 1, 1, H, 128, 1600, 64, 0, compact=True)
        one.append(0, k, v)
        for kv in (0, 1):
            codes, S16, Zc = one.main_arrays(0, kv)
            got = cache.seq_canonical_codes(0, kv, b, n).cpu().numpy()
            assert np.array_equal(_unpack(fmt, got), codes), (b, kv)
        ref[b] = one.decode_attention(0, q[b:b + 1])[0]
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert_attention_close(out, ref, "compact ragged paged")
    assert cache.device_status() == 0
