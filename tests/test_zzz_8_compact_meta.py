"""INT4 g64 caches with compact group metadata (f16 S, i8 Z: 8 meta bytes
per token and head instead of 16) against the oracle's
OracleCache(compact=True): codes, S and Z bit-exact, the dequantization
bit-exact, attention and the fused step within tolerance.  Inputs include
groups shifted away from zero (Z far from the code range, still inside
int8).
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


def _check(cache, oc):
    torch.cuda.synchronize()
    assert cache.lengths(0) == oc.lengths(0)
    n, r = oc.lengths(0)
    for kv in (0, 1):
        codes, S16, Z8 = oc.main_arrays(0, kv)
        c = cache.canonical_codes(0, kv, 0, n).cpu().numpy()
        unpacked = np.stack([c & 0xF, c >> 4], axis=-1).reshape(c.shape[:3] + (128,))
        assert np.array_equal(unpacked, codes), kv
        raw = cache.raw(0, kv)
        assert np.array_equal(raw["meta_s16"][:, :, :n].cpu().numpy().view(np.uint16), S16.view(np.uint16))
        assert np.array_equal(raw["meta_z8"][:, :, :n].cpu().numpy(), Z8)
        assert torch.count_nonzero(raw["meta"][:, :, :n, 6:]).item() == 0
        if r:
            assert np.array_equal(raw["ring"][:, :, :r].float().cpu().numpy(), oc.ring_tokens(0, kv))


@pytest.mark.parametrize("R", [0, 128])
def test_compact_int4_against_the_oracle(R):
    B, H, G, n, steps = 2, 2, 4, 700, 6
    rng = np.random.default_rng(9900 + R)
    k = _inputs(rng, B, H, n + steps)
    v = _inputs(rng, B, H, n + steps)
    cache = kvq.KVCache(kvq.INT4, 1, B, H, n + steps + 8, 128, 64, R, compact_meta=True)
    oc = oracle.OracleCache(oracle.INT4, 1, B, H, 128, n + steps + 8, 64, R, compact=True)
    pos = 0
    for step in [300, 1, 129, 7, 263]:
        cache.append(0, to_dev(k[:, :, pos:pos + step]), to_dev(v[:, :, pos:pos + step]))
        oc.append(0, k[:, :, pos:pos + step], v[:, :, pos:pos + step])
        pos += step
    _check(cache, oc)
    q = W.to_bf16_values(rng.standard_normal((B, H * G, 128)).astype(np.float32))
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert_attention_close(out, oc.decode_attention(0, q), "compact R%d" % R)
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
