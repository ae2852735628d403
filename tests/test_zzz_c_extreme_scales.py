"""Quantized codes at extreme magnitudes and scales, against the oracle.

The bulk append kernels form each code from the correctly rounded quotient
x / d computed without a division (a reciprocal product with one FMA
correction), which is exact only while the residual cannot underflow and
the product cannot overflow; outside that range they divide.  These inputs
reach both edges on purpose:

- tokens whose magnitudes span 2^-128 (BF16 subnormals) to 2^40, so group
  and block scales fall below 2^-92 (the divided path) or sit near it;
- caller-given NVFP4 / FP8 scales of 2^-100, so that quotients overflow
  binary32 and every such code must saturate like the IEEE quotient does;
- compact INT metadata (binary16 S, saturated at 65504) with values up to
  about 1e11, whose quotients pass 2^22, and values so small that S is
  raised to the binary16 floor of 2^-24.

Codes, scales and zero points must match bit for bit; the appends come in
chunks of different lengths so the bulk kernels and the per-token kernel
both run."""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_13_b200 as kvq
from quantized_kv_cache_13_b200 import workloads as W

from _support import assert_cache_bit_exact, make_pair, to_dev

pytestmark = pytest.mark.gpu

CHUNKS = (64, 1, 95, 33, 7)   # 200 tokens: bulk launches, odd starts, a single token


def _spanning_tokens(rng, B, H, n, exps):
    """N(0, 1) tokens, each scaled by 2^e for an e drawn from exps."""
    e = rng.choice(np.asarray(exps, np.float64), size=(B, H, n, 1))
    x = rng.standard_normal((B, H, n, 128)) * np.exp2(e)
    return W.to_bf16_values(x.astype(np.float32))


def _append_all(cache, oc, k, v):
    pos = 0
    for step in CHUNKS:
        cache.append(0, to_dev(k[:, :, pos:pos + step]), to_dev(v[:, :, pos:pos + step]))
        oc.append(0, k[:, :, pos:pos + step], v[:, :, pos:pos + step])
        pos += step


@pytest.mark.parametrize("fmt", [kvq.NVFP4, kvq.FP8, kvq.INT4, kvq.INT8, kvq.INT2])
@pytest.mark.parametrize("scales", ["calibrated", "given_1", "given_tiny"])
def test_codes_across_magnitudes(fmt, scales):
    if fmt in kvq.INT_AFFINE and scales != "calibrated":
        pytest.skip("the affine formats have no per-tensor scale")
    B, H, n = 2, 2, sum(CHUNKS)
    rng = np.random.default_rng(13100 + 7 * fmt + len(scales))
    exps = [-128, -112, -96, -91, -60, 0, 40]
    k = _spanning_tokens(rng, B, H, n, exps)
    v = _spanning_tokens(rng, B, H, n, exps)
    gs = {"calibrated": None, "given_1": [[1.0, 1.0]],
          "given_tiny": [[2.0 ** -100, 2.0 ** -100]]}[scales]
    w = W.custom(fmt, B, H, H, n, seed=1)
    cache, oc = make_pair(w, max_len=n + 8, global_scales=gs)
    _append_all(cache, oc, k, v)
    assert_cache_bit_exact(cache, oc)
    assert cache.device_status() == 0


def _unpack(fmt, c):
    """Canonical code bytes [B, H, n, bytes] -> one code per value."""
    if fmt == kvq.INT8:
        return c
    if fmt == kvq.INT4:
        return np.stack([c & 0xF, c >> 4], axis=-1).reshape(c.shape[:3] + (128,))
    return np.stack([(c >> s) & 3 for s in (0, 2, 4, 6)], axis=-1).reshape(c.shape[:3] + (128,))


@pytest.mark.parametrize("fmt", [kvq.INT4, kvq.INT8, kvq.INT2])
def test_compact_metadata_at_saturated_and_floor_scales(fmt):
    B, H, n = 2, 2, sum(CHUNKS)
    rng = np.random.default_rng(13200 + fmt)
    # 2^36.5 ~ 1e11: S saturates at 65504 and |x / S| reaches ~7e6 > 2^22
    # (still far below 2^31); 2^-30: S32 < 2^-24, raised to the floor
    exps = [-30, 0, 20, 30, 36.5]
    k = _spanning_tokens(rng, B, H, n, exps)
    v = _spanning_tokens(rng, B, H, n, exps)
    cache = kvq.KVCache(fmt, 1, B, H, n + 8, 128, 64, 0, compact_meta=True)
    oc = oracle.OracleCache(fmt, 1, B, H, 128, n + 8, 64, 0, compact=True)
    _append_all(cache, oc, k, v)
    torch.cuda.synchronize()
    assert cache.lengths(0) == oc.lengths(0)
    for kv in (0, 1):
        codes, S16, Zc = oc.main_arrays(0, kv)
        got = _unpack(fmt, cache.canonical_codes(0, kv, 0, n).cpu().numpy())
        bad = np.argwhere(got != codes)
        assert bad.size == 0, "codes differ at %d places, first %s" % (len(bad), bad[0].tolist())
        raw = cache.raw(0, kv)
        assert np.array_equal(raw["meta_s16"][:, :, :n].cpu().numpy().view(np.uint16), S16.view(np.uint16))
        z = raw["meta_z16"] if fmt == kvq.INT8 else raw["meta_z8"]
        assert np.array_equal(z[:, :, :n].cpu().numpy(), Zc)
    # the saturated groups do reach the clamp on both sides
    assert (np.abs(oc.main_arrays(0, 0)[1].astype(np.float32)) == 65504.0).any()
    assert cache.device_status() == 0
