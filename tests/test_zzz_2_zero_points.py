"""Zero points outside 0 .. 2^bits - 1 in the INT formats' decode attention.

A group whose values are all positive has Z = round(-min/S) < 0, and one
whose values are all negative has Z above the top code.  The PV product of
the INT formats subtracts the zero-point term sum_t (1024 + Z_t) S_t P_t
with an FP16 operand, which has to hold such Z too.  Every token here has
groups shifted by -2, 0 or +2 (about 7 standard deviations), so Z falls
far on both sides of the code range: about -26 .. 40 for INT4 g64,
-41 .. 56 for INT4 g32, -480 .. 780 for INT8 and -5 .. 9 for INT2.  All of
these lie where 1024 + Z is exact in FP16.  Codes, S and Z must match the oracle bit
for bit and the attention output the oracle's within the tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_13_b200 as kvq

from _support import (assert_attention_close, assert_cache_bit_exact, reference_attention,
                      to_dev)

pytestmark = pytest.mark.gpu


def _shifted(rng, B, H, L, group):
    x = 0.3 * rng.standard_normal((B, H, L, 128))
    shift = rng.choice([-2.0, 0.0, 2.0], size=(B, H, L, 128 // group))
    x = x + np.repeat(shift, group, axis=-1)
    return torch.from_numpy(x.astype(np.float32)).bfloat16().float().numpy()


@pytest.mark.parametrize("fmt,grp,R", [(kvq.INT4, 64, 0), (kvq.INT4, 32, 128), (kvq.INT8, 64, 0),
                                       (kvq.INT8, 64, 128), (kvq.INT2, 64, 0)])
def test_zero_points_outside_the_code_range(fmt, grp, R):
    B, H, G, L = 2, 2, 4, 700
    rng = np.random.default_rng(7700 + 10 * fmt + grp + R)
    k = _shifted(rng, B, H, L, grp)
    v = _shifted(rng, B, H, L, grp)
    cache = kvq.KVCache(fmt, 1, B, H, L + 8, 128, grp, R)
    oc = oracle.OracleCache(fmt, 1, B, H, 128, L + 8, grp, R)
    cache.append(0, to_dev(k), to_dev(v))
    oc.append(0, k, v)
    assert_cache_bit_exact(cache, oc)
    n = oc.lengths(0)[0]
    Z = oc.main_arrays(0, 1)[2][:, :, :n]
    assert Z.min() < 0 and Z.max() > (3 if fmt == kvq.INT2 else 15 if fmt == kvq.INT4 else 255)
    q = torch.from_numpy(rng.standard_normal((B, H * G, 128)).astype(np.float32)).bfloat16().float().numpy()
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert np.isfinite(out).all()
    assert_attention_close(out, reference_attention(cache, q), "zero points fmt %d g%d R%d" % (fmt, grp, R))
    # and one fused step
    k1 = _shifted(rng, B, H, 1, grp)
    v1 = _shifted(rng, B, H, 1, grp)
    out1 = cache.decode_step(0, to_dev(k1), to_dev(v1), to_dev(q)).cpu().numpy()
    oc.append(0, k1, v1)
    assert_cache_bit_exact(cache, oc)
    assert_attention_close(out1, reference_attention(cache, q), "zero points, fused step")
    assert cache.device_status() == 0


@pytest.mark.parametrize("fmt", [kvq.INT4, kvq.INT8, kvq.INT2])
def test_constant_groups(fmt):
    """Groups whose 64 values are all equal (S = |value|, Z = -1 or 1, every
    code 0) and all-zero groups (S = 1, Z = 0) next to ordinary ones: codes,
    S and Z bit-exact, the reconstruction exact, attention within tolerance."""
    B, H, G, L = 1, 2, 4, 300
    rng = np.random.default_rng(7800 + fmt)
    k = torch.from_numpy(rng.standard_normal((B, H, L, 128)).astype(np.float32)).bfloat16().float().numpy()
    v = k[:, :, ::-1].copy()
    k[:, :, 0::3, :64] = 1.5          # constant positive group
    k[:, :, 1::3, 64:] = -0.75        # constant negative group
    v[:, :, 2::3, :64] = 0.0          # all-zero group
    cache = kvq.KVCache(fmt, 1, B, H, L + 8, 128, 64, 0)
    oc = oracle.OracleCache(fmt, 1, B, H, 128, L + 8, 64, 0)
    cache.append(0, to_dev(k), to_dev(v))
    oc.append(0, k, v)
    assert_cache_bit_exact(cache, oc)
    for kv, x in ((0, k), (1, v)):
        got = cache.dequantize(0, kv, 0, L).cpu().numpy()
        g = x.reshape(x.shape[:3] + (2, 64))
        const = g.min(-1) == g.max(-1)
        assert const.any()
        exact = np.repeat(const, 64, axis=-1)
        assert np.array_equal(got[exact], x[exact])
    q = torch.from_numpy(rng.standard_normal((B, H * G, 128)).astype(np.float32)).bfloat16().float().numpy()
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert_attention_close(out, reference_attention(cache, q), "constant groups fmt %d" % fmt)
