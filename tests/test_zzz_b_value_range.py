"""Attention accuracy at large value magnitudes, against the oracle.

The P.V product uses FP16 probabilities (2^-11 relative rounding each); the
softmax denominators are summed from the same FP16 values (an MMA with an
all-ones operand), so the output is an exactly normalised weighted mean of
the values and its error is bounded by 2^-10 of the values' spread around
it, not by their magnitude.  Checked at the required tolerance (max-abs 1e-2, rel-L2 2e-3) for NVFP4
and FP8, and at the bound stated for the INT formats (see check):

- V with the outlier channels of the 32K workload's K (lognormal(0, 0.5)
  per channel, 2 % of the channels x8), times 3: |V| about 100;
- a dominant key (its score tens of nats above the rest) whose value is
  about 100: the output equals that value;
- queries of magnitude about 1000 (Q' = q * softmax_scale * log2(e) stays
  far inside the FP16 range)."""
import math

import numpy as np
import pytest

import quantized_kv_cache_13_b200 as kvq
from quantized_kv_cache_13_b200 import workloads as W

from _support import ATOL, RTOL_L2, assert_attention_close, make_pair, reference_attention, to_dev

pytestmark = pytest.mark.gpu

FMTS = [kvq.NVFP4, kvq.FP8, kvq.INT4, kvq.INT8, kvq.INT2]


def check(fmt, cache, out, ref, what):
    """NVFP4 / FP8: the required tolerance (max-abs 1e-2, rel-L2 2e-3).  The INT formats multiply each
    FP16 probability by its group's scale S in FP16, one more rounding of
    2^-11 per weight: with the bound stated in kvq.h, 2^-10 max|v - out| +
    2^-11 max|v|, which is below 2^-9 max|v| over the dequantized values (the
    required max-abs as a floor), and the required rel-L2."""
    if fmt not in kvq.INT_AFFINE:
        assert_attention_close(out, ref, what)
        return
    n = cache.lengths(0)[0]
    vmax = float(np.abs(cache.dequantize(0, 1, 0, n).cpu().numpy()).max())
    err = np.abs(out.astype(np.float64) - ref).max()
    rel = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert np.all(np.isfinite(out)), what
    assert err <= max(ATOL, 2.0 ** -9 * vmax), (what, err, vmax)
    assert rel <= RTOL_L2, (what, rel)


@pytest.mark.parametrize("fmt", FMTS)
def test_value_outlier_channels(fmt):
    B, H, G, L = 2, 2, 4, 3000
    w = W.custom(fmt, B, H, H * G, L, seed=13000 + fmt, k_dist="lognormal_outlier",
                 v_dist="lognormal_outlier")
    k = W.kv_tensor(w, "k", 0, L)
    v = W.to_bf16_values(3.0 * W.kv_tensor(w, "v", 0, L))
    assert np.abs(v).max() > 60
    cache, oc = make_pair(w, max_len=L + 8)
    cache.append(0, to_dev(k), to_dev(v))
    oc.append(0, k, v)
    q = W.q_tensor(w)
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    check(fmt, cache, out, reference_attention(cache, q), "value outliers fmt %d" % fmt)
    assert cache.device_status() == 0


@pytest.mark.parametrize("fmt", FMTS)
def test_dominant_key_with_a_large_value(fmt):
    """Key j0 of every unit is 4 in every dim and each query 1: its score is
    4 * 128 / sqrt(128) = 45, tens of nats above the N(0,1) keys; its value
    is about 100.  The output is that key's (dequantized) value."""
    B, H, G, L = 2, 2, 4, 1537
    w = W.custom(fmt, B, H, H * G, L, seed=13100 + fmt)
    k = W.kv_tensor(w, "k", 0, L)
    v = W.kv_tensor(w, "v", 0, L)
    j0 = 1000
    k[:, :, j0] = 4.0
    rng = np.random.default_rng(13200 + fmt)
    v[:, :, j0] = W.to_bf16_values((96.0 + 4.0 * rng.standard_normal((B, H, 128))).astype(np.float32))
    cache, oc = make_pair(w, max_len=L + 8)
    cache.append(0, to_dev(k), to_dev(v))
    oc.append(0, k, v)
    q = np.ones((B, H * G, 128), np.float32)
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    ref = reference_attention(cache, q)
    assert np.abs(ref).max() > 80
    check(fmt, cache, out, ref, "dominant key fmt %d" % fmt)
    assert cache.device_status() == 0


@pytest.mark.parametrize("fmt", [kvq.NVFP4, kvq.INT4])
def test_large_queries(fmt):
    B, H, G, L = 2, 2, 4, 2049
    w = W.custom(fmt, B, H, H * G, L, seed=13300 + fmt)
    k = W.kv_tensor(w, "k", 0, L)
    v = W.kv_tensor(w, "v", 0, L)
    cache, oc = make_pair(w, max_len=L + 8)
    cache.append(0, to_dev(k), to_dev(v))
    oc.append(0, k, v)
    q = W.to_bf16_values(1000.0 * W.q_tensor(w))
    assert np.abs(q).max() * (1 / math.sqrt(128)) * math.log2(math.e) < 65504
    out = cache.decode_attention(0, to_dev(q)).cpu().numpy()
    assert_attention_close(out, reference_attention(cache, q), "large q fmt %d" % fmt)
    assert cache.device_status() == 0
