"""Pins for the oracle's cache bookkeeping and the KV size formula (CPU only).

* Size formula and savings: the tables printed on
  "KV Cache量化实战：Model Optimizer为大模型长上下文省下50%显存" (savings
  table) and "KV缓存量化技术：提升大模型长文本生成效率" (section 1 and the
  section 3.1 table), stored under tests/golden/.
* Residual ring (section 2.2 of the second page): closed-form lengths after
  n appends, and bulk append = token-by-token append, bit for bit; a ring
  only delays the encoding of a token, never changes its codes.
* Scale recalibration every P tokens (section 3.1 of the NVFP4 KV-cache
  article): segment boundaries and the lag-one scale rule, pinned with
  inputs whose per-segment amax is planted as a power of two.
"""
import os

import numpy as np
import pytest

import oracle
from quantized_kv_cache_13_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
GiB = 1024 ** 3


def _rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def test_size_formula_matches_savings_table():
    rows = _rows("p2_savings_table.txt")
    table = [r for r in rows if len(r) == 4]
    for ctx, fp16, fp8, nvfp4 in table:
        ctx = int(ctx)
        assert oracle.kv_cache_bytes(32, 8, 128, ctx, 2) == float(fp16) * GiB
        assert oracle.kv_cache_bytes(32, 8, 128, ctx, 1) == float(fp8) * GiB
        assert oracle.kv_cache_bytes(32, 8, 128, ctx, 0.5) == float(nvfp4) * GiB
        # the table's -50 % / -75 %: 2x and 4x savings over FP16
        assert oracle.kv_cache_bytes(32, 8, 128, ctx, 2) / oracle.kv_cache_bytes(32, 8, 128, ctx, 1) == 2
        assert oracle.kv_cache_bytes(32, 8, 128, ctx, 2) / oracle.kv_cache_bytes(32, 8, 128, ctx, 0.5) == 4
    (ctx, conc, saving), = [r for r in rows if len(r) == 3]
    per_seq = oracle.kv_cache_bytes(32, 8, 128, int(ctx), 2) - oracle.kv_cache_bytes(32, 8, 128, int(ctx), 1)
    assert per_seq * int(conc) == float(saving) * GiB


def test_size_formula_matches_llama2_table():
    rows = _rows("p3_memory_table.txt")
    table = [r for r in rows if len(r) == 3 and not r[0].isdigit()]
    base = {r[0]: float(r[2]) for r in table}
    for name, bits, mem in table:
        ratio = oracle.kv_cache_bytes(32, 32, 128, 10000, int(bits) / 8) / oracle.kv_cache_bytes(32, 32, 128, 10000, 2)
        assert ratio == float(mem) / base["FP16"]
    (heads, dim, tokens, approx_gb), = [r for r in rows if r[0].isdigit()]
    b = oracle.kv_cache_bytes(32, int(heads), int(dim), int(tokens), 2)     # 32 layers, FP16
    assert abs(b / 1e9 - float(approx_gb)) / float(approx_gb) < 0.05


def test_storage_bytes_per_token():
    # K or V, one token, one KV head, head_dim 128
    assert oracle.cache_storage_bytes_per_token_head(oracle.NVFP4, 128) == 72
    assert oracle.cache_storage_bytes_per_token_head(oracle.INT4, 128, 64) == 80
    assert oracle.cache_storage_bytes_per_token_head(oracle.FP8, 128) == 128
    assert oracle.cache_storage_bytes_per_token_head(oracle.INT8, 128, 64) == 144
    assert oracle.cache_storage_bytes_per_token_head(oracle.INT2, 128, 64) == 48
    assert oracle.cache_storage_bytes_per_token_head(oracle.INT2, 128, 32) == 64
    # code bytes alone follow the 16 : 8 : 4 : 2 bits of the FP16 / INT8 /
    # INT4 / INT2 rows of the Llama-2 table (5.0 : 2.5 : 1.25 : 0.625 GB)
    codes = {f: oracle.cache_storage_bytes_per_token_head(f, 128, 128) - 8
             for f in (oracle.INT8, oracle.INT4, oracle.INT2)}
    assert [256 / codes[f] for f in (oracle.INT8, oracle.INT4, oracle.INT2)] == [2, 4, 8]


def _kv(seed, B, H, n, D=128):
    w = W.custom(oracle.INT4, B, H, H, n, seed)
    return W.kv_tensor(w, "k", 0, n), W.kv_tensor(w, "v", 0, n)


@pytest.mark.parametrize("n", [1, 5, 127, 128, 129, 300, 384])
def test_ring_lengths_closed_form(n):
    k, v = _kv(7, 1, 2, n)
    c = oracle.OracleCache(oracle.INT4, 1, 1, 2, 128, 1024, 64, 128)
    c.append(0, k, v)
    assert c.lengths(0) == (128 * (n // 128), n % 128)
    c.flush_residual(0)
    assert c.lengths(0) == (n, 0)


@pytest.mark.parametrize("fmt,R", [(oracle.NVFP4, 0), (oracle.FP8, 0), (oracle.INT4, 0), (oracle.INT4, 128),
                                   (oracle.INT4, 16), (oracle.INT8, 0), (oracle.INT8, 128),
                                   (oracle.INT2, 0), (oracle.INT2, 128), (oracle.INT2, 16),
                                   (oracle.NVFP4, 128), (oracle.FP8, 16)])
def test_bulk_append_equals_token_by_token(fmt, R):
    n = 300
    k, v = _kv(8, 2, 2, n)
    # calibrate both caches from the same first append
    gs = None
    if fmt not in oracle.INT_AFFINE:
        gs = [[oracle.global_scale(fmt, oracle.amax(k)), oracle.global_scale(fmt, oracle.amax(v))]]
    grp = 64 if fmt in oracle.INT_AFFINE else 0
    a = oracle.OracleCache(fmt, 1, 2, 2, 128, 512, grp, R, gs)
    b = oracle.OracleCache(fmt, 1, 2, 2, 128, 512, grp, R, gs)
    a.append(0, k, v)
    for t in range(n):
        b.append(0, k[:, :, t:t + 1], v[:, :, t:t + 1])
    assert a.lengths(0) == b.lengths(0)
    for kv in (0, 1):
        ma, mb = a.main_arrays(0, kv), b.main_arrays(0, kv)
        for x, y in zip(ma, mb):
            assert np.array_equal(x, y)
        assert np.array_equal(a.ring_tokens(0, kv), b.ring_tokens(0, kv))


def test_calibration_from_first_append_only():
    k, v = _kv(9, 1, 2, 64)
    c = oracle.OracleCache(oracle.NVFP4, 1, 1, 2, 128, 256)
    c.append(0, k[:, :, :32], v[:, :, :32])
    g = c.scale(0, 0)
    assert g == oracle.global_scale(oracle.NVFP4, oracle.amax(k[:, :, :32]))
    c.append(0, 10 * k[:, :, 32:], v[:, :, 32:])
    assert c.scale(0, 0) == g


def test_ring_tokens_kept_exact_and_attention_reads_both():
    """Ring tokens take part in attention at full precision; the quantized
    prefix through its dequantization."""
    k, v = _kv(10, 1, 1, 130)
    c = oracle.OracleCache(oracle.INT4, 1, 1, 1, 128, 512, 64, 128)
    c.append(0, k, v)
    assert c.lengths(0) == (128, 2)
    assert np.array_equal(c.ring_tokens(0, 0)[0, 0], k[0, 0, 128:])
    q = np.random.default_rng(0).standard_normal((1, 1, 128)).astype(np.float32)
    K = np.concatenate([c.dequantize_main(0, 0), k[:, :, 128:]], axis=2)
    V = np.concatenate([c.dequantize_main(0, 1), v[:, :, 128:]], axis=2)
    ref = oracle.attention(q[0], K[0, 0], V[0, 0])
    assert np.array_equal(c.decode_attention(0, q)[0], ref)


def test_capacity_and_format_checks():
    k, v = _kv(11, 1, 1, 10)
    c = oracle.OracleCache(oracle.FP8, 1, 1, 1, 128, 8)
    with pytest.raises(ValueError):
        c.append(0, k, v)
    with pytest.raises(ValueError):
        oracle.OracleCache(9, 1, 1, 1, 128, 8)
    # recalibration is defined for the per-tensor-scaled formats without a ring
    with pytest.raises(ValueError):
        oracle.OracleCache(oracle.NVFP4, 1, 1, 1, 128, 8, 16, 128, recalibrate_every=512)
    with pytest.raises(ValueError):
        oracle.OracleCache(oracle.INT4, 1, 1, 1, 128, 8, 64, 0, recalibrate_every=512)


@pytest.mark.parametrize("fmt", [oracle.NVFP4, oracle.FP8, oracle.INT4, oracle.INT8, oracle.INT2])
def test_ring_delays_encoding_but_not_codes(fmt):
    """Every format quantizes each token on its own (groups run along
    head_dim), so once the ring is flushed the main cache holds the very
    codes a ring-less cache holds."""
    n = 200
    k, v = _kv(12, 1, 2, n)
    gs = [[oracle.global_scale(fmt, oracle.amax(k)), oracle.global_scale(fmt, oracle.amax(v))]] \
        if fmt in (oracle.NVFP4, oracle.FP8) else None
    grp = 64 if fmt in oracle.INT_AFFINE else 0
    plain = oracle.OracleCache(fmt, 1, 1, 2, 128, 256, grp, 0, gs)
    ring = oracle.OracleCache(fmt, 1, 1, 2, 128, 256, grp, 64, gs)
    for t0 in range(0, n, 37):
        plain.append(0, k[:, :, t0:t0 + 37], v[:, :, t0:t0 + 37])
        ring.append(0, k[:, :, t0:t0 + 37], v[:, :, t0:t0 + 37])
    assert ring.lengths(0) == (192, 8)
    ring.flush_residual(0)
    for kv in (0, 1):
        for x, y in zip(plain.main_arrays(0, kv), ring.main_arrays(0, kv)):
            assert np.array_equal(x, y)


def test_nvfp4_ring_calibrates_on_first_append():
    k, v = _kv(13, 1, 1, 40)
    c = oracle.OracleCache(oracle.NVFP4, 1, 1, 1, 128, 256, 16, 32)
    c.append(0, k[:, :, :20], v[:, :, :20])
    assert c.lengths(0) == (0, 20)
    assert c.scale(0, 0) == oracle.global_scale(oracle.NVFP4, oracle.amax(k[:, :, :20]))
    c.append(0, k[:, :, 20:], v[:, :, 20:])
    assert c.lengths(0) == (32, 8)


# --------------------------------------------------------------------------
# Recalibration every P tokens
# --------------------------------------------------------------------------

P = 32


def _planted(seed, B, H, n, exps, M=3.0):
    """Tokens whose segment s (P tokens) is 2^exps[s] times a random block
    with |x| < M everywhere and M planted once among its first 8 tokens, so
    that the segment's amax over all batch rows and heads is exactly
    2^exps[s] * M."""
    rng = np.random.default_rng(seed)
    x = np.clip(rng.standard_normal((B, H, n, 128)), -2.9, 2.9).astype(np.float32)
    x = oracle._f32(np.asarray(__import__("torch").from_numpy(x).bfloat16().float()))
    for s in range((n + P - 1) // P):
        t0, t1 = s * P, min(n, (s + 1) * P)
        x[rng.integers(B), rng.integers(H), t0 + rng.integers(0, min(8, t1 - t0)), rng.integers(128)] = -M if s % 2 else M
        x[:, :, t0:t1] *= np.float32(2.0 ** exps[s])
    return x


@pytest.mark.parametrize("fmt", [oracle.NVFP4, oracle.FP8])
def test_recalibration_segments_and_lag_one_rule(fmt):
    """Segment s >= 1 is encoded with the scale of segment s-1's amax: with
    segment amaxes 2^e_s * M, the scales are 2^e_(s-1) * g(M) exactly and
    segment s's codes are those of (2^(e_s - e_(s-1)) * its block) at g(M)."""
    exps = [0, 0, 1, 3, 3, -2, 0]
    n = 7 * P - 5                                     # ragged last segment
    B, H = 2, 2
    k = _planted(14, B, H, n, exps)
    v = _planted(15, B, H, n, [-e for e in exps])
    c = oracle.OracleCache(fmt, 1, B, H, 128, 512, recalibrate_every=P)
    # a first append that spans two and a half segments, then ragged pieces
    for t0, t1 in [(0, 80), (80, 81), (81, 120), (120, n)]:
        c.append(0, k[:, :, t0:t1], v[:, :, t0:t1])
    assert c.lengths(0) == (n, 0)
    for kv, x, e in ((0, k, exps), (1, v, [-a for a in exps])):
        g0 = oracle.global_scale(fmt, oracle.amax(x[:, :, :80]))     # first append
        gM = oracle.global_scale(fmt, 3.0 * 2.0 ** e[0])
        assert g0 == max(gM, oracle.global_scale(fmt, 3.0 * 2.0 ** max(e[1], e[2])))
        segs = c.segment_scales(0, kv)
        assert [t for t, _ in segs] == [s * P for s in range(7)]
        assert segs[0][1] == g0
        for s in range(1, 7):
            assert segs[s][1] == np.float32(oracle.global_scale(fmt, 3.0) * 2.0 ** e[s - 1])
        codes = c.main_arrays(0, kv)
        for s in range(1, 7):
            t0, t1 = s * P, min(n, (s + 1) * P)
            block = x[:, :, t0:t1] * np.float32(2.0 ** -e[s - 1])      # exact rescale
            ref = c._encode(block, oracle.global_scale(fmt, 3.0))
            for a, b in zip(codes, ref):
                assert np.array_equal(a[:, :, t0:t1], b)
        # the dequantization applies each segment's own scale
        xh = c.dequantize_main(0, kv)
        for s in range(1, 7):
            t0, t1 = s * P, min(n, (s + 1) * P)
            ref = oracle.dequantize_arrays(fmt, tuple(a[:, :, t0:t1] for a in codes), segs[s][1], c.group)
            assert np.array_equal(xh[:, :, t0:t1], ref)


def test_recalibration_of_a_stationary_sequence_changes_nothing():
    """When every segment holds the same amax the renewed scales all equal
    the calibrated one, and the codes equal those of a frozen-scale cache."""
    n = 5 * P
    k = _planted(16, 1, 2, n, [0] * 5)
    v = _planted(17, 1, 2, n, [0] * 5)
    a = oracle.OracleCache(oracle.NVFP4, 1, 1, 2, 128, 256, recalibrate_every=P)
    b = oracle.OracleCache(oracle.NVFP4, 1, 1, 2, 128, 256)
    for t0 in range(0, n, 48):
        a.append(0, k[:, :, t0:t0 + 48], v[:, :, t0:t0 + 48])
        b.append(0, k[:, :, t0:t0 + 48], v[:, :, t0:t0 + 48])
    assert len(set(sc for _, sc in a.segment_scales(0, 0))) == 1
    for kv in (0, 1):
        for x, y in zip(a.main_arrays(0, kv), b.main_arrays(0, kv)):
            assert np.array_equal(x, y)


@pytest.mark.parametrize("fmt", [oracle.NVFP4, oracle.FP8])
def test_recalibration_bulk_equals_token_by_token(fmt):
    n = 3 * P + 7
    k, v = _kv(18, 1, 2, n)
    gs = [[oracle.global_scale(fmt, oracle.amax(k)), oracle.global_scale(fmt, oracle.amax(v))]]
    a = oracle.OracleCache(fmt, 1, 1, 2, 128, 256, global_scales=gs, recalibrate_every=P)
    b = oracle.OracleCache(fmt, 1, 1, 2, 128, 256, global_scales=gs, recalibrate_every=P)
    a.append(0, k, v)
    for t in range(n):
        b.append(0, k[:, :, t:t + 1], v[:, :, t:t + 1])
    for kv in (0, 1):
        assert a.segment_scales(0, kv) == b.segment_scales(0, kv)
        for x, y in zip(a.main_arrays(0, kv), b.main_arrays(0, kv)):
            assert np.array_equal(x, y)
    a.reset()
    assert a.scale(0, 0) == np.float32(gs[0][0]) and a.lengths(0) == (0, 0)


def test_recalibration_follows_a_growing_sequence():
    """Values that grow 8x after calibration saturate under a frozen scale;
    renewing it every P tokens keeps the reconstruction error near the
    stationary level."""
    n = 8 * P
    exps = [0, 0, 3, 3, 3, 3, 3, 3]
    k = _planted(19, 1, 2, n, exps)
    frozen = oracle.OracleCache(oracle.NVFP4, 1, 1, 2, 128, 256)
    recal = oracle.OracleCache(oracle.NVFP4, 1, 1, 2, 128, 256, recalibrate_every=P)
    for c in (frozen, recal):
        c.append(0, k[:, :, :P], k[:, :, :P])
        for t in range(P, n):
            c.append(0, k[:, :, t:t + 1], k[:, :, t:t + 1])
    tail = slice(4 * P, n)
    def err(c):
        xh = c.dequantize_main(0, 0)[:, :, tail].astype(np.float64)
        return np.linalg.norm(xh - k[:, :, tail]) / np.linalg.norm(k[:, :, tail])
    assert err(frozen) > 0.5
    assert err(recal) < 0.12
