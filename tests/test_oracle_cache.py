"""Pins for the oracle's cache bookkeeping and the KV size formula (CPU only).

* Size formula and savings: the tables printed on
  "KV Cache量化实战：Model Optimizer为大模型长上下文省下50%显存" (savings
  table) and "KV缓存量化技术：提升大模型长文本生成效率" (section 1 and the
  section 3.1 table), stored under tests/golden/.
* Residual ring (section 2.2 of the second page): closed-form lengths after
  n appends, and bulk append = token-by-token append, bit for bit.
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
                                   (oracle.INT4, 16), (oracle.INT8, 0), (oracle.INT8, 128)])
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
        oracle.OracleCache(oracle.NVFP4, 1, 1, 1, 128, 8, 16, 128)
