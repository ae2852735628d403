"""kvq_decode_step (append one token + decode attention in one launch)
against the two separate calls and the oracle.

Two caches receive the same prefill; one then runs decode steps through
kvq_decode_step, the other through kvq_append + kvq_decode_attention.  After
every step the attention outputs must agree within the attention tolerance,
and at the end both caches must hold bit-identical codes, scales and rings,
equal to the oracle's.  Covered: every format, even and odd token positions
(NVFP4 V is stored pair-interleaved), INT4 rings including the step that
fills the ring (which falls back to the two calls), the uncalibrated first
append, several CTA counts, and one-tile caches where the tile holding the
new token is the CTA's first tile.
"""
import pytest
import torch

import oracle
import quantized_kv_cache_13_b200 as kvq
from quantized_kv_cache_13_b200 import workloads as W

from _support import assert_attention_close, assert_cache_bit_exact, to_dev

pytestmark = pytest.mark.gpu


def _pair(fmt, B, H, max_len, R, gs=None, layers=1):
    grp = 64 if fmt in kvq.INT_AFFINE else 0
    a = kvq.KVCache(fmt, layers, B, H, max_len, 128, grp, R, gs)
    b = kvq.KVCache(fmt, layers, B, H, max_len, 128, grp, R, gs)
    o = oracle.OracleCache(fmt, layers, B, H, 128, max_len, grp, R, gs)
    return a, b, o


@pytest.mark.parametrize("fmt,R,G,L,steps", [
    (kvq.NVFP4, 0, 4, 700, 9),
    (kvq.NVFP4, 0, 8, 256, 5),
    (kvq.NVFP4, 0, 4, 381, 6),      # new tokens cross the 384-token tile boundary
    (kvq.NVFP4, 0, 2, 765, 6),      # ... and the 768-token capacity boundary
    (kvq.FP8, 0, 4, 511, 6),
    (kvq.INT4, 0, 1, 300, 5),
    (kvq.INT4, 128, 1, 1000, 6),
    (kvq.INT4, 16, 2, 40, 30),      # crosses two ring flushes (fallback steps)
    (kvq.INT8, 0, 4, 300, 5),
    (kvq.INT8, 128, 1, 1000, 6),
    (kvq.INT8, 16, 2, 40, 30),
])
def test_decode_step_matches_separate_calls(fmt, R, G, L, steps):
    B, H = 2, 3
    w = W.custom(fmt, B, H, H * G, L + steps, seed=5150 + L, residual_length=R)
    k = W.kv_tensor(w, "k", 0, L + steps)
    v = W.kv_tensor(w, "v", 0, L + steps)
    a, b, o = _pair(fmt, B, H, L + steps + 4, R)
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
        assert_attention_close(out_a.cpu().numpy(), out_b.double().cpu().numpy(), "step %d" % s)
    assert_cache_bit_exact(a, o)
    assert_cache_bit_exact(b, o)
    assert a.device_status() == 0


def test_uncalibrated_first_step_and_other_layer():
    B, H, G = 1, 2, 4
    w = W.custom(kvq.NVFP4, B, H, H * G, 40, seed=606)
    k = W.kv_tensor(w, "k", 0, 40)
    v = W.kv_tensor(w, "v", 0, 40)
    a, b, o = _pair(kvq.NVFP4, B, H, 64, 0, layers=2)
    for s in range(40):
        kn, vn = k[:, :, s:s + 1], v[:, :, s:s + 1]
        q = to_dev(W.q_tensor(w, s))
        out_a = a.decode_step(1, to_dev(kn), to_dev(vn), q)
        b.append(1, to_dev(kn), to_dev(vn))
        out_b = b.decode_attention(1, q)
        o.append(1, kn, vn)
        assert_attention_close(out_a.cpu().numpy(), out_b.double().cpu().numpy(), "step %d" % s)
    assert_cache_bit_exact(a, o, 1)
    assert a.lengths(0) == (0, 0)


@pytest.mark.parametrize("ctas", ["1", "2", "6", "1000"])
def test_decode_step_split_counts(ctas, monkeypatch):
    """Short caches (one tile per sequence): the new token's tile is the
    first tile a CTA copies."""
    monkeypatch.setenv("KVQ_CTAS", ctas)
    B, H, G, L = 2, 3, 4, 100
    w = W.custom(kvq.NVFP4, B, H, H * G, L + 3, seed=777)
    k = W.kv_tensor(w, "k", 0, L + 3)
    v = W.kv_tensor(w, "v", 0, L + 3)
    a, b, o = _pair(kvq.NVFP4, B, H, L + 8, 0)
    for c in (a, b):
        c.append(0, to_dev(k[:, :, :L]), to_dev(v[:, :, :L]))
    o.append(0, k[:, :, :L], v[:, :, :L])
    for s in range(3):
        kn, vn = k[:, :, L + s:L + s + 1], v[:, :, L + s:L + s + 1]
        q = to_dev(W.q_tensor(w, s))
        out_a = a.decode_step(0, to_dev(kn), to_dev(vn), q)
        b.append(0, to_dev(kn), to_dev(vn))
        out_b = b.decode_attention(0, q)
        o.append(0, kn, vn)
        assert_attention_close(out_a.cpu().numpy(), out_b.double().cpu().numpy(), "step %d" % s)
        ref = o.decode_attention(0, W.q_tensor(w, s))
        assert_attention_close(out_a.cpu().numpy(), ref, "oracle step %d" % s)
    assert_cache_bit_exact(a, o)


def test_decode_step_errors_leave_lengths():
    a = kvq.KVCache(kvq.NVFP4, 1, 1, 2, 4)
    z = torch.zeros((1, 2, 4, 128), dtype=torch.bfloat16, device="cuda")
    a.append(0, z, z)
    one = torch.zeros((1, 2, 1, 128), dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((1, 8, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        a.decode_step(0, one, one, q)
    assert e.value.status == 2          # CAPACITY
    assert a.lengths(0) == (4, 0)
    with pytest.raises(kvq.KVQError) as e:
        a.decode_step(0, one, one, torch.zeros((1, 5, 128), dtype=torch.bfloat16, device="cuda"))
    assert e.value.status == 1
    assert a.lengths(0) == (4, 0)
