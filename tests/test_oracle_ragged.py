"""Pins of the oracle's ragged batch (RaggedOracleCache): a batch whose
sequences hold different numbers of tokens is B independent one-sequence
caches that share each layer's per-tensor scale."""
import numpy as np
import pytest

import oracle

FMTS = [oracle.NVFP4, oracle.FP8, oracle.INT4, oracle.INT8, oracle.INT2]


def _grp(fmt):
    return 64 if fmt in oracle.INT_AFFINE else 0


def _data(seed, B, H, n, D=128, scale=1.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, H, n, D)).astype(np.float32) * scale
    import torch
    return torch.from_numpy(x).to(torch.bfloat16).float().numpy()


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("R", [0, 16])
def test_equal_lengths_match_the_batched_cache(fmt, R):
    B, H, n = 3, 2, 45
    k, v = _data(1, B, H, n), _data(2, B, H, n)
    q = _data(3, B, H * 2, 1)[:, :, 0]
    rc = oracle.RaggedOracleCache(fmt, 1, B, H, 128, 64, _grp(fmt), R)
    oc = oracle.OracleCache(fmt, 1, B, H, 128, 64, _grp(fmt), R)
    rc.append(0, k[:, :, :20], v[:, :, :20])
    oc.append(0, k[:, :, :20], v[:, :, :20])
    rc.append(0, k[:, :, 20:], v[:, :, 20:], n=[n - 20] * B)
    oc.append(0, k[:, :, 20:], v[:, :, 20:])
    for kv in (0, 1):
        assert rc.scale(0, kv) == oc.scale(0, kv)
        ref = oc.main_arrays(0, kv)
        for b in range(B):
            assert rc.lengths(0, b) == oc.lengths(0)
            if ref is not None:
                for a, r in zip(rc.main_arrays(0, kv, b), ref):
                    assert np.array_equal(a[0], r[b])
            assert np.array_equal(rc.ring_tokens(0, kv, b)[0], oc.ring_tokens(0, kv)[b])
    assert np.array_equal(rc.decode_attention(0, q), oc.decode_attention(0, q))


@pytest.mark.parametrize("fmt", FMTS)
def test_a_sequence_is_independent_of_the_others(fmt):
    """Sequence b's codes and attention equal those of a one-sequence cache
    fed the same tokens with the same per-tensor scale, whatever the other
    sequences hold."""
    B, H, R = 4, 2, 16 if fmt in oracle.INT_AFFINE else 0
    lens = [0, 5, 33, 70]
    k, v = _data(10, B, H, 70), _data(11, B, H, 70)
    q = _data(12, B, H * 3, 1)[:, :, 0]
    rc = oracle.RaggedOracleCache(fmt, 1, B, H, 128, 80, _grp(fmt), R)
    rc.append(0, k, v, n=lens)
    out = rc.decode_attention(0, q)
    assert np.all(out[0] == 0.0)                          # empty sequence
    gs = None if fmt in oracle.INT_AFFINE else [[rc.scale(0, 0), rc.scale(0, 1)]]
    for b in range(1, B):
        one = oracle.OracleCache(fmt, 1, 1, H, 128, 80, _grp(fmt), R, global_scales=gs)
        one.append(0, k[b:b + 1, :, :lens[b]], v[b:b + 1, :, :lens[b]])
        assert rc.lengths(0, b) == one.lengths(0)
        assert np.array_equal(out[b], one.decode_attention(0, q[b:b + 1])[0])
        for kv in (0, 1):
            ref = one.main_arrays(0, kv)
            if ref is not None:
                for a, r in zip(rc.main_arrays(0, kv, b), ref):
                    assert np.array_equal(a, r)
    # other sequences' data does not move sequence 3's result
    k2 = k.copy()
    k2[1] *= 0.5
    rc2 = oracle.RaggedOracleCache(fmt, 1, B, H, 128, 80, _grp(fmt), R, global_scales=gs)
    rc2.append(0, k2, v, n=lens)
    assert np.array_equal(rc2.decode_attention(0, q)[3], out[3])


@pytest.mark.parametrize("fmt", [oracle.NVFP4, oracle.FP8])
def test_calibration_reads_only_appended_tokens(fmt):
    """The per-tensor amax of a ragged append covers each sequence's first
    n[b] tokens only: padding past them does not count."""
    B, H = 2, 2
    k, v = _data(20, B, H, 12), _data(21, B, H, 12)
    k[0, :, 5:] = 1000.0                  # padding of sequence 0 (n = 5)
    rc = oracle.RaggedOracleCache(fmt, 1, B, H, 128, 32)
    rc.append(0, k, v, n=[5, 12])
    want = oracle.global_scale(fmt, max(oracle.amax(k[0, :, :5]), oracle.amax(k[1])))
    assert rc.scale(0, 0) == want
    # the first append calibrates, whichever sequence it feeds; later ones do not
    rc2 = oracle.RaggedOracleCache(fmt, 1, B, H, 128, 32)
    rc2.append_seq(0, 1, k[1, :, :3], v[1, :, :3])
    g = rc2.scale(0, 0)
    assert g == oracle.global_scale(fmt, oracle.amax(k[1, :, :3]))
    rc2.append_seq(0, 0, k[0], v[0])
    assert rc2.scale(0, 0) == g


@pytest.mark.parametrize("fmt", FMTS)
def test_reset_of_one_sequence(fmt):
    B, H = 3, 1
    R = 8 if fmt in oracle.INT_AFFINE else 0
    k, v = _data(30, B, H, 40), _data(31, B, H, 40)
    q = _data(32, B, H, 1)[:, :, 0]
    rc = oracle.RaggedOracleCache(fmt, 1, B, H, 128, 64, _grp(fmt), R)
    rc.append(0, k, v, n=[40, 20, 9])
    before = rc.decode_attention(0, q)
    rc.reset_seq(1)
    assert rc.lengths(0, 1) == (0, 0)
    out = rc.decode_attention(0, q)
    assert np.all(out[1] == 0.0)
    assert np.array_equal(out[0], before[0]) and np.array_equal(out[2], before[2])
    rc.append_seq(0, 1, k[1, :, :20], v[1, :, :20])
    assert np.array_equal(rc.decode_attention(0, q), before)


def test_one_token_sequence_attends_to_its_value():
    """Closed form: with one key, softmax gives it weight 1, so the output is
    that key's (dequantized) value."""
    B, H = 2, 1
    k, v = _data(40, B, H, 30), _data(41, B, H, 30)
    q = _data(42, B, H * 4, 1)[:, :, 0]
    rc = oracle.RaggedOracleCache(oracle.INT8, 1, B, H, 128, 64, 64, 0)
    rc.append(0, k, v, n=[1, 30])
    vhat = oracle.dequantize_arrays(oracle.INT8, rc.main_arrays(0, 1, 0), None, 64)[0, 0, 0]
    out = rc.decode_attention(0, q)
    assert np.allclose(out[0], np.broadcast_to(vhat, (4, 128)), rtol=0, atol=1e-12)
