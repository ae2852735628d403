"""Pins for the oracle's decode attention (CPU only).

The oracle computes softmax attention in binary64 by its definition.  It is
checked here against torch's scaled_dot_product_attention in float64 (an
independent library routine) and against closed forms that any correct
softmax attention must satisfy.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _sdpa(q, K, V, scale):
    qt = torch.from_numpy(q.astype(np.float64))[None, :, None, :]    # [1, G, 1, D]
    Kt = torch.from_numpy(K.astype(np.float64))[None, None].expand(1, q.shape[0], -1, -1)
    Vt = torch.from_numpy(V.astype(np.float64))[None, None].expand(1, q.shape[0], -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=scale)
    return o[0, :, 0, :].numpy()


@pytest.mark.parametrize("G,L,D", [(1, 1, 4), (4, 7, 4), (8, 300, 128), (3, 1000, 64)])
def test_attention_matches_torch_sdpa_float64(G, L, D):
    rng = np.random.default_rng(100 + L)
    q = rng.standard_normal((G, D)).astype(np.float32)
    K = rng.standard_normal((L, D)).astype(np.float32)
    V = rng.standard_normal((L, D)).astype(np.float32)
    scale = 1.0 / math.sqrt(D)
    ours = oracle.attention(q, K, V, scale)
    ref = _sdpa(q, K, V, scale)
    np.testing.assert_allclose(ours, ref, rtol=1e-12, atol=1e-13)


def test_attention_single_key_returns_its_value():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((4, 128)).astype(np.float32)
    K = rng.standard_normal((1, 128)).astype(np.float32)
    V = rng.standard_normal((1, 128)).astype(np.float32)
    out = oracle.attention(q, K, V)
    assert np.array_equal(out, np.repeat(V.astype(np.float64), 4, axis=0))


def test_attention_equal_keys_give_mean_value():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((2, 32)).astype(np.float32)
    K = np.repeat(rng.standard_normal((1, 32)).astype(np.float32), 50, axis=0)
    V = rng.standard_normal((50, 32)).astype(np.float32)
    out = oracle.attention(q, K, V)
    np.testing.assert_allclose(out, np.repeat(V.astype(np.float64).mean(0, keepdims=True), 2, 0),
                               rtol=0, atol=1e-14)


def test_attention_two_keys_closed_form():
    # scores differ by ln 3 -> weights 3/4 and 1/4
    D = 4
    q = np.array([[1.0, 0.0, 0.0, 0.0]], np.float32)
    K = np.array([[math.log(3.0) * 2.0, 0, 0, 0], [0, 0, 0, 0]], np.float32)   # scale 1/2
    V = np.array([[4.0, 0, 0, 0], [0, 8.0, 0, 0]], np.float32)
    out = oracle.attention(q, K, V, 0.5)
    k0 = float(np.float32(math.log(3.0) * 2.0)) * 0.5
    w0 = math.exp(k0) / (math.exp(k0) + 1.0)
    np.testing.assert_allclose(out[0], [4.0 * w0, 8.0 * (1 - w0), 0, 0], rtol=1e-15)
    assert abs(w0 - 0.75) < 1e-7


def test_attention_dominant_key_and_shift_invariance():
    rng = np.random.default_rng(3)
    D, L = 16, 20
    q = np.zeros((1, D), np.float32)
    q[0, 0] = 1.0
    K = rng.standard_normal((L, D)).astype(np.float32)
    K[5, 0] = 1000.0
    V = rng.standard_normal((L, D)).astype(np.float32)
    out = oracle.attention(q, K, V, 1.0)
    np.testing.assert_allclose(out[0], V[5].astype(np.float64), rtol=0, atol=1e-12)
    # adding the same vector-independent amount to every score changes nothing:
    # a key component along a direction q ignores (q[1] = 0)
    K2 = K.copy()
    K2[:, 1] += 7.0
    assert np.array_equal(oracle.attention(q, K2, V, 1.0), out)


def test_gqa_head_mapping():
    """Query head h reads KV head h // G."""
    rng = np.random.default_rng(4)
    B, Hkv, G, L, D = 2, 3, 2, 9, 8
    q = rng.standard_normal((B, Hkv * G, D)).astype(np.float32)
    K = rng.standard_normal((B, Hkv, L, D)).astype(np.float32)
    V = rng.standard_normal((B, Hkv, L, D)).astype(np.float32)
    out = oracle.gqa_decode_attention(q, K, V)
    for b in range(B):
        for h in range(Hkv * G):
            ref = _sdpa(q[b, h:h + 1], K[b, h // G], V[b, h // G], 1 / math.sqrt(D))
            np.testing.assert_allclose(out[b, h], ref[0], rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# Log-sum-exp of the scores, and the merge of attention over disjoint parts
# (context parallelism: the split-K combine taken across devices)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("G,L", [(1, 1), (4, 33), (8, 700)])
def test_lse_matches_torch_logsumexp(G, L):
    rng = np.random.default_rng(200 + L)
    q = rng.standard_normal((G, 128)).astype(np.float32)
    K = rng.standard_normal((L, 128)).astype(np.float32)
    V = rng.standard_normal((L, 128)).astype(np.float32)
    out, lse = oracle.attention_lse(q, K, V)
    s = torch.from_numpy(q.astype(np.float64)) @ torch.from_numpy(K.astype(np.float64)).T / math.sqrt(128)
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=1).numpy(), rtol=1e-13, atol=1e-13)
    assert np.array_equal(out, oracle.attention(q, K, V))


def test_lse_closed_forms():
    # one key: the score itself; L equal keys: score + ln L; scores s and
    # s - ln 3: s + ln(4/3); no keys: -inf and a zero output
    q = np.zeros((1, 4), np.float32)
    q[0, 0] = 2.0
    k = np.array([[1.5, 0, 0, 0]], np.float32)
    v = np.ones((1, 4), np.float32)
    assert oracle.attention_lse(q, k, v, 1.0)[1][0] == 3.0
    assert math.isclose(oracle.attention_lse(q, np.repeat(k, 5, 0), np.repeat(v, 5, 0), 1.0)[1][0],
                        3.0 + math.log(5), rel_tol=1e-15)
    k2 = np.array([[1.5, 0, 0, 0], [1.5 - math.log(3) / 2, 0, 0, 0]], np.float32)
    s1 = 2.0 * float(k2[1, 0])
    ref = 3.0 + math.log(1 + math.exp(s1 - 3.0))
    assert math.isclose(oracle.attention_lse(q, k2, np.ones((2, 4), np.float32), 1.0)[1][0], ref,
                        rel_tol=1e-15)
    o, l = oracle.attention_lse(q, np.zeros((0, 4), np.float32), np.zeros((0, 4), np.float32), 1.0)
    assert l[0] == -np.inf and np.all(o == 0)


@pytest.mark.parametrize("cuts", [[0, 700], [0, 1, 700], [0, 300, 301, 650, 700], [0, 0, 350, 700]])
def test_combine_of_any_split_equals_the_single_pass(cuts):
    rng = np.random.default_rng(300 + len(cuts))
    G, L = 4, 700
    q = rng.standard_normal((G, 128)).astype(np.float32)
    K = rng.standard_normal((L, 128)).astype(np.float32)
    V = rng.standard_normal((L, 128)).astype(np.float32)
    full_o, full_l = oracle.attention_lse(q, K, V)
    parts = [oracle.attention_lse(q, K[a:b], V[a:b]) for a, b in zip(cuts[:-1], cuts[1:])]
    o, l = oracle.combine_partials(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    np.testing.assert_allclose(o, full_o, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(l, full_l, rtol=1e-14)
    # the parts' order does not matter, and an interleaved split works too
    rev = oracle.combine_partials(np.stack([p[0] for p in parts][::-1]),
                                  np.stack([p[1] for p in parts][::-1]))
    np.testing.assert_allclose(rev[0], full_o, rtol=1e-12, atol=1e-14)
    ev = oracle.attention_lse(q, K[0::2], V[0::2])
    od = oracle.attention_lse(q, K[1::2], V[1::2])
    o2, _ = oracle.combine_partials(np.stack([ev[0], od[0]]), np.stack([ev[1], od[1]]))
    np.testing.assert_allclose(o2, full_o, rtol=1e-12, atol=1e-14)


def test_combine_of_empty_parts():
    o = np.ones((2, 3, 128))
    lse = np.full((2, 3), -np.inf)
    out, l = oracle.combine_partials(o, lse)
    assert np.all(out == 0) and np.all(l == -np.inf)
    lse[1, :] = 0.5
    out, l = oracle.combine_partials(o * np.arange(2)[:, None, None], lse)
    assert np.all(out == 1.0) and np.all(l == 0.5)
