"""Context-parallel decode on one GPU: a sequence split over several caches
(the caches stand in for the ranks; the all-gather is over NCCL between
GPUs and is covered on the CPU by tests/test_dist_context_parallel.py).

Every cache runs kvq_decode_attention_lse over its part; the parts' outputs
and log-sum-exps are merged by kvq_combine_partials and must equal the
oracle's attention over the whole sequence (the union of the parts' codes,
dequantized), within the attention tolerance.  The per-part log-sum-exp is
compared with the oracle's over the same dequantized part: the only error
is the FP16 rounding of the scaled query (relative 2^-12 per element),
which moves a score by at most 2^-12 * scale * |q| |k|, below 1e-2 for these
inputs.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_13_b200 as kvq
from quantized_kv_cache_13_b200 import workloads as W

from _support import assert_attention_close, gpu_arrays, gpu_ring, gpu_scale, to_dev

pytestmark = pytest.mark.gpu

LSE_ATOL = 1e-2


def _dequant_all(cache):
    """Dequantized K, V of a cache (main then ring), float32 [B, H, L, D]."""
    n, r = cache.lengths(0)
    KV = []
    for kv in (0, 1):
        parts = []
        if n:
            parts.append(oracle.dequantize_arrays(cache.fmt, gpu_arrays(cache, 0, kv, n),
                                                  gpu_scale(cache, 0, kv), cache.group_size or 16))
        if r:
            parts.append(gpu_ring(cache, 0, kv, r))
        KV.append(np.concatenate(parts, axis=2) if parts else
                  np.zeros((cache.batch, cache.kv_heads, 0, 128), np.float32))
    return KV


@pytest.mark.parametrize("fmt,R,cuts", [
    (kvq.NVFP4, 0, [0, 700, 701, 1500]),
    (kvq.FP8, 0, [0, 384, 1500]),
    (kvq.INT4, 128, [0, 1000, 1000, 1500]),      # the middle part holds no tokens
    (kvq.INT8, 128, [0, 129, 1500]),
    (kvq.INT2, 0, [0, 500, 1000, 1500]),
])
def test_split_sequence_merges_to_the_whole(fmt, R, cuts):
    B, H, G, L = 2, 2, 4, 1500
    w = W.custom(fmt, B, H, H * G, L, seed=8800 + fmt, residual_length=R)
    k = W.kv_tensor(w, "k", 0, L)
    v = W.kv_tensor(w, "v", 0, L)
    gs = None
    if fmt in (kvq.NVFP4, kvq.FP8):   # one per-tensor scale for all parts, as the ranks would share
        gs = [[oracle.global_scale(fmt, oracle.amax(k)), oracle.global_scale(fmt, oracle.amax(v))]]
    grp = 64 if fmt in kvq.INT_AFFINE else 0
    q = W.q_tensor(w)
    qd = to_dev(q)
    outs, lses, Ks, Vs = [], [], [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        c = kvq.KVCache(fmt, 1, B, H, max(b - a, 1), 128, grp, R, gs)
        if b > a:
            c.append(0, to_dev(k[:, :, a:b]), to_dev(v[:, :, a:b]))
        o, l = c.decode_attention_lse(0, qd)
        torch.cuda.synchronize()
        Kp, Vp = _dequant_all(c)
        lse_ref = np.zeros((B, H * G))
        for bb in range(B):
            for h in range(H):
                lse_ref[bb, h * G:(h + 1) * G] = oracle.attention_lse(
                    q[bb, h * G:(h + 1) * G], Kp[bb, h], Vp[bb, h])[1]
        l_np = l.cpu().numpy()
        if b == a:
            assert np.all(l_np == -np.inf) and np.all(o.cpu().numpy() == 0)
        else:
            assert np.abs(l_np - lse_ref).max() <= LSE_ATOL
            # the same launch as kvq_decode_attention: identical outputs
            assert torch.equal(o, c.decode_attention(0, qd))
        outs.append(o.reshape(B * H * G, 128))
        lses.append(l.reshape(B * H * G))
        Ks.append(Kp)
        Vs.append(Vp)
        assert c.device_status() == 0
    o_parts = torch.stack(outs)
    lse_parts = torch.stack(lses)
    out = torch.empty((B * H * G, 128), dtype=torch.float32, device="cuda")
    lse_out = torch.empty(B * H * G, dtype=torch.float32, device="cuda")
    kvq.kvq_combine_partials(o_parts, lse_parts, out, lse_out)
    Kall = np.concatenate(Ks, axis=2)
    Vall = np.concatenate(Vs, axis=2)
    ref = oracle.gqa_decode_attention(q, Kall, Vall)
    assert_attention_close(out.cpu().numpy().reshape(B, H * G, 128), ref, "merged parts")
    lse_full = np.zeros((B, H * G))
    for bb in range(B):
        for h in range(H):
            lse_full[bb, h * G:(h + 1) * G] = oracle.attention_lse(
                q[bb, h * G:(h + 1) * G], Kall[bb, h], Vall[bb, h])[1]
    assert np.abs(lse_out.cpu().numpy().reshape(B, H * G) - lse_full).max() <= LSE_ATOL


def test_combine_kernel_against_the_oracle_merge():
    """The merge alone on random records, including rows with empty parts."""
    rng = np.random.default_rng(8900)
    n, rows = 4, 300
    o = rng.standard_normal((n, rows, 128)).astype(np.float32)
    lse = (5 * rng.standard_normal((n, rows))).astype(np.float32)
    lse[1, ::3] = -np.inf
    lse[:, 7] = -np.inf                           # a row no part covers
    out = torch.empty((rows, 128), dtype=torch.float32, device="cuda")
    lse_out = torch.empty(rows, dtype=torch.float32, device="cuda")
    kvq.kvq_combine_partials(torch.from_numpy(o).cuda(), torch.from_numpy(lse).cuda(), out, lse_out)
    ref, ref_lse = oracle.combine_partials(o, lse)
    got = out.cpu().numpy()
    assert np.all(got[7] == 0) and lse_out[7].item() == -np.inf
    keep = np.arange(rows) != 7
    np.testing.assert_allclose(got[keep], ref[keep], rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(lse_out.cpu().numpy()[keep], ref_lse[keep], rtol=1e-6, atol=1e-5)
