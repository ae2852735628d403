"""The five named workloads at full size, in the launch configuration the
benchmark times, checked against the oracle on sampled outputs.

For each workload the whole prefill is quantize-appended on the GPU (with
amax calibration where the format has a per-tensor scale), then decode
steps append one token and run attention.  The oracle then recomputes, on
the host and from the same seeded generators:
  * the per-tensor scales (amax over the whole prefill, slice by slice),
  * the codes / scales / zero points of sampled (batch, kv-head) units over
    sampled token ranges (bit-exact),
  * the attention output of every query head of the sampled units, over the
    oracle's dequantization of the GPU's full-length codes (max-abs 1e-2,
    rel-L2 2e-3),
and every output element is checked finite.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_13_b200 as kvq
from quantized_kv_cache_13_b200 import workloads as W

from _support import assert_attention_close, gpu_ring, gpu_scale, gpu_unit_arrays

pytestmark = pytest.mark.gpu


def _upload(w, cache):
    """Prefill the GPU cache slice by slice; return the oracle's amax of K, V."""
    amax = [0.0, 0.0]
    k = torch.empty((w.batch, w.kv_heads, w.context, w.head_dim), dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    for b in range(w.batch):
        for h in range(w.kv_heads):
            for i, (name, t) in enumerate((("k", k), ("v", v))):
                x = W.kv_slice(w, name, b, h, 0, w.context)
                amax[i] = max(amax[i], oracle.amax(x))
                t[b, h].copy_(torch.from_numpy(x).to(torch.bfloat16))
    cache.append(0, k, v)
    del k, v
    torch.cuda.synchronize()
    return amax


def _encode(w, x, g):
    if w.fmt == kvq.NVFP4:
        return oracle.nvfp4_quantize(x, g)
    if w.fmt == kvq.FP8:
        return (oracle.fp8_quantize(x, g),)
    if w.fmt == kvq.INT8:
        return oracle.int8_quantize(x, w.group_size)
    if w.fmt == kvq.INT2:
        return oracle.int2_quantize(x, w.group_size)
    return oracle.int4_quantize(x, w.group_size)


def _units(w):
    return sorted({(0, 0), (w.batch - 1, w.kv_heads - 1), (w.batch // 2, w.kv_heads // 3)})


@pytest.mark.parametrize("name,steps", [("gqa_nvfp4_32k", 1), ("mha_int4_16k", 1),
                                        ("gqa_fp8_32k", 1), ("gqa_nvfp4_32k_b16", 1),
                                        ("long_nvfp4_128k", 2), ("mha_int8_16k", 1)])
def test_full_size_workload(name, steps):
    w = W.WORKLOADS[name]
    grp = w.group_size if w.fmt in kvq.INT_AFFINE else 0
    cache = kvq.KVCache(w.fmt, 1, w.batch, w.kv_heads, w.context + w.decode_steps, w.head_dim,
                        grp, w.residual_length)
    amax = _upload(w, cache)
    g = [None, None]
    if w.fmt not in kvq.INT_AFFINE:
        g = [oracle.global_scale(w.fmt, a) for a in amax]
        for kv in (0, 1):
            assert np.float32(gpu_scale(cache, 0, kv)).view(np.uint32) == np.float32(g[kv]).view(np.uint32)
    # decode steps
    q = W.q_tensor(w)
    qd = torch.from_numpy(q).to(torch.bfloat16).cuda()
    for s in range(steps):
        kn = torch.from_numpy(W.kv_tensor(w, "k", w.context + s, 1)).to(torch.bfloat16).cuda()
        vn = torch.from_numpy(W.kv_tensor(w, "v", w.context + s, 1)).to(torch.bfloat16).cuda()
        cache.append(0, kn, vn)
        out = cache.decode_attention(0, qd)
    out = out.cpu().numpy()
    assert np.all(np.isfinite(out))
    n, r = cache.lengths(0)
    assert n + r == w.context + steps
    if w.residual_length:
        assert (n, r) == ((w.context + steps) // w.residual_length * w.residual_length,
                          (w.context + steps) % w.residual_length)
    G = w.G
    for (b, h) in _units(w):
        mine = [gpu_unit_arrays(cache, 0, kv, b, h, n) for kv in (0, 1)]
        # codes of sampled token ranges, bit-exact
        for kv, which in ((0, "k"), (1, "v")):
            for t0, t1 in ((0, 256), (n // 2 - 100, n // 2 + 100), (n - 200, n)):
                ref = _encode(w, W.kv_slice(w, which, b, h, t0, t1 - t0), g[kv])
                for a, r_ in zip(mine[kv], ref):
                    a = a[t0:t1]
                    if a.dtype == np.float32:
                        a, r_ = a.view(np.uint32), np.asarray(r_, np.float32).view(np.uint32)
                    assert np.array_equal(a, r_), "%s %s unit %s tokens %d..%d" % (name, which, (b, h), t0, t1)
        # attention of the unit's query heads over the GPU's own codes
        K = oracle.dequantize_arrays(w.fmt, mine[0], g[0], w.group_size)
        V = oracle.dequantize_arrays(w.fmt, mine[1], g[1], w.group_size)
        if r:
            rk, rv = gpu_ring(cache, 0, 0, r)[b, h], gpu_ring(cache, 0, 1, r)[b, h]
            assert np.array_equal(rk, W.kv_slice(w, "k", b, h, n, r))
            assert np.array_equal(rv, W.kv_slice(w, "v", b, h, n, r))
            K = np.concatenate([K, rk], 0)
            V = np.concatenate([V, rv], 0)
        ref = oracle.attention(q[b, h * G:(h + 1) * G], K, V)
        assert_attention_close(out[b, h * G:(h + 1) * G], ref, "%s unit %s" % (name, (b, h)))
    assert cache.device_status() == 0
