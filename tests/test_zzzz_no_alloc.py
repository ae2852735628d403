"""kvq_decode_attention_noalloc: decode attention for callers that cannot
allocate device memory (plugin callbacks that must not allocate, decode
loops that must not call cudaMalloc because it can block and synchronise).

It is called through the C ABI and compared with kvq_decode_attention (with a
caller workspace) on the same cache, twice in a row with different queries,
so that records left in the shared scratch by one call cannot leak into the
next.  The file name sorts after every other test file, so pytest collects
it last.
"""
import numpy as np
import pytest
import torch

import quantized_kv_cache_13_b200 as kvq
from quantized_kv_cache_13_b200 import workloads as W

from _support import ATOL, RTOL_L2, to_dev

pytestmark = pytest.mark.gpu


def _noalloc(cache, q, out):
    lib = kvq.lib()
    st = lib.kvq_decode_attention_noalloc(cache.handle, 0, q.data_ptr(), q.shape[1], 0.0,
                                          out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    return st


def _close(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    assert np.abs(a - b).max() <= ATOL
    assert np.linalg.norm(a - b) / np.linalg.norm(b) <= RTOL_L2


@pytest.mark.parametrize("fmt,R,G,L", [(kvq.NVFP4, 0, 4, 3000), (kvq.INT4, 128, 1, 1000),
                                       (kvq.FP8, 0, 8, 777)])
def test_noalloc_matches_workspace_call_twice(fmt, R, G, L):
    w = W.custom(fmt, 2, 3, 3 * G, L, seed=4242 + L, residual_length=R)
    cache = kvq.KVCache(fmt, 1, 2, 3, L + 8, 128, 64 if fmt in kvq.INT_AFFINE else 0, R)
    cache.append(0, to_dev(W.kv_tensor(w, "k", 0, L)), to_dev(W.kv_tensor(w, "v", 0, L)))
    for step in range(2):
        q = to_dev(W.q_tensor(w, step))
        ref = cache.decode_attention(0, q)
        out = torch.full_like(ref, float("nan"))
        assert _noalloc(cache, q, out) == 0, kvq.lib().kvq_last_error()
        torch.cuda.synchronize()
        _close(out, ref)
    assert cache.device_status() == 0


def test_noalloc_refuses_oversized_scratch():
    # 2048 (batch, kv-head) units x 8 query heads each needs more than 4 MiB
    cache = kvq.KVCache(kvq.NVFP4, 1, 64, 32, 16)
    k = torch.zeros((64, 32, 16, 128), dtype=torch.bfloat16, device="cuda")
    cache.append(0, k, k)
    q = torch.zeros((64, 32 * 8, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((64, 32 * 8, 128), dtype=torch.float32, device="cuda")
    assert kvq.kvq_workspace_bytes(cache.handle, 32 * 8) > 4 << 20
    assert _noalloc(cache, q, out) == 3          # KVQ_ERR_WORKSPACE
    assert b"scratch" in kvq.lib().kvq_last_error()
