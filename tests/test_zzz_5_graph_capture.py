"""Decode steps captured in a CUDA graph (the launch sequence of a decode
loop, captured once and replayed) give the eager results bit for bit.

Every library call on the decode path only enqueues kernels on the given
stream (lengths are host-side, nothing allocates or synchronises), so a
loop of kvq_decode_step calls can be captured; capturing runs the host
bookkeeping, and a replay runs the device work.  The steps cover a ring
that fills during the loop (its step runs as an append, a flush and an
attention launch).
"""
import pytest
import torch

import quantized_kv_cache_13_b200 as kvq
from quantized_kv_cache_13_b200 import workloads as W

from _support import to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt,R,L", [(kvq.NVFP4, 0, 700), (kvq.INT4, 16, 40), (kvq.FP8, 0, 383),
                                     (kvq.INT2, 0, 500)])
def test_captured_decode_steps_match_eager(fmt, R, L):
    S, B, H, G = 8, 2, 2, 4
    w = W.custom(fmt, B, H, H * G, L + S, seed=9900 + fmt, residual_length=R)
    k = W.kv_tensor(w, "k", 0, L + S)
    v = W.kv_tensor(w, "v", 0, L + S)
    grp = 64 if fmt in kvq.INT_AFFINE else 0
    eager = kvq.KVCache(fmt, 1, B, H, L + S + 4, 128, grp, R)
    graphed = kvq.KVCache(fmt, 1, B, H, L + S + 4, 128, grp, R)
    for c in (eager, graphed):
        c.append(0, to_dev(k[:, :, :L]), to_dev(v[:, :, :L]))
    kn = [to_dev(k[:, :, L + s:L + s + 1]) for s in range(S)]
    vn = [to_dev(v[:, :, L + s:L + s + 1]) for s in range(S)]
    qs = [to_dev(W.q_tensor(w, s)) for s in range(S)]
    ref = [eager.decode_step(0, kn[s], vn[s], qs[s]).clone() for s in range(S)]

    outs = [torch.empty((B, H * G, 128), dtype=torch.float32, device="cuda") for _ in range(S)]
    graphed.workspace(H * G)               # allocated before the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=side):
        for s in range(S):
            graphed.decode_step(0, kn[s], vn[s], qs[s], out=outs[s])
    # the capture did the host bookkeeping; the device work runs on replay
    assert graphed.lengths(0) == eager.lengths(0)
    for replay in range(2):                # a second replay rewrites the same tokens in place
        g.replay()
        torch.cuda.synchronize()
        for s in range(S):
            assert torch.equal(outs[s], ref[s]), "replay %d, step %d" % (replay, s)
        for kv in (0, 1):
            a, b = eager.raw(0, kv), graphed.raw(0, kv)
            for name in a:
                assert torch.equal(a[name], b[name]), (replay, kv, name)
    del g
    assert graphed.device_status() == 0
