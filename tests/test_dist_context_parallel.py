"""The context-parallel exchange on CPU, with the gloo backend.

Each of 2 (or 3) ranks holds a part of every sequence's keys and values.  A
rank computes attention over its part with the log-sum-exp of the scores,
the ranks all-gather the packed (out, lse) records with the package's
gather_partials, and the merge of the gathered parts must equal attention
over the whole sequence.  On the GPU the local attention and the merge are
kernels (kvq_decode_attention_lse, kvq_combine_partials); here the oracle
stands in for both, so that the exchange itself (packing, rank order,
unpacking) runs as several processes.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    rng = np.random.default_rng(4242)
    B, Hkv, G, L = 2, 2, 4, 301
    q = rng.standard_normal((B, Hkv * G, 128)).astype(np.float32)
    K = rng.standard_normal((B, Hkv, L, 128)).astype(np.float32)
    V = rng.standard_normal((B, Hkv, L, 128)).astype(np.float32)
    return q, K, V, G


def _local(q, K, V, G, sel):
    import oracle
    B, Hq, D = q.shape
    out = np.zeros((B, Hq, D))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for h in range(K.shape[1]):
            o, l = oracle.attention_lse(q[b, h * G:(h + 1) * G], K[b, h, sel], V[b, h, sel])
            out[b, h * G:(h + 1) * G], lse[b, h * G:(h + 1) * G] = o, l
    return out, lse


def _rank_main(rank, world, port, split, q_res):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist
    import oracle
    from quantized_kv_cache_13_b200 import cp
    dist.init_process_group("gloo", rank=rank, world_size=world)
    q, K, V, G = _inputs()
    L = K.shape[2]
    if split == "interleaved":
        sel = np.arange(rank, L, world)
    elif split == "empty_rank":            # the last rank holds no tokens yet
        sel = np.arange(L) if rank == 0 else np.arange(0)
    else:                                  # contiguous, uneven parts
        cuts = [0, 100, 101, L][:world] + [L]
        sel = np.arange(cuts[rank], cuts[rank + 1])
    out, lse = _local(q, K, V, G, sel)
    o_parts, lse_parts = cp.gather_partials(torch.from_numpy(out.astype(np.float32)),
                                            torch.from_numpy(lse.astype(np.float32)))
    assert o_parts.shape == (world, q.shape[0] * q.shape[1], 128)
    # this rank's own record sits at its rank index
    assert np.array_equal(o_parts[rank].numpy(), out.astype(np.float32).reshape(-1, 128))
    merged, merged_lse = oracle.combine_partials(o_parts.numpy(), lse_parts.numpy())
    full, full_lse = _local(q, K, V, G, np.arange(L))
    err = float(np.abs(merged.reshape(full.shape) - full).max())
    lerr = float(np.abs(merged_lse.reshape(full_lse.shape) - full_lse).max())
    dist.destroy_process_group()
    q_res.put((rank, err, lerr))


@pytest.mark.parametrize("world,split", [(2, "interleaved"), (3, "contiguous"), (2, "empty_rank")])
def test_context_parallel_exchange(world, split):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, split, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=10) for _ in range(world))
    for r, err, lerr in res:
        # the records travel as f32: agreement to f32 rounding
        assert err < 1e-5 and lerr < 1e-5, (r, err, lerr)


def test_pack_and_unpack_are_inverse():
    import torch
    from quantized_kv_cache_13_b200 import cp
    outs = [torch.randn(2, 8, 128) for _ in range(3)]
    lses = [torch.randn(2, 8) for _ in range(3)]
    gathered = torch.cat([cp.pack_partials(o, l) for o, l in zip(outs, lses)])
    o_parts, lse_parts = cp.unpack_gathered(gathered, 3, 16, 128)
    for r in range(3):
        assert torch.equal(o_parts[r], outs[r].reshape(16, 128))
        assert torch.equal(lse_parts[r], lses[r].reshape(16))
    assert o_parts.stride(1) == 128 and o_parts.stride(2) == 1 and lse_parts.stride(1) == 1
