"""Context-parallel decode attention: each rank's cache holds its own part of
every sequence (the part's tokens, in any order: attention does not depend
on key order), and the ranks merge their results.

One step on every rank:
  1. kvq_decode_attention_lse over the local cache: out [B, Hq, D] and the
     log-sum-exp of the scores lse [B, Hq] (0 and -inf for a rank that holds
     no tokens yet);
  2. an all-gather of the packed (out, lse) records of all ranks over the
     process group (NCCL over NVLink on GPUs);
  3. kvq_combine_partials: the log-sum-exp merge of split-K decoding, taken
     across ranks, gives every rank the attention over the whole sequence.

The exchange is B * Hq * (D + 1) floats per rank and step; the records cross
NVLink once through NCCL and are read from local memory by the merge.
"""
from __future__ import annotations

from typing import Tuple


def pack_partials(out, lse):
    """One flat f32 record per rank: out [B, Hq, D] then lse [B, Hq]."""
    import torch
    return torch.cat([out.reshape(-1), lse.reshape(-1)])


def unpack_gathered(gathered, world: int, rows: int, head_dim: int) -> Tuple[object, object]:
    """Views of an all-gathered [world * rec] buffer (rec = rows * (D + 1)):
    o_parts [world, rows, D] and lse_parts [world, rows], rank order."""
    per = gathered.view(world, rows * (head_dim + 1))
    o_parts = per[:, :rows * head_dim].view(world, rows, head_dim)
    lse_parts = per[:, rows * head_dim:]
    return o_parts, lse_parts


def gather_partials(out, lse, group=None):
    """All-gather every rank's (out, lse) over `group`; returns (o_parts
    [world, B*Hq, D], lse_parts [world, B*Hq]) in rank order."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rec = pack_partials(out, lse)
    gathered = torch.empty(world * rec.numel(), dtype=rec.dtype, device=rec.device)
    dist.all_gather_into_tensor(gathered, rec, group=group)
    rows = lse.numel()
    return unpack_gathered(gathered, world, rows, out.shape[-1])


def context_parallel_decode(cache, layer: int, q, group=None, out=None,
                            softmax_scale: float = 0.0, stream=None):
    """Attention of q [B, Hq, D] (bf16, on this rank's GPU) over the whole
    sequence whose parts the ranks of `group` hold: local attention with its
    log-sum-exp, all-gather, merge.  Returns out f32 [B, Hq, D] (the same on
    every rank)."""
    import torch
    from . import kvq_combine_partials
    o_loc, lse_loc = cache.decode_attention_lse(layer, q, softmax_scale=softmax_scale, stream=stream)
    o_parts, lse_parts = gather_partials(o_loc, lse_loc, group)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    kvq_combine_partials(o_parts, lse_parts, out.view(-1, q.shape[-1]), stream=stream)
    return out
