"""Context-parallel attention forward: the key sequence split across GPUs.

Every rank holds the same queries Q and one contiguous shard of the keys and
values (rank r holds keys [k0_r, k0_r + n_r) of S_k).  The forward is the
"local attention, then global reduction" of the rkmt.cn GPU attention
operator page (section 3.1.1) with the key shards on different GPUs, the
cross-GPU sharding the csdn page (section 5, item 3) points to for long
sequences:

1. each rank computes its shard's partial with ``attn_fwd_partials_shard``:
   O_r (softmax over the shard's keys times V, FP32) and LSE_r;
2. one NCCL all-gather brings every rank's (O_r, LSE_r) into this GPU's own
   buffers, in rank order (no kernel ever reads a peer's memory);
3. ``attn_merge_partials`` forms LSE = log sum_r exp LSE_r and
   O = sum_r exp(LSE_r - LSE) O_r on every rank.

Under the causal mask the queries are the last s_q positions of the whole
key sequence (attn_fwd's bottom-right mask); shard r then has the diagonal
S_k - s_q - k0_r, and rows that see none of its keys carry LSE_r = -inf.

Python here only orders the steps and calls ``torch.distributed`` for the
exchange (plumbing); the arithmetic of steps 1 and 3 runs in the CUDA
library.  ``ops`` exists so the host logic can be tested on CPU ranks with
stand-in steps; the default is the CUDA library and nothing else.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable


@dataclass(frozen=True)
class PartialOps:
    """The two device steps: ``partials(q, k, v, causal, scale, diag_offset)
    -> (o_r [b, h_q, s_q, d] FP32, lse_r [b, h_q, s_q])`` and
    ``merge(o_parts [n, b, h_q, s_q, d], lse_parts [n, b, h_q, s_q]) ->
    (o [b, s_q, h_q, d], lse [b, h_q, s_q])``."""
    partials: Callable
    merge: Callable


def cuda_ops() -> PartialOps:
    from . import attn

    def partials(q, k, v, causal, scale, diag_offset):
        return attn.attn_fwd_partials_shard(q, k, v, causal=causal, scale=scale,
                                            diag_offset=diag_offset)

    def merge(o_parts, lse_parts):
        return attn.merge_partials(o_parts, lse_parts)

    return PartialOps(partials, merge)


def shard_bounds(lengths, rank):
    """(first key, total keys) of ``rank``'s shard for per-rank shard lengths."""
    return int(sum(lengths[:rank])), int(sum(lengths))


def context_parallel_attn_fwd(q, k_shard, v_shard, causal: bool = False,
                              scale: float | None = None, group=None,
                              key_offset: int | None = None, s_k_total: int | None = None,
                              ops: PartialOps | None = None):
    """Attention of ``q`` over the keys of all ranks' shards, on every rank.

    q: [b, s_q, h_q, d] (the same on every rank); k_shard, v_shard:
    [b, n_r, h_kv, d], this rank's keys.  ``key_offset`` / ``s_k_total``: this
    shard's first global key and the global key count; if None (on every
    rank alike), the shard lengths are all-gathered and the shards are taken
    in rank order.  Returns (o [b, s_q, h_q, d] BF16, lse [b, h_q, s_q] FP32).

    Collectives, the same on every rank: [one all-gather of the shard
    lengths], then one all-gather of O_r and one of LSE_r.
    """
    import math

    import torch
    import torch.distributed as dist

    ops = ops or cuda_ops()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    b, s_q, h_q, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dev = q.device
    if (key_offset is None) != (s_k_total is None):
        raise ValueError("give both key_offset and s_k_total, or neither")
    if key_offset is None:
        n = torch.tensor([k_shard.shape[1]], dtype=torch.int64, device=dev)
        lens = [torch.zeros_like(n) for _ in range(world)]
        dist.all_gather(lens, n, group=group)
        key_offset, s_k_total = shard_bounds([int(t.item()) for t in lens], rank)
    diag = int(s_k_total) - s_q - int(key_offset)

    o_r, lse_r = ops.partials(q, k_shard, v_shard, bool(causal), float(scale), diag)
    o_all = torch.empty((world,) + tuple(o_r.shape), dtype=o_r.dtype, device=o_r.device)
    lse_all = torch.empty((world,) + tuple(lse_r.shape), dtype=lse_r.dtype, device=lse_r.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(o_all, o_r.contiguous(), group=group)
        dist.all_gather_into_tensor(lse_all, lse_r.contiguous(), group=group)
    else:
        dist.all_gather(list(o_all.unbind(0)), o_r.contiguous(), group=group)
        dist.all_gather(list(lse_all.unbind(0)), lse_r.contiguous(), group=group)
    return ops.merge(o_all, lse_all)
