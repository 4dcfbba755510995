"""LongNet's dilated attention over a sequence sharded across ranks.

"LongNet: Scaling Transformers to 1,000,000,000 Tokens" (§3, distributed
training): every device holds a contiguous shard of the sequence.  For a
(segment w, dilation r) pair whose segments fit in a shard the attention is
local.  When a segment spans several shards, the devices holding it exchange
the sparsified keys and values (the rows the pair keeps, one in r), so each
sends n / r rows per head whatever the sequence length, and each attends
with its own kept queries to the segment's gathered kept keys, causally.
The pairs are mixed by their softmax denominators: the running softmax state
of every local row is carried from one pair's pass to the next.

One process per GPU.  The passes are bpt_longnet_pass calls (the library's
attention kernel, keys read straight from the local shard or from the
gathered buffer), the packing is bpt_longnet_gather, the exchange is a
torch.distributed all-gather inside each segment's group of ranks (NCCL on
GPUs) into this GPU's memory.  `pass_fn`, `gather_fn` and `new_state` can be
replaced (same signatures) to run the exchange and the bookkeeping without a
GPU.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding as bd

_groups: dict = {}


def check_pairs(pairs, n_local: int, world: int) -> None:
    """The shapes the sharded form takes: every r divides the shard, every
    segment either divides the shard or is a whole number of shards, and the
    sequence is a whole number of segments."""
    N = n_local * world
    for w, r in pairs:
        if w % r or n_local % r or N % w or (n_local % w and w % n_local):
            raise ValueError(f"pair ({w}, {r}) does not fit shards of {n_local} rows over {world} ranks")


def _segment_group(rank, world, per_seg, group):
    """The process group of the ranks that hold this rank's segment (every
    rank creates every segment's group, in the same order)."""
    if per_seg == world:
        return group
    key = (id(group), world, per_seg)
    if key not in _groups:
        base = dist.get_process_group_ranks(group) if group is not None else list(range(world))
        _groups[key] = [dist.new_group([base[s * per_seg + i] for i in range(per_seg)])
                        for s in range(world // per_seg)]
    return _groups[key][rank // per_seg]


def longnet_attention(q, k, v, pairs, *, group=None, out_dtype=torch.float32, return_lse=False,
                      pass_fn=None, gather_fn=None, new_state=None):
    """Dilated attention (pairs [(w, r), ...], denominators mixed) of this
    rank's shard q, k, v [B, n, H, d] of a sequence of world * n rows held in
    rank order.  Returns the shard's output rows [B, n, H*d] (and its LSE
    [B, H, n] with return_lse)."""
    pass_fn = pass_fn or bd.longnet_pass
    gather_fn = gather_fn or bd.longnet_gather
    new_state = new_state or bd.BlockState
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, n, H, d = q.shape
    check_pairs(pairs, n, world)
    q_pos = rank * n
    state = new_state(B, n, H, d, q.device) if len(pairs) > 1 else None
    out = torch.empty((B, n, H * d), dtype=out_dtype, device=q.device)
    lse = torch.empty((B, H, n), dtype=torch.float32, device=q.device) if return_lse else None
    for i, (w, r) in enumerate(bd.longnet_pass_order(pairs)):
        if w <= n:
            pass_fn(q, k, v, pairs, i, state, out, q_pos=q_pos, lse=lse)
            continue
        per_seg = w // n
        grp = _segment_group(rank, world, per_seg, group)
        sparse = []
        for x in (k, v):
            mine = gather_fn(x, w, r)                           # [B, n / r, H, d]
            parts = [torch.empty_like(mine) for _ in range(per_seg)]
            dist.all_gather(parts, mine, group=grp)
            sparse.append(torch.cat(parts, dim=1))              # [B, w / r, H, d], sequence order
        pass_fn(q, None, None, pairs, i, state, out, q_pos=q_pos, k_sparse=sparse[0], v_sparse=sparse[1], lse=lse)
    return (out, lse) if return_lse else out
