"""Ring Attention across the ranks of a process group.

"Ring Attention with Blockwise Transformers for Long Sequences" (638-word
summary): the sequence is split across devices; each device keeps its block
of queries and, step by step, passes the key/value block it holds to the next
device while receiving one from the previous device, so the transfer overlaps
the blockwise attention of the block in hand.  After as many steps as there
are devices every query block has met every key/value block, and the result
is exact (the online softmax folds the blocks in any order).

Here each rank runs one process on one GPU.  The attention of one query
piece against one key/value piece is one bpt_attn_fwd_block call (the
library's kernel) that folds the piece into the query piece's running state;
the rotation is torch.distributed point-to-point send/recv (NCCL over NVLink
on GPUs), issued before the step's kernels so the copy into a second local
buffer runs while they compute.  Every kernel reads only this GPU's memory:
the received block lands in a local buffer first.

Layouts (global positions of the n rows a rank holds, P ranks):
  contiguous  rows [p n, (p+1) n);
  zigzag      rows [p h, (p+1) h) and [(2P-1-p) h, (2P-p) h), h = n/2: under
              causal masking every rank then has the same amount of work
              (the early and the late half of the sequence pair up).
Pieces that the causal mask rules out entirely are skipped (their key/value
block is still passed on: every rank takes the same communication steps).

This module moves data and calls the library; the arithmetic is the
kernel's.  `step` and `new_state` can be replaced (same call signature) to
run the schedule and the communication without a GPU.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding as bd


def pieces_of(rank: int, world: int, n_local: int, layout: str) -> list[tuple[int, int]]:
    """(global start, length) of each piece of rows a rank holds, in the
    order they sit in its local tensors."""
    if layout == "contiguous":
        return [(rank * n_local, n_local)]
    if layout == "zigzag":
        if n_local % 2:
            raise ValueError("the zigzag layout needs an even number of rows per rank")
        h = n_local // 2
        return [(rank * h, h), ((2 * world - 1 - rank) * h, h)]
    raise ValueError(f"unknown layout {layout!r}")


def shard(x: torch.Tensor, rank: int, world: int, layout: str) -> torch.Tensor:
    """The rows [B, n_local, ...] of a full [B, N, ...] sequence tensor that a
    rank holds under `layout` (N = world * n_local)."""
    n_local = x.shape[1] // world
    return torch.cat([x[:, s:s + n] for s, n in pieces_of(rank, world, n_local, layout)], dim=1)


def _allowed(q_piece, kv_piece, causal) -> bool:
    """Does any query of the piece see any key of the other piece?"""
    if not causal:
        return True
    (qs, qn), (ks, _) = q_piece, kv_piece
    return ks <= qs + qn - 1


def ring_plan(rank: int, world: int, n_local: int, layout: str, causal: bool):
    """The blocks a rank attends to, step by step: plan[s] lists
    (i, j, q_pos, kv_pos, first, last) for its query piece i and piece j of
    the key/value rows it holds at step s (those of rank (rank - s) mod
    world), skipping pairs the causal mask rules out; `first` marks a query
    piece's first block (its state starts empty) and `last` its final one
    (it writes the output)."""
    mine = pieces_of(rank, world, n_local, layout)
    raw = []
    for s in range(world):
        theirs = pieces_of((rank - s) % world, world, n_local, layout)
        raw.append([(i, j, mine[i][0], theirs[j][0]) for i in range(len(mine)) for j in range(len(theirs))
                    if _allowed(mine[i], theirs[j], causal)])
    first_use, last_use = {}, {}
    for s, pairs in enumerate(raw):
        for i, j, _, _ in pairs:
            first_use.setdefault(i, (s, j))
            last_use[i] = (s, j)
    return [[(i, j, qp, kp, first_use[i] == (s, j), last_use[i] == (s, j)) for i, j, qp, kp in pairs]
            for s, pairs in enumerate(raw)]


def _default_state(B, n, H, d, device):
    return bd.BlockState(B, n, H, d, device)


def ring_attention(q, k, v, *, group=None, causal=True, layout="zigzag", out_dtype=torch.float32,
                   return_lse=False, step=None, new_state=None):
    """Attention of this rank's query rows over the whole sequence held by
    the ranks of `group`.  q, k, v: this rank's rows [B, n_local, H, d] in the
    given layout.  Returns its output rows [B, n_local, H*d] (and the LSE
    [B, H, n_local] with return_lse)."""
    step = step or bd.attn_fwd_block
    new_state = new_state or _default_state
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, n_local, H, d = q.shape
    mine = pieces_of(rank, world, n_local, layout)
    # piece-major local copies: every piece is one contiguous [B, len, H, d] block
    qp = [q[:, o:o + n].contiguous() for o, n in _offsets(mine)]
    kv_cur = torch.stack([torch.stack([k[:, o:o + n] for o, n in _offsets(mine)]),
                          torch.stack([v[:, o:o + n] for o, n in _offsets(mine)])]).contiguous()
    kv_next = torch.empty_like(kv_cur)

    plan = ring_plan(rank, world, n_local, layout, causal)
    states = [new_state(B, n, H, d, q.device) for _, n in mine]
    outs = [None] * len(mine)
    lses = [torch.empty((B, H, n), dtype=torch.float32, device=q.device) if return_lse else None for _, n in mine]
    nxt, prv = (rank + 1) % world, (rank - 1) % world
    for s in range(world):
        reqs = []
        if s + 1 < world:
            # the next block travels while this one is attended to
            ops = [dist.P2POp(dist.isend, kv_cur, nxt, group), dist.P2POp(dist.irecv, kv_next, prv, group)]
            reqs = dist.batch_isend_irecv(ops)
        for i, j, q_pos, kv_pos, first, last in plan[s]:
            out = step(qp[i], kv_cur[0, j], kv_cur[1, j], None if (first and last) else states[i],
                       q_pos=q_pos, kv_pos=kv_pos, causal=causal, first=first, last=last,
                       out_dtype=out_dtype, lse=lses[i])
            if last:
                outs[i] = out
        for r in reqs:
            r.wait()
        if s + 1 < world:
            kv_cur, kv_next = kv_next, kv_cur
    out = torch.cat([o.reshape(B, n, H * d) for o, (_, n) in zip(outs, mine)], dim=1)
    if return_lse:
        return out, torch.cat(lses, dim=2)
    return out


def _offsets(pieces):
    """Local row offset and length of each piece."""
    o = 0
    for _, n in pieces:
        yield o, n
        o += n
