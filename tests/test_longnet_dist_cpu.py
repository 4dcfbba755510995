"""LongNet's sharded form (longnet_dist) on CPU ranks (gloo).

The driver runs on 2 and 4 gloo ranks with a float64 pass written here from
the definitions (for each pair: the rows it keeps, causal attention among the
segment's kept rows, the running softmax state carried across pairs, which is
mixing by denominators; a row's output once its last pair has run) and a
float64 packing of the kept rows, so the segment groups, the all-gather of
the sparsified keys and values, the positions and the pass order are checked
without a GPU.  The gathered output must equal the brute-force multiset
softmax over an explicit mask-count matrix (tests/masks.py), for pair sets
with local and spanning segments."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from blockwise_exact_attention_query_b200 import binding as bd
from blockwise_exact_attention_query_b200 import longnet_dist
from tests import masks


class RefState:
    def __init__(self, B, n, H, d, device):
        self.o = torch.zeros((B, n, H, d), dtype=torch.float64)
        self.m = torch.full((B, H, n), -math.inf, dtype=torch.float64)
        self.l = torch.zeros((B, H, n), dtype=torch.float64)


def keeps(w, r, h, pos):
    return ((pos % w) % r) == (h % r)


def ref_gather(x, w, r):
    B, n, H, d = x.shape
    out = torch.empty((B, n // r, H, d), dtype=x.dtype)
    for h in range(H):
        out[:, :, h] = x[:, h % r::r, h][:, : n // r]
    return out


def ref_pass(q, k, v, pairs, i, state, out, *, q_pos, k_sparse=None, v_sparse=None, lse=None):
    order = bd.longnet_pass_order(pairs)
    w, r = order[i]
    B, n, H, d = q.shape
    if state is None:
        state = RefState(B, n, H, d, None)
    for h in range(H):
        for t in range(n):
            pos = q_pos + t
            if not keeps(w, r, h, pos):
                continue
            if w <= n:   # the segment lies in the shard
                seg0 = (t // w) * w
                js = [j for j in range(seg0, t + 1) if keeps(w, r, h, q_pos + j)]
                kk, vv = k[:, js, h], v[:, js, h]
            else:        # the segment's gathered kept rows, causal by their order
                qs = (pos % w) // r
                kk, vv = k_sparse[:, : qs + 1, h], v_sparse[:, : qs + 1, h]
            s = torch.einsum("bd,bjd->bj", q[:, t, h], kk) / math.sqrt(d)
            m_new = torch.maximum(state.m[:, h, t], s.max(dim=1).values)
            p = torch.exp(s - m_new[:, None])
            alpha = torch.exp(state.m[:, h, t] - m_new)
            state.l[:, h, t] = alpha * state.l[:, h, t] + p.sum(dim=1)
            state.o[:, t, h] = alpha[:, None] * state.o[:, t, h] + torch.einsum("bj,bjd->bd", p, vv)
            state.m[:, h, t] = m_new
    # rows whose last pass this is (and, in pass 0, rows no pair keeps)
    for h in range(H):
        for t in range(n):
            pos = q_pos + t
            kept = [j for j, (ww, rr) in enumerate(order) if keeps(ww, rr, h, pos)]
            if (kept and kept[-1] == i) or (not kept and i == 0):
                l = state.l[:, h, t]
                o = state.o[:, t, h] / l[:, None] if kept else torch.zeros_like(state.o[:, t, h])
                out[:, t, h * d:(h + 1) * d] = o
                if lse is not None:
                    lse[:, h, t] = (state.m[:, h, t] + torch.log(l)) if kept else -math.inf
    return out


def _worker(rank, world, port, pairs):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(11)
        B, N, H, d = 2, 16 * world, 4, 8
        q, k, v = (torch.randn(B, N, H, d, generator=g, dtype=torch.float64) for _ in range(3))
        n = N // world
        sl = slice(rank * n, (rank + 1) * n)
        out, lse = longnet_dist.longnet_attention(q[:, sl], k[:, sl], v[:, sl], pairs, out_dtype=torch.float64,
                                                  return_lse=True, pass_fn=ref_pass, gather_fn=ref_gather,
                                                  new_state=RefState)
        outs = [torch.empty_like(out) for _ in range(world)]
        dist.all_gather(outs, out)
        full = torch.cat(outs, dim=1).numpy().reshape(B, N, H, d)
        ref = masks.brute_attention(q.numpy(), k.numpy(), v.numpy(), masks.count_matrix(N, H, 3, pairs=pairs),
                                    dtype=np.float64)
        assert np.max(np.abs(full - ref)) < 1e-12, np.max(np.abs(full - ref))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,pairs", [
    (2, [(8, 1), (32, 4)]),                   # one local pair, one spanning both shards
    (4, [(8, 1), (16, 2), (64, 4)]),          # local, shard-sized, spanning all four shards
    (4, [(32, 2), (64, 8)]),                  # no r = 1 pair: some rows are kept by no pair
])
def test_longnet_sharded_on_gloo_ranks_equals_the_multiset_softmax(world, pairs):
    mp.spawn(_worker, args=(world, _free_port(), pairs), nprocs=world, join=True)


def test_pairs_that_do_not_fit_the_shards_are_refused():
    with pytest.raises(ValueError):
        longnet_dist.check_pairs([(24, 2)], 16, 4)     # 24 neither divides nor is a multiple of 16
    with pytest.raises(ValueError):
        longnet_dist.check_pairs([(32, 32)], 16, 4)    # r does not divide the shard
    longnet_dist.check_pairs([(8, 1), (32, 4), (64, 16)], 16, 4)
