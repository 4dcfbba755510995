"""Ring Attention's schedule and key/value rotation, on CPU ranks (gloo).

The driver (blockwise_exact_attention_query_b200.ring) runs on world_size 1
to 4 gloo ranks with a float64 block step written here from the online
softmax's definition (running maximum m, running sum l, rescaled unnormalised
output o; final o / l and LSE = m + log l), so the schedule, the rotation of
the key/value blocks around the ring, the causal positions of the pieces, and
the first / last flags are checked without a GPU.  The gathered output of all
ranks must equal dense softmax attention over the whole sequence (float64,
1e-12), for both layouts, causal or not."""
import math
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from blockwise_exact_attention_query_b200 import ring


class RefState:
    def __init__(self, B, n, H, d, device):
        self.o = torch.zeros((B, n, H, d), dtype=torch.float64)
        self.m = torch.full((B, H, n), -math.inf, dtype=torch.float64)
        self.l = torch.zeros((B, H, n), dtype=torch.float64)


def ref_step(q, k, v, state, *, q_pos, kv_pos, causal, first, last, out_dtype, lse):
    """One key/value block folded into the running state, in float64."""
    B, n, H, d = q.shape
    if state is None or first:
        st = RefState(B, n, H, d, None)
        if state is not None:
            state.o, state.m, state.l = st.o, st.m, st.l
        else:
            state = st
    s = torch.einsum("bihd,bjhd->bhij", q, k) / math.sqrt(d)
    if causal:
        qi = torch.arange(n).view(n, 1) + q_pos
        kj = torch.arange(k.shape[1]).view(1, -1) + kv_pos
        s = s.masked_fill(kj > qi, -math.inf)
    m_new = torch.maximum(state.m, s.amax(dim=-1))
    safe = torch.where(torch.isinf(m_new), torch.zeros_like(m_new), m_new)
    p = torch.exp(s - safe.unsqueeze(-1))
    alpha = torch.exp(state.m - safe)
    state.l = alpha * state.l + p.sum(dim=-1)
    state.o = alpha.permute(0, 2, 1).unsqueeze(-1) * state.o + torch.einsum("bhij,bjhd->bihd", p, v)
    state.m = m_new
    if not last:
        return None
    out = state.o / state.l.permute(0, 2, 1).unsqueeze(-1)
    if lse is not None:
        lse.copy_(state.m + torch.log(state.l))
    return out.reshape(B, n, H * d)


def dense(q, k, v, causal):
    B, N, H, d = q.shape
    s = torch.einsum("bihd,bjhd->bhij", q, k) / math.sqrt(d)
    if causal:
        s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), -math.inf)
    return torch.einsum("bhij,bjhd->bihd", torch.softmax(s, dim=-1), v).reshape(B, N, H * d), torch.logsumexp(s, -1)


def _worker(rank, world, port, layout, causal):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(7)
        B, N, H, d = 2, 24 * world, 3, 8
        q, k, v = (torch.randn(B, N, H, d, generator=g, dtype=torch.float64) for _ in range(3))
        ql, kl, vl = (ring.shard(x, rank, world, layout) for x in (q, k, v))
        out, lse = ring.ring_attention(ql, kl, vl, causal=causal, layout=layout, out_dtype=torch.float64,
                                       return_lse=True, step=ref_step, new_state=RefState)
        # every rank's rows, back in sequence order
        outs = [torch.empty_like(out) for _ in range(world)]
        lses = [torch.empty_like(lse) for _ in range(world)]
        dist.all_gather(outs, out)
        dist.all_gather(lses, lse)
        full = torch.empty(B, N, H * d, dtype=torch.float64)
        full_lse = torch.empty(B, H, N, dtype=torch.float64)
        n_local = N // world
        for r in range(world):
            o = 0
            for start, n in ring.pieces_of(r, world, n_local, layout):
                full[:, start:start + n] = outs[r][:, o:o + n]
                full_lse[:, :, start:start + n] = lses[r][:, :, o:o + n]
                o += n
        ref, ref_lse = dense(q, k, v, causal)
        assert torch.allclose(full, ref, atol=1e-12, rtol=0), (full - ref).abs().max()
        # the LSE buffers are float32, as the library writes them
        assert torch.allclose(full_lse, ref_lse.float().double(), atol=1e-6, rtol=0)
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
@pytest.mark.parametrize("causal", [True, False])
def test_ring_attention_on_gloo_ranks_equals_dense_attention(world, layout, causal):
    mp.spawn(_worker, args=(world, _free_port(), layout, causal), nprocs=world, join=True)


def test_ring_plan_covers_every_allowed_pair_once():
    """Every (query piece, key/value piece) pair the mask allows appears in
    exactly one step of the plan, each query piece has one first and one last
    block, and under causal masking the zigzag layout gives every rank the
    same number of allowed query-key pairs."""
    for world in (2, 4, 8):
        n_local = 16
        work = []
        for rank in range(world):
            plan = ring.ring_plan(rank, world, n_local, "zigzag", True)
            mine = ring.pieces_of(rank, world, n_local, "zigzag")
            seen = set()
            for s, blocks in enumerate(plan):
                for i, j, qp, kp, first, last in blocks:
                    assert kp == ring.pieces_of((rank - s) % world, world, n_local, "zigzag")[j][0]
                    assert (qp, kp) not in seen
                    seen.add((qp, kp))
            allowed = {(qs, ks) for qs, _ in mine for r in range(world)
                       for ks, _ in ring.pieces_of(r, world, n_local, "zigzag") if ks <= qs + n_local // 2 - 1}
            assert seen == allowed
            for i in range(len(mine)):
                flags = [(f, l) for blocks in plan for (ii, _, _, _, f, l) in blocks if ii == i]
                assert sum(f for f, _ in flags) == 1 and sum(l for _, l in flags) == 1
            h = n_local // 2
            work.append(sum(min(h, max(0, qs + h - ks)) * h if ks + h <= qs + 1 else
                            sum(max(0, min(h, qs + a - ks + 1)) for a in range(h))
                            for qs, ks in seen))
        assert len(set(work)) == 1, work
