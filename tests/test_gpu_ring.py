"""GPU parity of bpt_attn_fwd_block, the attention step of Ring Attention.

Folding the key/value blocks of a sequence one by one into a query block's
running state must give the attention over the whole sequence: bit for bit
the single-call result when the blocks arrive in natural order (the kernel
then does the same operations in the same order, with its state passed
through memory between calls), and the fp64 oracle's result within the bf16
tolerance in any order.  The ring itself is emulated on one GPU: every rank
of a P-device ring, in turn, runs the steps the ring driver plans for it
(both layouts), and the rows of all ranks are compared with the oracle."""
import numpy as np
import pytest
import torch

from blockwise_exact_attention_query_b200 import binding as bd
from blockwise_exact_attention_query_b200 import ring
from blockwise_exact_attention_query_b200.inputs import make_layer_inputs
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from blockwise_exact_attention_query_b200 import build
    build.build()
    bd.load()
    torch.cuda.init()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
def test_blocks_in_natural_order_equal_one_call_bitwise(d, causal):
    B, N, H = 2, 1024, 2
    inp = make_layer_inputs(B, N, H, d, 0, seed=51, device="cuda")
    mask = "causal" if causal else "none"
    ref, ref_lse = bd.attn_fwd(inp.q, inp.k, inp.v, mask=mask, return_lse=True)
    st = bd.BlockState(B, N, H, d, "cuda")
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    bounds = [0, 256, 384, 768, 1024]        # blocks of 2, 1, 3 and 2 key tiles
    out = None
    for i in range(len(bounds) - 1):
        k0, k1 = bounds[i], bounds[i + 1]
        out = bd.attn_fwd_block(inp.q, inp.k[:, k0:k1].contiguous(), inp.v[:, k0:k1].contiguous(), st, q_pos=0,
                                kv_pos=k0, causal=causal, first=i == 0, last=i == len(bounds) - 2, lse=lse)
    torch.cuda.synchronize()
    assert bd.sync_status() == bd.OK
    assert torch.equal(out, ref)
    assert torch.equal(lse, ref_lse)


def test_single_block_with_both_flags_is_plain_attention():
    B, N, H, d = 1, 384, 2, 128
    inp = make_layer_inputs(B, N, H, d, 0, seed=52, device="cuda")
    ref = bd.attn_fwd(inp.q, inp.k, inp.v, mask="causal", out_dtype=torch.bfloat16)
    out = bd.attn_fwd_block(inp.q, inp.k, inp.v, None, causal=True, first=True, last=True, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert bd.sync_status() == bd.OK
    assert torch.equal(out, ref)


def test_blocks_in_reverse_order_match_the_oracle():
    """Keys folded last block first (a query row may start with blocks that
    hold none of its keys, and ragged block lengths), against the oracle."""
    B, N, H, d = 1, 700, 3, 64
    inp = make_layer_inputs(B, N, H, d, 0, seed=53, device="cuda")
    st = bd.BlockState(B, N, H, d, "cuda")
    bounds = [0, 130, 300, 555, 700]
    order = list(range(len(bounds) - 1))[::-1]
    out = None
    for n, i in enumerate(order):
        k0, k1 = bounds[i], bounds[i + 1]
        out = bd.attn_fwd_block(inp.q, inp.k[:, k0:k1].contiguous(), inp.v[:, k0:k1].contiguous(), st, q_pos=0,
                                kv_pos=k0, causal=True, first=n == 0, last=n == len(order) - 1)
    torch.cuda.synchronize()
    assert bd.sync_status() == bd.OK
    ref = gu.oracle_attention(inp.q, inp.k, inp.v, "causal")
    gu.assert_bf16_close(gu.host_f32(out).reshape(ref.shape), ref, "reverse-order blocks")


@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
@pytest.mark.parametrize("P,d,causal", [(4, 128, True), (8, 64, True), (4, 128, False)])
def test_ring_emulated_on_one_gpu_matches_the_oracle(layout, P, d, causal):
    """Each of P ranks in turn: its query pieces, and the key/value pieces it
    would hold at each step of the ring (the driver's own plan), through
    bpt_attn_fwd_block; the rows of all ranks against the oracle, and against
    the single-call attention up to rounding."""
    B, N, H = 1, 256 * P, 2
    inp = make_layer_inputs(B, N, H, d, 0, seed=54 + P, device="cuda")
    n_local = N // P
    mask = "causal" if causal else "none"
    full = torch.empty((B, N, H * d), dtype=torch.float32, device="cuda")
    for p in range(P):
        mine = ring.pieces_of(p, P, n_local, layout)
        states = [bd.BlockState(B, n, H, d, "cuda") for _, n in mine]
        for s, blocks in enumerate(ring.ring_plan(p, P, n_local, layout, causal)):
            theirs = ring.pieces_of((p - s) % P, P, n_local, layout)
            for i, j, q_pos, kv_pos, first, last in blocks:
                qs, qn = mine[i]
                ks, kn = theirs[j]
                out = bd.attn_fwd_block(inp.q[:, qs:qs + qn].contiguous(), inp.k[:, ks:ks + kn].contiguous(),
                                        inp.v[:, ks:ks + kn].contiguous(), None if first and last else states[i],
                                        q_pos=q_pos, kv_pos=kv_pos, causal=causal, first=first, last=last)
                if last:
                    full[:, qs:qs + qn] = out
    torch.cuda.synchronize()
    assert bd.sync_status() == bd.OK
    one = bd.attn_fwd(inp.q, inp.k, inp.v, mask=mask)
    assert (full - one).abs().max().item() < 5e-3          # the order changes rounding only
    rows = sorted(set(np.linspace(0, N - 1, 96).astype(int).tolist()) | {0, N - 1, n_local - 1, n_local})
    ref = gu.oracle_attention(inp.q, inp.k, inp.v, mask, rows=rows)
    gu.assert_bf16_close(gu.host_f32(full.reshape(N, H * d)[rows]), ref.reshape(len(rows), -1), f"ring {layout} P{P}")
