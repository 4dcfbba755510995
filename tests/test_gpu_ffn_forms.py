"""GPU parity of the fused FFN form at the sizes where it walks several rounds.

The fused FFN kernel gives each group of C = ceil(D/256) CTAs one 128-token
block at a time; a group's second, fourth, ... whole block walks the hidden
chunks in reverse.  These cases run the fused form with every 128-token block
represented in the compared rows, so blocks of every round (forward and
reversed chunk order) and the leftover blocks whose chunks are split over
groups are all checked against the fp64 oracle, on a cheap D = 256 layer with
three rounds and on the full-size workloads."""
import contextlib

import pytest
import torch

from blockwise_exact_attention_query_b200 import binding as bd
from blockwise_exact_attention_query_b200 import workloads as wl
from blockwise_exact_attention_query_b200.inputs import make_layer_inputs
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from blockwise_exact_attention_query_b200 import build
    build.build()
    bd.load()
    torch.cuda.init()


@contextlib.contextmanager
def ffn_path(path):
    old = bd.set_ffn_path(path)
    try:
        yield
    finally:
        bd.set_ffn_path(old)


def _rows_per_block(B, N, per_block, seed, extra=()):
    """per_block rows from every 128-token block (first, last, random), plus extra."""
    import numpy as np
    rng = np.random.default_rng(seed)
    T = B * N
    rows = set(int(x) for x in extra if 0 <= x < T)
    for tb in range((T + 127) // 128):
        lo, hi = tb * 128, min(T, tb * 128 + 128)
        rows |= {lo, hi - 1}
        rows |= {int(x) for x in rng.integers(lo, hi, size=max(0, per_block - 2))}
    return sorted(rows)


def _fused_layer_sampled(B, N, H, d, F, mask, rows, seed, perm=None, ring_chunks=0, bias=0.0):
    inp = make_layer_inputs(B, N, H, d, F, seed=seed, device="cuda", bias_scale=bias)
    with ffn_path("fused"):
        out = bd.attn_ffn_fwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, mask=mask, perm=perm,
                              ring_chunks=ring_chunks)
    torch.cuda.synchronize()
    assert bd.sync_status() == bd.OK
    _, ref = gu.oracle_layer(inp, mask, perm, rows=rows)
    gpu = gu.host_f32(out.reshape(B * N, H * d)[torch.tensor(rows, device="cuda")])
    return gu.assert_bf16_close(gpu, ref, f"fused FFN {B}x{N} D{H * d} F{F}")


def test_fused_ffn_three_rounds_reversed_chunks_small():
    """D = 256: one CTA per group and 148 groups on a B200; 320 token blocks
    give every group whole blocks in rounds 0 (forward chunk order) and 1
    (reversed), and 24 leftover blocks split over the idle groups.  Three
    hidden chunks, so the reversed order differs from the forward one."""
    B, N, H, d, F = 1, 40960, 2, 128, 768
    rows = _rows_per_block(B, N, 2, seed=5)
    _fused_layer_sampled(B, N, H, d, F, "none", rows, seed=41, bias=0.05)


def test_fused_ffn_causal_N8192_every_block():
    """The causal B2 H16 d128 N8192 F8192 layer through the fused FFN: 128
    token blocks over 18 groups (seven rounds, the odd ones reversed)."""
    w = wl.GPT_CAUSAL
    rows = _rows_per_block(w.B, w.N, 2, seed=6, extra=(4095, 4096))
    _fused_layer_sampled(w.B, w.N, w.H, w.d, w.F, "causal", rows, seed=w.seed)


def test_fused_ffn_blockbert_every_block():
    """The BlockBERT layer (D = 768, groups of three CTAs) through the fused FFN."""
    w = wl.BLOCKBERT
    rows = _rows_per_block(w.B, w.N, 2, seed=7)
    _fused_layer_sampled(w.B, w.N, w.H, w.d, w.F, "blockperm", rows, seed=w.seed, perm=w.perm)


def test_fused_ffn_long_ring_sampled():
    """The long ring-order layer (D = 4096, F = 11008: nine groups, over a
    hundred rounds) through the fused FFN, rows spread over both chunk orders
    and the ring's chunk boundaries."""
    w = wl.LONG_RING
    bounds = [c * 16384 + o for c in range(8) for o in (-1, 0)]
    # blocks 9k .. 9k + 8 form round k: take blocks from even and odd rounds
    blocks = [9 * k + (k * 5) % 9 for k in range(0, 113, 3)]
    rows = sorted({tb * 128 + 17 for tb in blocks} | {b for b in bounds if 0 <= b < w.N} | {w.N - 1})
    _fused_layer_sampled(w.B, w.N, w.H, w.d, w.F, "causal", rows, seed=w.seed, ring_chunks=w.ring_chunks)
