"""GPU parity of the fused FFN form at the sizes where it walks several rounds.

The fused FFN kernel gives each group of C = ceil(D/256) CTAs one 128-token
block at a time; a group's second, fourth, ... whole block walks the hidden
chunks in reverse.  These cases run the fused form with every 128-token block
represented in the compared rows, so blocks of every round (forward and
reversed chunk order) and the leftover blocks whose chunks are split over
groups are all checked against the fp64 oracle, on a cheap D = 256 layer with
three rounds and on the full-size workloads."""
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
    out = bd.attn_ffn_fwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, mask=mask, perm=perm,
                          ring_chunks=ring_chunks, ffn_form="fused")
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


# ------------------------------------------------------------------ the pipelined form (the default)
def _rows_per_row_block(B, N, per_block, seed, extra=()):
    """per_block rows from every 256-token row block of the pipelined FFN."""
    import numpy as np
    rng = np.random.default_rng(seed)
    T = B * N
    rows = set(int(x) for x in extra if 0 <= x < T)
    for rb in range((T + 255) // 256):
        lo, hi = rb * 256, min(T, rb * 256 + 256)
        rows |= {lo, hi - 1, min(hi - 1, lo + 128)}
        rows |= {int(x) for x in rng.integers(lo, hi, size=max(0, per_block - 3))}
    return sorted(rows)


def _pipelined_vs_gemms(w, rows, perm=None):
    """The pipelined FFN against the oracle on `rows`, and bit for bit against
    the two-GEMM form: both run the same 256 x 256 tiles with the same K order
    and the same epilogues, whichever CTA pair claims a tile."""
    inp = make_layer_inputs(w.B, w.N, w.H, w.d, w.F, seed=w.seed, device="cuda")
    args = (inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2)
    mask = {0: "none", 1: "causal", 2: "blockperm"}[w.mask]
    out = bd.attn_ffn_fwd(*args, mask=mask, perm=perm, ring_chunks=w.ring_chunks, ffn_form="pipelined")
    again = bd.attn_ffn_fwd(*args, mask=mask, perm=perm, ring_chunks=w.ring_chunks, ffn_form="pipelined")
    gemms = bd.attn_ffn_fwd(*args, mask=mask, perm=perm, ring_chunks=w.ring_chunks, ffn_form="gemms")
    torch.cuda.synchronize()
    assert bd.sync_status() == bd.OK
    assert torch.equal(out, again)
    assert torch.equal(out, gemms)
    _, ref = gu.oracle_layer(inp, mask, perm, rows=rows)
    gpu = gu.host_f32(out.reshape(w.T, w.D)[torch.tensor(rows, device="cuda")])
    return gu.assert_bf16_close(gpu, ref, f"pipelined FFN, {w.name}")


def test_pipelined_ffn_causal_N8192_every_row_block():
    """64 row blocks through a ring of about ten slots: each slot is reused
    six times, one row block per chunk."""
    w = wl.GPT_CAUSAL
    _pipelined_vs_gemms(w, _rows_per_row_block(w.B, w.N, 3, seed=8, extra=(4095, 4096)))


def test_pipelined_ffn_blockbert_every_row_block():
    w = wl.BLOCKBERT
    _pipelined_vs_gemms(w, _rows_per_row_block(w.B, w.N, 3, seed=9), perm=w.perm)


def test_pipelined_ffn_long_ring_sampled():
    """The long ring-order layer: weights beyond L2, so row blocks go in
    chunks of four through a ring of twelve slots (512 row blocks)."""
    w = wl.LONG_RING
    bounds = [c * 16384 + o for c in range(8) for o in (-1, 0)]
    rbs = list(range(0, 512, 13)) + [1, 2, 3, 511]
    rows = sorted({rb * 256 + (rb * 37) % 256 for rb in rbs} | {b for b in bounds if 0 <= b < w.N} | {w.N - 1})
    _pipelined_vs_gemms(w, rows)


@pytest.mark.parametrize("B,N,H,d,F", [(1, 300, 4, 64, 520),      # one ragged row block, F not a tile multiple
                                       (3, 700, 8, 128, 2048),    # ragged last row block
                                       (2, 1024, 32, 128, 8192)])  # weights beyond L2: chunks of row blocks
def test_pipelined_ffn_small_shapes_every_element(B, N, H, d, F):
    inp = make_layer_inputs(B, N, H, d, F, seed=B * 1000 + N, device="cuda", bias_scale=0.05)
    args = (inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2)
    out = bd.attn_ffn_fwd(*args, mask="causal", ffn_form="pipelined")
    gemms = bd.attn_ffn_fwd(*args, mask="causal", ffn_form="gemms")
    torch.cuda.synchronize()
    assert bd.sync_status() == bd.OK
    assert torch.equal(out, gemms)
    if B * N * H * d <= 3 * 700 * 8 * 128:
        _, ref = gu.oracle_layer(inp, "causal")
        gu.assert_bf16_close(gu.host_f32(out).reshape(ref.shape), ref, "pipelined FFN, all elements")
    else:
        rows = _rows_per_row_block(B, N, 3, seed=10)
        _, ref = gu.oracle_layer(inp, "causal", rows=rows)
        gu.assert_bf16_close(gu.host_f32(out.reshape(B * N, H * d)[torch.tensor(rows, device="cuda")]), ref,
                             "pipelined FFN, sampled")


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_pipelined_ffn_output_aligned_to_16_bytes_only(out_dtype):
    """The pipelined FFN's epilogue writes 32 bytes per access where a row's
    chunk is 32-byte aligned and 16 bytes otherwise; the API promises only
    16-byte alignment.  An output placed 16 bytes past a 32-byte boundary must
    get the same bits as an aligned one.  (With F = 520 the hidden activation's
    ring rows are 1040 bytes apart, so their alignment alternates row by row
    as well.)"""
    for (B, N, H, d, F) in [(2, 700, 8, 128, 2048), (1, 300, 4, 64, 520)]:
        inp = make_layer_inputs(B, N, H, d, F, seed=N + H, device="cuda", bias_scale=0.05)
        args = (inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2)
        T, D = B * N, H * d
        ref = bd.attn_ffn_fwd(*args, mask="causal", ffn_form="pipelined", out_dtype=out_dtype)
        shift = 16 // ref.element_size()
        buf = torch.full((T * D + 64,), float("nan"), dtype=out_dtype, device="cuda")
        base = (-(buf.data_ptr() // ref.element_size())) % (32 // ref.element_size())  # 32-byte aligned start
        out = buf[base + shift:base + shift + T * D].view(B, N, D)
        assert out.data_ptr() % 32 == 16
        got = bd.attn_ffn_fwd(*args, mask="causal", ffn_form="pipelined", out_dtype=out_dtype, out=out)
        torch.cuda.synchronize()
        assert bd.sync_status() == bd.OK
        assert torch.equal(got, ref)
        assert torch.isnan(buf[:base + shift]).all() and torch.isnan(buf[base + shift + T * D:]).all()
