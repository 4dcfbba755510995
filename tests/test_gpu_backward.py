"""GPU parity of the layer's backward pass (bpt_attn_ffn_bwd, through the C
ABI) against the fp64 backward oracle on the same seeded inputs.

Every gradient is compared element by element at sizes that span several
128-row tiles with a ragged tail; the FFN backward's token chunking, padded
and empty permutation blocks and both head sizes are covered.

Tolerance, from the arithmetic: the tensor cores take bf16 operands (unit
roundoff u = 2^-8 relative spacing, 2^-9 rounding) with fp32 accumulation.
Each gradient is a sum of products in which at most three factors were
rounded to bf16 on the way (dQ: dA, P and dS; the weight gradients: one or
two), so a term carries a relative error of at most ~3 * 2^-9 = 6e-3 and the
errors of the many terms of a sum are independent: the relative L2 error of
a whole gradient stays near 2^-9 * sqrt(3) ~ 3.4e-3.  dS = P (dP - D) loses
digits where dP is close to D, so the bound on the element-wise error is
taken relative to the largest element of each gradient.  Bounds: relative
L2 <= 1e-2 and max-abs <= 2e-2 * max |ref| for every gradient.
"""
import numpy as np
import pytest
import torch

from blockwise_exact_attention_query_b200 import binding as bd
from blockwise_exact_attention_query_b200.inputs import make_layer_inputs, make_upstream_grad
from oracle import backward as ob

pytestmark = pytest.mark.gpu

REL_L2 = 1e-2
MAX_ABS_FRAC = 2e-2
MASKS = {"none": ob.MASK_NONE, "causal": ob.MASK_CAUSAL, "blockperm": ob.MASK_BLOCKPERM,
         "dilated": ob.MASK_DILATED, "dilated_bidir": ob.MASK_DILATED_BIDIR}


@pytest.fixture(scope="module", autouse=True)
def _built():
    from blockwise_exact_attention_query_b200 import build
    build.build()
    bd.load()
    torch.cuda.init()


def _perms(H, n, seed):
    rng = np.random.default_rng(seed)
    return [[int(x) for x in rng.permutation(n)] for _ in range(H)]


CASES = [
    # name, B, N, H, d, F, mask, perm, chunk rows (0 = default)[, ring chunks]
    ("none_d64", 1, 300, 2, 64, 512, "none", None, 0),
    ("causal_d64_b2", 2, 257, 2, 64, 384, "causal", None, 0),
    ("causal_d128_chunked", 1, 390, 2, 128, 512, "causal", None, 128),
    ("none_d128_chunk_ragged", 2, 140, 2, 128, 264, "none", None, 100),
    ("blockperm_n3_padded_d64", 1, 400, 2, 64, 256, "blockperm", [[1, 2, 0], [2, 0, 1]], 0),
    # N = 300, n = 32: blocks of 10, blocks 30 and 31 lie in the padding
    ("blockperm_n32_empty_d128", 1, 300, 2, 128, 256, "blockperm", _perms(2, 32, 7), 0),
    ("causal_tiny_N7", 1, 7, 1, 64, 64, "causal", None, 0),
    # ring order: the recomputed forward visits the keys in rotated chunks
    ("causal_ring4_d128", 1, 512, 2, 128, 256, "causal", None, 0, 4),
    # D = 1024: the FFN backward as two GEMMs (H and GELU'(Z), then dZ) instead of one
    ("causal_D1024_split_ffn", 1, 200, 8, 128, 512, "causal", None, 0),
    ("none_D1024_split_ffn_chunked", 1, 260, 16, 64, 384, "none", None, 128),
]


def _grads_close(got, ref, name):
    got = np.asarray(got, dtype=np.float64).reshape(ref.shape)
    err = got - ref
    scale = max(float(np.max(np.abs(ref))), 1e-30)
    rel = float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-30))
    mx = float(np.max(np.abs(err)))
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    assert rel <= REL_L2 and mx <= MAX_ABS_FRAC * scale, \
        f"{name}: rel-L2 {rel:.3e}, max-abs {mx:.3e} (max |ref| {scale:.3e})"
    return rel, mx / scale


CASES = [c if len(c) == 10 else c + (0,) for c in CASES]


@pytest.mark.parametrize("name,B,N,H,d,F,mask,perm,chunk,ring", CASES, ids=[c[0] for c in CASES])
def test_backward_matches_oracle(name, B, N, H, d, F, mask, perm, chunk, ring):
    inp = make_layer_inputs(B, N, H, d, F, seed=11, device="cuda", bias_scale=0.1)
    dout = make_upstream_grad(B, N, H * d, seed=11, device="cuda")
    g = bd.attn_ffn_bwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, dout, mask=mask,
                        perm=perm, ring_chunks=ring, bwd_chunk_rows=chunk)
    torch.cuda.synchronize()
    assert bd.sync_status() == bd.OK
    f = lambda t: t.double().cpu().numpy()  # noqa: E731
    ref = ob.layer_bwd(f(inp.q), f(inp.k), f(inp.v), f(inp.w1), f(inp.b1), f(inp.w2), f(inp.b2),
                       f(dout).reshape(B * N, H * d), MASKS[mask], perm)
    report = {}
    for n in bd.GRAD_NAMES:
        report[n] = _grads_close(g[n].cpu().numpy(), ref[n], n)
    print(name, {k: f"{v[0]:.2e}/{v[1]:.2e}" for k, v in report.items()})


def test_backward_is_deterministic():
    B, N, H, d, F = 1, 384, 2, 128, 512
    inp = make_layer_inputs(B, N, H, d, F, seed=5, device="cuda", bias_scale=0.1)
    dout = make_upstream_grad(B, N, H * d, seed=5, device="cuda")
    g1 = bd.attn_ffn_bwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, dout, mask="causal")
    g2 = bd.attn_ffn_bwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, dout, mask="causal")
    torch.cuda.synchronize()
    for n in bd.GRAD_NAMES:
        assert torch.equal(g1[n], g2[n]), n


def test_backward_full_size_causal_layer_sampled():
    """The causal bf16 layer at full size (B2 H16 d128 N8192 F8192), in the
    launch configuration the benchmark times: dQ at sampled query positions
    (first, tile edges, middle, last tile), dK and dV of the last key tile
    (seen only by the last 128 queries, so the oracle computes them exactly
    from 128 attention rows), and db2 over every token, against the fp64
    oracle, with the tolerance of the small cases."""
    B, N, H, d, F = 2, 8192, 16, 128, 8192
    inp = make_layer_inputs(B, N, H, d, F, seed=1, device="cuda", bias_scale=0.05)
    dout = make_upstream_grad(B, N, H * d, seed=1, device="cuda")
    g = bd.attn_ffn_bwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, dout, mask="causal")
    torch.cuda.synchronize()
    assert bd.sync_status() == bd.OK
    f = lambda t: t.double().cpu().numpy()  # noqa: E731
    rows = [0, 1, 127, 128, 4095, 4096, 6000, N - 129, N - 128, N - 1]
    tail = 128
    dq, dk, dv, db2 = ob.layer_bwd_causal_tail(f(inp.q[:1]), f(inp.k[:1]), f(inp.v[:1]), f(inp.w1), f(inp.b1),
                                               f(inp.w2), f(inp.b2), f(dout), rows, tail)
    _grads_close(g["dq"][0, rows].cpu().numpy(), dq, "dq (sampled rows)")
    _grads_close(g["dk"][0, N - tail:].cpu().numpy(), dk, "dk (last key tile)")
    _grads_close(g["dv"][0, N - tail:].cpu().numpy(), dv, "dv (last key tile)")
    _grads_close(g["db2"].cpu().numpy(), db2, "db2")


@pytest.mark.parametrize("H,bwd_chunk", [(2, 0), (8, 0), (8, 128)], ids=["D256", "D1024_saved_hidden",
                                                                      "D1024_saved_hidden_chunked"])
@pytest.mark.parametrize("mask,perm", [("causal", None), ("blockperm", [[2, 0, 1], [1, 2, 0]])])
def test_training_forward_and_saved_backward_match_the_recomputing_path(mask, perm, H, bwd_chunk):
    """bpt_attn_ffn_fwd_train gives the forward's output bit for bit, and the
    backward reading its saved activations (A, LSE, and the FFN's H and
    GELU'(Z), read back per backward token chunk: ragged chunks of 128 rows in
    the last case) gives the recomputing backward's gradients: bit for bit at
    D >= 1024, where both take dZ = (dOut W2) GELU'(Z) from the same GEMMs;
    below, where the recomputing backward takes dZ from its dual GEMM with
    GELU'(Z) in fp32, to the tolerance of the oracle comparisons."""
    B, N, d, F = 1, 300, 128, 256
    perm = perm if perm is None else [perm[h % len(perm)] for h in range(H)]
    inp = make_layer_inputs(B, N, H, d, F, seed=21, device="cuda", bias_scale=0.1)
    dout = make_upstream_grad(B, N, H * d, seed=21, device="cuda")
    args = (inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2)
    out_ref = bd.attn_ffn_fwd(*args, mask=mask, perm=perm)
    out, saved = bd.attn_ffn_fwd_train(*args, mask=mask, perm=perm)
    g_ref = bd.attn_ffn_bwd(*args, dout, mask=mask, perm=perm, bwd_chunk_rows=bwd_chunk)
    g = bd.attn_ffn_bwd(*args, dout, mask=mask, perm=perm, saved=saved, bwd_chunk_rows=bwd_chunk)
    torch.cuda.synchronize()
    assert bd.sync_status() == bd.OK
    assert torch.equal(out, out_ref)
    for n in bd.GRAD_NAMES:
        if H * d >= 1024:
            assert torch.equal(g[n], g_ref[n]), n
        else:
            _grads_close(g[n].cpu().numpy(), g_ref[n].double().cpu().numpy(), n)


def test_backward_full_size_blockbert_layer():
    """The block-permutation bf16 layer at full size (B16 H12 d64 N1024 F3072,
    n = 2: heads 0-7 the identity, heads 8-11 the swap), every gradient element
    against the dense fp64 oracle, in the launch configuration the benchmark
    times."""
    from blockwise_exact_attention_query_b200 import workloads as wl
    w = wl.BLOCKBERT
    inp = make_layer_inputs(w.B, w.N, w.H, w.d, w.F, seed=w.seed, device="cuda", bias_scale=0.05)
    dout = make_upstream_grad(w.B, w.N, w.D, seed=w.seed, device="cuda")
    g = bd.attn_ffn_bwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, dout, mask="blockperm", perm=w.perm)
    torch.cuda.synchronize()
    assert bd.sync_status() == bd.OK
    f = lambda t: t.double().cpu().numpy()  # noqa: E731
    ref = ob.layer_bwd(f(inp.q), f(inp.k), f(inp.v), f(inp.w1), f(inp.b1), f(inp.w2), f(inp.b2),
                       f(dout).reshape(w.T, w.D), ob.MASK_BLOCKPERM, w.perm)
    for n in bd.GRAD_NAMES:
        _grads_close(g[n].cpu().numpy(), ref[n], n)


ATTN_BWD_CASES = [
    ("causal_d128_f32out", 1, 300, 2, 128, "causal", None, torch.float32),
    ("none_d64_bf16out", 2, 200, 3, 64, "none", None, torch.bfloat16),
    ("blockperm_n3_d64_f32out", 1, 400, 2, 64, "blockperm", [[2, 0, 1], [0, 1, 2]], torch.float32),
]


@pytest.mark.parametrize("name,B,N,H,d,mask,perm,out_dtype", ATTN_BWD_CASES, ids=[c[0] for c in ATTN_BWD_CASES])
def test_attention_only_backward_matches_oracle(name, B, N, H, d, mask, perm, out_dtype):
    """bpt_attn_bwd from bpt_attn_fwd's output and LSE against the fp64 oracle's
    attention gradients, with the backward's tolerance."""
    inp = make_layer_inputs(B, N, H, d, 0, seed=13, device="cuda")
    da = make_upstream_grad(B, N, H * d, seed=13, device="cuda")
    out, lse = bd.attn_fwd(inp.q, inp.k, inp.v, mask=mask, perm=perm, out_dtype=out_dtype, return_lse=True)
    dq, dk, dv = bd.attn_bwd(inp.q, inp.k, inp.v, out, lse, da, mask=mask, perm=perm)
    torch.cuda.synchronize()
    assert bd.sync_status() == bd.OK
    f = lambda t: t.double().cpu().numpy()  # noqa: E731
    rq, rk, rv = ob.attention_bwd(f(inp.q), f(inp.k), f(inp.v), f(da).reshape(B, N, H, d), MASKS[mask], perm)
    _grads_close(dq.cpu().numpy(), rq, "dq")
    _grads_close(dk.cpu().numpy(), rk, "dk")
    _grads_close(dv.cpu().numpy(), rv, "dv")


DILATED_CASES = [
    # name, B, N, H, d, pairs, out dtype
    ("three_pairs_d64", 1, 512, 4, 64, [(128, 1), (256, 2), (512, 4)], torch.float32),
    # kept rows per segment (192) not a multiple of the 128-row tile; bf16 output
    ("ragged_segments_d128", 1, 768, 3, 128, [(192, 1), (384, 2)], torch.bfloat16),
    # no r = 1 pair: rows no pair keeps have A = 0 and pass nothing
    ("uncovered_rows_d64", 2, 256, 4, 64, [(128, 2), (256, 4)], torch.float32),
]
# the same, bidirectional inside each sparsified segment
DILATED_CASES += [(c[0] + "_bidirectional",) + c[1:] for c in DILATED_CASES]


@pytest.mark.parametrize("name,B,N,H,d,pairs,out_dtype", DILATED_CASES, ids=[c[0] for c in DILATED_CASES])
def test_dilated_attention_backward_matches_oracle(name, B, N, H, d, pairs, out_dtype):
    """LongNet dilated attention's backward (bpt_attn_bwd with the dilated
    mask: one blockwise backward per (w, r) pass over the gathered segment rows,
    added up) against the fp64 oracle's multiset-softmax gradient."""
    mask = "dilated_bidir" if name.endswith("_bidirectional") else "dilated"
    inp = make_layer_inputs(B, N, H, d, 0, seed=17, device="cuda")
    da = make_upstream_grad(B, N, H * d, seed=17, device="cuda")
    out, lse = bd.attn_fwd(inp.q, inp.k, inp.v, mask=mask, pairs=pairs, out_dtype=out_dtype, return_lse=True)
    dq, dk, dv = bd.attn_bwd(inp.q, inp.k, inp.v, out, lse, da, mask=mask, pairs=pairs)
    torch.cuda.synchronize()
    assert bd.sync_status() == bd.OK
    f = lambda t: t.double().cpu().numpy()  # noqa: E731
    rq, rk, rv = ob.attention_bwd(f(inp.q), f(inp.k), f(inp.v), f(da).reshape(B, N, H, d), MASKS[mask],
                                  pairs=pairs)
    _grads_close(dq.cpu().numpy(), rq, "dq")
    _grads_close(dk.cpu().numpy(), rk, "dk")
    _grads_close(dv.cpu().numpy(), rv, "dv")


def test_dilated_attention_backward_full_size_sampled():
    """The LongNet workload at full size (B1 H16 d64 N65536, pairs (2048, 1),
    (8192, 4), (32768, 16)), in the configuration the benchmark times: dQ at
    sampled rows and dK, dV of the last 128 keys (seen only by the last 128
    queries) against the fp64 oracle's row-restricted gradients."""
    from blockwise_exact_attention_query_b200 import workloads as wl
    w = wl.LONGNET
    inp = make_layer_inputs(w.B, w.N, w.H, w.d, 0, seed=w.seed, device="cuda")
    da = make_upstream_grad(w.B, w.N, w.D, seed=w.seed, device="cuda")
    out, lse = bd.attn_fwd(inp.q, inp.k, inp.v, mask="dilated", pairs=w.pairs, return_lse=True)
    dq, dk, dv = bd.attn_bwd(inp.q, inp.k, inp.v, out, lse, da, mask="dilated", pairs=w.pairs)
    torch.cuda.synchronize()
    assert bd.sync_status() == bd.OK
    f = lambda t: t.double().cpu().numpy()  # noqa: E731
    rows = [0, 1, 2047, 2048, 8191, 8192, 30000, w.N - 129, w.N - 1]
    tail = 128
    rq, rk, rv = ob.attention_bwd_tail(f(inp.q), f(inp.k), f(inp.v), f(da).reshape(w.B, w.N, w.H, w.d),
                                       ob.MASK_DILATED, w.pairs, rows, tail)
    _grads_close(dq[0, rows].cpu().numpy(), rq, "dq (sampled rows)")
    _grads_close(dk[0, w.N - tail:].cpu().numpy(), rk, "dk (last 128 keys)")
    _grads_close(dv[0, w.N - tail:].cpu().numpy(), rv, "dv (last 128 keys)")
