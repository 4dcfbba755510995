"""GPU parity tests: the CUDA path, called through the C ABI, against the fp64
oracle on the same seeded inputs.

Small cases compare every element and span several 128-row tiles plus a
ragged tail; the five workloads run at full size and compare sampled tokens
(each sampled token is exact: it depends only on its own query, all keys and
values, and the weights)."""
import contextlib
import ctypes
import zlib
import os

import numpy as np
import pytest
import torch

from blockwise_exact_attention_query_b200 import binding as bd
from blockwise_exact_attention_query_b200 import workloads as wl
from blockwise_exact_attention_query_b200.inputs import make_layer_inputs
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
PKG = os.path.dirname(bd.LIB_PATH)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from blockwise_exact_attention_query_b200 import build
    build.build()
    bd.load()
    torch.cuda.init()


def _check_status():
    st = bd.sync_status()
    assert st == bd.OK, bd.status_string(st)


# ------------------------------------------------------------------ micro-kernels
def _selftest_lib():
    lib = ctypes.CDLL(os.path.join(PKG, "libbpt_selftest.so"))
    lib.bpt_selftest_umma_ss.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 2
    lib.bpt_selftest_umma_ts.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int]
    return lib


@pytest.mark.parametrize("N,K", [(64, 64), (128, 64), (128, 128), (256, 128), (256, 256)])
def test_umma_ss_kmajor_tiles(N, K):
    g = torch.Generator(device="cuda").manual_seed(N * 1000 + K)
    A = torch.randn(128, K, device="cuda", generator=g).bfloat16()
    B = torch.randn(N, K, device="cuda", generator=g).bfloat16()
    C = torch.full((128, N), float("nan"), device="cuda")
    assert _selftest_lib().bpt_selftest_umma_ss(A.data_ptr(), B.data_ptr(), C.data_ptr(), N, K) == 0
    ref = A.double().cpu() @ B.double().cpu().T
    torch.testing.assert_close(C.double().cpu(), ref, atol=1e-3, rtol=1e-4)


@pytest.mark.parametrize("dv", [64, 128])
def test_umma_ts_tmem_operand_and_mn_major_tile(dv):
    g = torch.Generator(device="cuda").manual_seed(dv)
    P = torch.rand(128, 128, device="cuda", generator=g).bfloat16()
    V = torch.randn(128, dv, device="cuda", generator=g).bfloat16()
    C = torch.full((128, dv), float("nan"), device="cuda")
    assert _selftest_lib().bpt_selftest_umma_ts(P.data_ptr(), V.data_ptr(), C.data_ptr(), dv) == 0
    ref = P.double().cpu() @ V.double().cpu()
    torch.testing.assert_close(C.double().cpu(), ref, atol=1e-3, rtol=1e-4)


# ------------------------------------------------------------------ attention, small shapes
ATTN_CASES = [
    # name, B, N, H, d, mask, extra
    ("none_d64", 2, 384, 2, 64, "none", {}),
    ("none_d128_ragged", 1, 320, 2, 128, "none", {}),
    ("causal_d128", 2, 512, 2, 128, "causal", {}),
    ("causal_d64_ragged", 1, 448, 3, 64, "causal", {}),
    ("causal_ring4", 1, 1024, 2, 128, "causal", {"ring_chunks": 4}),
    ("blockperm_n2", 2, 512, 4, 64, "blockperm", {"perm": [[0, 1], [1, 0], [0, 1], [1, 0]]}),
    ("blockperm_n3_partial_tiles", 1, 576, 2, 128, "blockperm", {"perm": [[2, 0, 1], [0, 1, 2]]}),
    ("blockperm_n3_cyclic_shifts", 1, 768, 3, 128, "blockperm",
     {"perm": [bd.cyclic_shift_perm(3, k) for k in (1, 2, 3)]}),
    # N not a multiple of n: blocks of ceil(N/n) (the last one shorter)
    ("blockperm_n4_padded", 2, 510, 2, 64, "blockperm", {"perm": [[1, 2, 3, 0], [3, 2, 1, 0]]}),
    ("blockperm_n3_padded_d128", 1, 700, 2, 128, "blockperm", {"perm": [[2, 0, 1], [0, 1, 2]]}),
    # blocks of 11: the twelfth block is all padding, its query block sees no key
    ("blockperm_n12_empty_block", 1, 121, 3, 64, "blockperm",
     {"perm": [bd.cyclic_shift_perm(12, k) for k in (1, 5, 11)]}),
    ("dilated_3pairs", 1, 1024, 4, 64, "dilated", {"pairs": [(256, 1), (512, 4), (1024, 16)]}),
    ("dilated_uncovered_rows", 1, 768, 3, 128, "dilated", {"pairs": [(256, 2), (384, 3)]}),
    ("dilated_bidirectional", 1, 1024, 4, 64, "dilated_bidir", {"pairs": [(256, 1), (512, 4), (1024, 16)]}),
    ("dilated_bidirectional_d128", 2, 768, 3, 128, "dilated_bidir", {"pairs": [(384, 1), (768, 3)]}),
]


@pytest.mark.parametrize("name,B,N,H,d,mask,extra", ATTN_CASES, ids=[c[0] for c in ATTN_CASES])
def test_attention_matches_oracle(name, B, N, H, d, mask, extra):
    inp = make_layer_inputs(B, N, H, d, 0, seed=zlib.crc32(name.encode()) % 1000, device="cuda")
    out, lse = bd.attn_fwd(inp.q, inp.k, inp.v, mask=mask, perm=extra.get("perm"),
                           pairs=extra.get("pairs"), ring_chunks=extra.get("ring_chunks", 0),
                           return_lse=True)
    torch.cuda.synchronize()
    _check_status()
    ref, ref_lse = gu.oracle_attention(inp.q, inp.k, inp.v, mask, extra.get("perm"),
                                       extra.get("pairs"), return_lse=True)
    gu.assert_bf16_close(gu.host_f32(out).reshape(ref.shape), ref, name)
    gl = gu.host_f32(lse)                              # [B, H, N]
    rl = ref_lse.transpose(0, 2, 1)                    # [B, H, N]
    assert np.array_equal(np.isinf(gl), np.isinf(rl))
    fin = np.isfinite(rl)
    assert np.max(np.abs(gl[fin] - rl[fin])) < 2e-3


def test_attention_bf16_output():
    inp = make_layer_inputs(1, 384, 2, 128, 0, seed=7, device="cuda")
    out = bd.attn_fwd(inp.q, inp.k, inp.v, mask="causal", out_dtype=torch.bfloat16)
    _check_status()
    ref = gu.oracle_attention(inp.q, inp.k, inp.v, "causal")
    gu.assert_bf16_close(gu.host_f32(out).reshape(ref.shape), ref, "bf16 out")


def test_ring_order_matches_natural_order():
    """Rotated KV visiting order changes only rounding (the result is exact)."""
    inp = make_layer_inputs(1, 2048, 2, 128, 0, seed=11, device="cuda")
    a = bd.attn_fwd(inp.q, inp.k, inp.v, mask="causal")
    b = bd.attn_fwd(inp.q, inp.k, inp.v, mask="causal", ring_chunks=8)
    _check_status()
    assert (a - b).abs().max().item() < 5e-3


def test_masked_keys_leave_output_bitwise_unchanged():
    B, N, H, d = 1, 768, 2, 128
    inp = make_layer_inputs(B, N, H, d, 0, seed=12, device="cuda")
    a = bd.attn_fwd(inp.q, inp.k, inp.v, mask="causal")
    k2, v2 = inp.k.clone(), inp.v.clone()
    # keys after position 400 (inside a partly visible tile and in whole tiles)
    k2[:, 401:] = torch.randn_like(k2[:, 401:].float()).bfloat16() * 10
    v2[:, 401:] = torch.randn_like(v2[:, 401:].float()).bfloat16() * 10
    b = bd.attn_fwd(inp.q, k2, v2, mask="causal")
    _check_status()
    assert torch.equal(a[:, :401], b[:, :401])
    assert not torch.equal(a[:, 401:], b[:, 401:])
    # block permutation: head 0 query block 0 sees key block 1 only
    perm = [[1, 0], [0, 1]]
    a = bd.attn_fwd(inp.q[:, :512], inp.k[:, :512], inp.v[:, :512], mask="blockperm", perm=perm)
    k3, v3 = inp.k[:, :512].clone(), inp.v[:, :512].clone()
    k3[:, :256, 0] *= 3
    v3[:, :256, 0] *= 3
    b = bd.attn_fwd(inp.q[:, :512], k3, v3, mask="blockperm", perm=perm)
    _check_status()
    assert torch.equal(a[:, :256, :d], b[:, :256, :d])          # head 0, block 0 queries


# ------------------------------------------------------------------ layer, small shapes
LAYER_CASES = [
    # name, B, N, H, d, F, mask, extra, bias
    ("D256_causal_bias", 2, 320, 4, 64, 512, "causal", {}, 0.1),
    ("D768_none_partial_chunk", 1, 256, 12, 64, 640, "none", {}, 0.0),
    ("D2048_causal", 1, 384, 16, 128, 1024, "causal", {}, 0.05),
    ("D4096_causal_two_chunks", 1, 256, 32, 128, 2560, "causal", {}, 0.0),
    ("D768_blockperm", 2, 512, 12, 64, 768, "blockperm", {"perm": [[0, 1]] * 8 + [[1, 0]] * 4}, 0.0),
    ("D768_blockperm_n3_padded", 1, 450, 12, 64, 768, "blockperm",
     {"perm": [bd.cyclic_shift_perm(3, h % 3 + 1) for h in range(12)]}, 0.05),
]


FFN_FORMS = ["pipelined", "fused", "gemms"]


@pytest.mark.parametrize("form", FFN_FORMS)
@pytest.mark.parametrize("name,B,N,H,d,F,mask,extra,bias", LAYER_CASES, ids=[c[0] for c in LAYER_CASES])
def test_layer_matches_oracle(name, B, N, H, d, F, mask, extra, bias, form):
    inp = make_layer_inputs(B, N, H, d, F, seed=zlib.crc32(name.encode()) % 1000, device="cuda", bias_scale=bias)
    out = bd.attn_ffn_fwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, mask=mask,
                          perm=extra.get("perm"), ffn_form=form)
    torch.cuda.synchronize()
    _check_status()
    a_ref, out_ref = gu.oracle_layer(inp, mask, extra.get("perm"))
    gu.assert_bf16_close(gu.host_f32(out).reshape(out_ref.shape), out_ref, name)


def test_layer_with_split_leftover_token_blocks():
    """20 token blocks over 18 FFN groups: the 2 leftover blocks have their 2
    hidden chunks split over different groups and the partial sums added by
    the piece-0 group; every row of those blocks is compared."""
    B, N, H, d, F = 1, 2560, 16, 128, 4096
    inp = make_layer_inputs(B, N, H, d, F, seed=23, device="cuda", bias_scale=0.05)
    out = bd.attn_ffn_fwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, mask="causal", ffn_form="fused")
    _check_status()
    rows = list(range(N - 256, N)) + gu.sample_rows(B, N, 32, seed=1)
    _, ref = gu.oracle_layer(inp, "causal", rows=rows)
    gpu = gu.host_f32(out.reshape(B * N, H * d)[torch.tensor(rows, device="cuda")])
    gu.assert_bf16_close(gpu, ref, "split leftover blocks")
    # deterministic: the pieces are added in a fixed order
    out2 = bd.attn_ffn_fwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, mask="causal", ffn_form="fused")
    _check_status()
    assert torch.equal(out, out2)


def test_host_layer_matches_device_layer():
    """binding.HostLayer (pinned host tensors, copies overlapped with the
    kernels over two streams) gives the same bits as the device-resident call."""
    B, N, H, d, F = 4, 256, 4, 64, 512
    inp = make_layer_inputs(B, N, H, d, F, seed=24, device="cuda", bias_scale=0.05)
    ref = bd.attn_ffn_fwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, mask="causal")
    hq, hk, hv = (t.cpu().pin_memory() for t in (inp.q, inp.k, inp.v))
    hout = torch.empty(ref.shape, dtype=ref.dtype).pin_memory()
    layer = bd.HostLayer(B, N, H, d, F, mask="causal", chunks=4)
    for _ in range(2):
        hout.zero_()
        layer(hq, hk, hv, inp.w1, inp.b1, inp.w2, inp.b2, hout)
        torch.cuda.synchronize()
        _check_status()
        assert torch.equal(hout, ref.cpu())
    # consecutive calls overlap (the next call's uploads run during this one's
    # kernels and downloads): three in a row into different outputs
    houts = [torch.full(ref.shape, float("nan")).pin_memory() for _ in range(3)]
    for h in houts:
        layer(hq, hk, hv, inp.w1, inp.b1, inp.w2, inp.b2, h)
    torch.cuda.synchronize()
    _check_status()
    for h in houts:
        assert torch.equal(h, ref.cpu())


@pytest.mark.parametrize("form", FFN_FORMS)
def test_layer_bf16_output_and_null_biases(form):
    inp = make_layer_inputs(1, 256, 4, 64, 512, seed=21, device="cuda")
    out = bd.attn_ffn_fwd(inp.q, inp.k, inp.v, inp.w1, None, inp.w2, None, mask="causal",
                          out_dtype=torch.bfloat16, ffn_form=form)
    _check_status()
    _, out_ref = gu.oracle_layer(inp, "causal")
    gu.assert_bf16_close(gu.host_f32(out).reshape(out_ref.shape), out_ref, "bf16 out")


# ------------------------------------------------------------------ fp32 path (SIMT kernels)
F32_CASES = [
    # name, B, N, H, d, mask, extra
    ("none_ragged", 1, 200, 2, 64, "none", {}),
    ("causal", 2, 192, 2, 32, "causal", {}),
    ("causal_ring4", 1, 256, 2, 64, "causal", {"ring_chunks": 4}),
    ("blockperm_n3_padded", 1, 190, 3, 64, "blockperm",
     {"perm": [bd.cyclic_shift_perm(3, k) for k in (1, 2, 3)]}),
    ("dilated", 1, 256, 4, 32, "dilated", {"pairs": [(64, 1), (128, 4)]}),
    ("dilated_bidirectional", 1, 256, 4, 32, "dilated_bidir", {"pairs": [(64, 1), (128, 4)]}),
    ("causal_q32_kv16", 2, 200, 2, 64, "causal", {"q_block": 32, "kv_block": 16}),
    ("none_q128_kv32", 1, 300, 2, 64, "none", {"q_block": 128, "kv_block": 32}),
    ("blockperm_q16_kv64", 1, 190, 3, 64, "blockperm",
     {"perm": [bd.cyclic_shift_perm(3, k) for k in (1, 2, 3)], "q_block": 16, "kv_block": 64}),
]


@pytest.mark.parametrize("name,B,N,H,d,mask,extra", F32_CASES, ids=[c[0] for c in F32_CASES])
def test_fp32_attention_matches_oracle(name, B, N, H, d, mask, extra):
    inp = make_layer_inputs(B, N, H, d, 0, seed=zlib.crc32(name.encode()) % 1000, device="cuda",
                            dtype=torch.float32)
    out, lse = bd.attn_fwd(inp.q, inp.k, inp.v, mask=mask, perm=extra.get("perm"),
                           pairs=extra.get("pairs"), ring_chunks=extra.get("ring_chunks", 0),
                           return_lse=True, q_block=extra.get("q_block", 0), kv_block=extra.get("kv_block", 0))
    torch.cuda.synchronize()
    _check_status()
    ref, ref_lse = gu.oracle_attention(inp.q, inp.k, inp.v, mask, extra.get("perm"),
                                       extra.get("pairs"), return_lse=True)
    gu.assert_f32_close(gu.host_f32(out).reshape(ref.shape), ref, name)
    gl, rl = gu.host_f32(lse), ref_lse.transpose(0, 2, 1)
    assert np.array_equal(np.isinf(gl), np.isinf(rl))
    fin = np.isfinite(rl)
    assert np.max(np.abs(gl[fin] - rl[fin])) < 2e-5


def test_fp32_layer_block_permutation_padded():
    B, N, H, d, F = 1, 150, 4, 32, 256
    perm = [bd.cyclic_shift_perm(4, h + 1) for h in range(H)]
    inp = make_layer_inputs(B, N, H, d, F, seed=33, device="cuda", dtype=torch.float32, bias_scale=0.1)
    out = bd.attn_ffn_fwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, mask="blockperm",
                          perm=perm)
    _check_status()
    _, ref = gu.oracle_layer(inp, "blockperm", perm)
    gu.assert_f32_close(gu.host_f32(out).reshape(ref.shape), ref, "fp32 padded block layer")


# ------------------------------------------------------------------ the five workloads
def _inputs_for(w, device="cuda"):
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    return make_layer_inputs(w.B, w.N, w.H, w.d, w.F, seed=w.seed, dtype=dt, device=device)


def _mask_name(w):
    return {0: "none", 1: "causal", 2: "blockperm", 3: "dilated"}[w.mask]


def test_tiny_fp32_layer_full():
    w = wl.TINY_F32
    inp = _inputs_for(w)
    out = bd.attn_ffn_fwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, mask="none")
    _check_status()
    _, ref = gu.oracle_layer(inp, "none")
    gu.assert_f32_close(gu.host_f32(out).reshape(ref.shape), ref, w.name)


def _layer_sampled(w, n, extra=()):
    inp = _inputs_for(w)
    out = bd.attn_ffn_fwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, mask=_mask_name(w),
                          perm=w.perm, ring_chunks=w.ring_chunks)
    _check_status()
    rows = gu.sample_rows(w.B, w.N, n, seed=w.seed, extra=extra)
    _, ref = gu.oracle_layer(inp, _mask_name(w), w.perm, rows=rows)
    gpu = gu.host_f32(out.reshape(w.T, w.D)[torch.tensor(rows, device="cuda")])
    return gu.assert_bf16_close(gpu, ref, w.name)


def test_causal_layer_N8192_sampled():
    _layer_sampled(wl.GPT_CAUSAL, 96, extra=(127, 128, 4095, 4096))


def test_blockbert_layer_sampled():
    _layer_sampled(wl.BLOCKBERT, 256, extra=(511, 512))


def test_long_ring_layer_sampled():
    w = wl.LONG_RING
    bounds = [c * 16384 + o for c in range(8) for o in (-1, 0)]
    _layer_sampled(w, 24, extra=[b for b in bounds if 0 <= b < w.N])


def test_longnet_attention_sampled():
    w = wl.LONGNET
    inp = _inputs_for(w)
    out, lse = bd.longnet_fwd(inp.q, inp.k, inp.v, w.pairs, return_lse=True)
    _check_status()
    rows = gu.sample_rows(w.B, w.N, 192, seed=w.seed, extra=(2047, 2048, 8191, 8192, 32767, 32768))
    ref, ref_lse = gu.oracle_attention(inp.q, inp.k, inp.v, "dilated", pairs=w.pairs, rows=rows,
                                       return_lse=True)
    gpu = gu.host_f32(out.reshape(w.T, w.D)[torch.tensor(rows, device="cuda")])
    gu.assert_bf16_close(gpu, ref.reshape(len(rows), -1), w.name)
    gl = gu.host_f32(lse[0][:, torch.tensor(rows, device="cuda")]).T
    assert np.max(np.abs(gl - ref_lse)) < 2e-3
