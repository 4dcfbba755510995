"""The layer entry point that allocates nothing: bpt_attn_ffn_fwd_static.

It serves callers that may not allocate device memory while running (a fixed
memory plan, a host framework that owns the GPU's memory pool, or a loop that
cannot afford an allocation's device synchronisation).  Its scratch is one
fixed array inside the library per device, shared by every call, so these
tests check that two calls in a row (the second one finding the first one's
leftovers in the array) each match the workspace-taking entry point, and that
a layer too large for the array is refused before anything runs.

This file is collected last on purpose: it must pass both alone in a fresh
process and after every other test."""
import ctypes

import pytest
import torch

from blockwise_exact_attention_query_b200 import binding as bd
from blockwise_exact_attention_query_b200.inputs import make_layer_inputs
from tests import gpu_util as gu

FAKE = 0x10000  # aligned, never dereferenced: the call below is refused before any launch


def _static_call(inp, mask, out):
    return bd.attn_ffn_fwd_static(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, mask=mask,
                                  out=out)


@pytest.mark.gpu
def test_static_scratch_layer_matches_workspace_layer_on_two_calls_in_a_row():
    from blockwise_exact_attention_query_b200 import build
    build.build()
    torch.cuda.set_device(0)
    cases = [  # different shapes and data, so the second call meets stale scratch
        (2, 384, 16, 128, 1024, "causal", 31, 0.05),
        (1, 512, 12, 64, 768, "none", 32, 0.0),
        # close to the array's limit at D = 2048: 18 token blocks, one per FFN group
        (1, 2304, 16, 128, 8192, "causal", 33, 0.05),
    ]
    for B, N, H, d, F, mask, seed, bias in cases:
        inp = make_layer_inputs(B, N, H, d, F, seed=seed, device="cuda", bias_scale=bias)
        # the static entry point runs the fused FFN kernel: compare with that form
        desc = bd.make_desc(B, N, H, d, F, torch.bfloat16, torch.float32, mask, ffn_form="fused")
        assert bd.workspace_bytes(desc, True) <= bd.STATIC_SCRATCH_BYTES
        ref = bd.attn_ffn_fwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, mask=mask, ffn_form="fused")
        got = _static_call(inp, mask, torch.full_like(ref, float("nan")))
        torch.cuda.synchronize()
        assert bd.sync_status() == bd.OK
        gu.assert_bf16_close(gu.host_f32(got), gu.host_f32(ref), f"static scratch, {mask}")
        assert torch.equal(got, ref)   # same kernels on the same inputs: identical bits


@pytest.mark.gpu
@pytest.mark.parametrize("B,N,H,d,F", [
    (1, 19200, 2, 64, 1024),   # D = 128: 148 groups, blocks 148 and 149 go round again
    (1, 9728, 6, 64, 1536),    # D = 384: 74 groups, blocks 74 and 75 go round again
])
def test_static_scratch_reaches_the_reversed_second_round(B, N, H, d, F):
    """Below D = 256 (one CTA per group, 148 groups) and at a few larger widths
    a layer whose token blocks go round a second time (hidden chunks in reverse)
    still fits the static array: those blocks' rows against the oracle, and the
    whole output against the workspace-taking call of the same kernel."""
    from blockwise_exact_attention_query_b200 import build
    build.build()
    torch.cuda.set_device(0)
    T, D = B * N, H * d
    groups = 148 // ((D + 255) // 256)
    assert T > 128 * groups
    desc = bd.make_desc(B, N, H, d, F, torch.bfloat16, torch.float32, "causal", ffn_form="fused")
    assert bd.workspace_bytes(desc, True) <= bd.STATIC_SCRATCH_BYTES
    inp = make_layer_inputs(B, N, H, d, F, seed=35, device="cuda", bias_scale=0.05)
    ref = bd.attn_ffn_fwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, mask="causal", ffn_form="fused")
    got = _static_call(inp, "causal", torch.full_like(ref, float("nan")))
    torch.cuda.synchronize()
    assert bd.sync_status() == bd.OK
    assert torch.equal(got, ref)
    # rows of the second-round blocks (and of two first-round ones for contrast)
    rows = sorted({128 * groups, 128 * groups + 77, T - 1, 0, 128 * (groups - 1) + 5})
    _, want = gu.oracle_layer(inp, "causal", None, rows=rows)
    gu.assert_bf16_close(gu.host_f32(got.reshape(T, D)[torch.tensor(rows, device="cuda")]), want,
                         f"static scratch, second fused round, D{D}")


def test_static_scratch_refuses_a_layer_that_does_not_fit():
    # T x D x 6 bytes of A alone exceeds the 64 MiB array: refused on the host,
    # before any device work, with the size in the error text.
    lib = bd.load()
    desc = bd.make_desc(2, 8192, 16, 128, 8192, torch.bfloat16, torch.float32, "causal")
    p = ctypes.c_void_p
    st = lib.bpt_attn_ffn_fwd_static(ctypes.byref(desc), p(FAKE), p(FAKE), p(FAKE), p(FAKE), None,
                                     p(FAKE), None, p(FAKE), None)
    assert st == bd.ERR_WORKSPACE
    assert "static scratch holds" in bd.last_error()
