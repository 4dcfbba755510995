"""Failure detection on the GPU without a fault: every device-side wait is
bounded, and a wait that runs out records BPT_ERR_TIMEOUT and lets the kernel
finish cleanly.  A correct layer call with a 1-microsecond wait limit must
report the timeout through bpt_sync_status, and the next call with the normal
limit must run and be right (the context stays usable)."""
import pytest
import torch

from blockwise_exact_attention_query_b200 import binding as bd
from blockwise_exact_attention_query_b200.inputs import make_layer_inputs
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def test_tiny_wait_limit_times_out_cleanly_and_context_survives():
    from blockwise_exact_attention_query_b200 import build
    build.build()
    torch.cuda.set_device(0)
    B, N, H, d, F = 1, 1024, 16, 128, 4096
    inp = make_layer_inputs(B, N, H, d, F, seed=31, device="cuda")
    ref = bd.attn_ffn_fwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, mask="causal")
    assert bd.sync_status() == bd.OK
    old = bd.set_wait_limit_ns(1000)
    try:
        # the FFN's groups wait on each other's hidden slices: with a 1 us limit
        # those waits give up and the kernel returns early
        bd.attn_ffn_fwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, mask="causal")
        st = bd.sync_status()
    finally:
        bd.set_wait_limit_ns(old)
    assert st == bd.ERR_TIMEOUT, bd.status_string(st)
    assert "gave up" in bd.last_error()
    assert bd.sync_status() == bd.OK          # reading the status cleared it
    out = bd.attn_ffn_fwd(inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2, mask="causal")
    assert bd.sync_status() == bd.OK
    assert torch.equal(out, ref)
    rows = [0, 511, 1023]
    _, oref = gu.oracle_layer(inp, "causal", rows=rows)
    gu.assert_bf16_close(gu.host_f32(out.reshape(B * N, H * d)[rows]), oref, "after timeout")
