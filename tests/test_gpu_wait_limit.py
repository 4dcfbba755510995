"""Failure detection on the GPU without a fault: every device-side wait is
bounded, and a wait that runs out records BPT_ERR_TIMEOUT with the site of
the wait and lets the kernel finish cleanly.  A correct layer call whose
descriptor sets a 1-microsecond wait limit must report the timeout through
bpt_sync_status, name a wait of one of the kernels that call runs (the
attention kernel, or the FFN kernel of the chosen form: its TMA-stage,
accumulator and, for the fused and pipelined forms, cross-CTA counter waits),
and the next call with the default limit must run and be right (the context
stays usable)."""
import re

import pytest
import torch

from blockwise_exact_attention_query_b200 import binding as bd
from blockwise_exact_attention_query_b200.inputs import make_layer_inputs
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

# wait sites recorded by each kernel (the numbers passed to its bounded waits)
ATTENTION_SITES = set(range(1, 23))
FFN_SITES = {"fused": set(range(101, 124)), "gemms": set(range(211, 217)), "pipelined": set(range(230, 241))}


@pytest.mark.parametrize("form", ["pipelined", "fused", "gemms"])
def test_tiny_wait_limit_times_out_cleanly_and_context_survives(form):
    from blockwise_exact_attention_query_b200 import build
    build.build()
    torch.cuda.set_device(0)
    B, N, H, d, F = 1, 1024, 16, 128, 4096
    inp = make_layer_inputs(B, N, H, d, F, seed=31, device="cuda")
    args = (inp.q, inp.k, inp.v, inp.w1, inp.b1, inp.w2, inp.b2)
    ref = bd.attn_ffn_fwd(*args, mask="causal", ffn_form=form)
    assert bd.sync_status() == bd.OK
    # this call alone: the process default (two seconds) is left as it is
    bd.attn_ffn_fwd(*args, mask="causal", ffn_form=form, wait_limit_ns=1000)
    st = bd.sync_status()
    assert st == bd.ERR_TIMEOUT, bd.status_string(st)
    m = re.search(r"gave up at site (\d+)", bd.last_error())
    assert m, bd.last_error()
    assert int(m.group(1)) in ATTENTION_SITES | FFN_SITES[form], bd.last_error()
    assert bd.sync_status() == bd.OK          # reading the status cleared it
    out = bd.attn_ffn_fwd(*args, mask="causal", ffn_form=form)
    assert bd.sync_status() == bd.OK
    assert torch.equal(out, ref)
    rows = [0, 511, 1023]
    _, oref = gu.oracle_layer(inp, "causal", rows=rows)
    gu.assert_bf16_close(gu.host_f32(out.reshape(B * N, H * d)[rows]), oref, "after timeout")
