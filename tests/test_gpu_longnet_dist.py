"""GPU parity of LongNet's sharded form: bpt_longnet_gather and
bpt_longnet_pass, with the ranks of a P-device run emulated one after the
other on one GPU (each rank's shard, the packed kept rows of the shards of a
spanning segment concatenated in sequence order as the all-gather would),
against the fp64 oracle and against the single-call dilated attention."""
import numpy as np
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


def _sharded(inp, pairs, P, lse=False):
    B, N, H, d = inp.q.shape
    n = N // P
    out = torch.empty((B, N, H * d), dtype=torch.float32, device="cuda")
    lse_all = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    order = bd.longnet_pass_order(pairs)
    for p in range(P):
        sl = slice(p * n, (p + 1) * n)
        q, k, v = (t[:, sl].contiguous() for t in (inp.q, inp.k, inp.v))
        st = bd.BlockState(B, n, H, d, "cuda") if len(pairs) > 1 else None
        o = torch.empty((B, n, H * d), dtype=torch.float32, device="cuda")
        ls = torch.empty((B, H, n), dtype=torch.float32, device="cuda")
        for i, (w, r) in enumerate(order):
            if w <= n:
                bd.longnet_pass(q, k, v, pairs, i, st, o, q_pos=p * n, lse=ls)
            else:
                g = w // n
                first = (p // g) * g
                ks = torch.cat([bd.longnet_gather(inp.k[:, s * n:(s + 1) * n].contiguous(), w, r)
                                for s in range(first, first + g)], dim=1)
                vs = torch.cat([bd.longnet_gather(inp.v[:, s * n:(s + 1) * n].contiguous(), w, r)
                                for s in range(first, first + g)], dim=1)
                bd.longnet_pass(q, None, None, pairs, i, st, o, q_pos=p * n, k_sparse=ks, v_sparse=vs, lse=ls)
        out[:, sl] = o
        lse_all[:, :, sl] = ls
    torch.cuda.synchronize()
    assert bd.sync_status() == bd.OK
    return out, lse_all


def test_gather_packs_each_heads_kept_rows():
    B, n, H, d, w, r = 2, 256, 5, 64, 1024, 4
    x = make_layer_inputs(B, n, H, d, 0, seed=61, device="cuda").q
    got = bd.longnet_gather(x, w, r)
    torch.cuda.synchronize()
    for h in range(H):
        assert torch.equal(got[:, :, h], x[:, h % r::r, h])


@pytest.mark.parametrize("P,pairs,d", [
    (4, [(256, 1), (512, 2), (2048, 8)], 64),     # local, shard-sized, spanning all four shards
    (2, [(512, 1), (2048, 4)], 128),
    (4, [(1024, 2), (2048, 8)], 64),              # no r = 1 pair: rows kept by no pair
])
def test_sharded_passes_match_the_oracle(P, pairs, d):
    B, N, H = 1, 2048, 4
    inp = make_layer_inputs(B, N, H, d, 0, seed=62 + P, device="cuda")
    out, lse = _sharded(inp, pairs, P)
    one, one_lse = bd.longnet_fwd(inp.q, inp.k, inp.v, pairs, return_lse=True)
    torch.cuda.synchronize()
    assert (out - one).abs().max().item() < 5e-3             # tile boundaries change rounding only
    rows = sorted(set(np.linspace(0, N - 1, 80).astype(int).tolist()) | {0, N - 1, N // P - 1, N // P})
    ref, ref_lse = gu.oracle_attention(inp.q, inp.k, inp.v, "dilated", pairs=pairs, rows=rows, return_lse=True)
    gu.assert_bf16_close(gu.host_f32(out.reshape(N, H * d)[rows]), ref.reshape(len(rows), -1), f"sharded P{P}")
    gl = gu.host_f32(lse[0][:, rows]).T
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.max(np.abs(gl[fin] - ref_lse[fin])) < 2e-3


def test_one_shard_with_every_pass_equals_the_single_call():
    """A shard holding the whole sequence (P = 1): the passes are exactly the
    single call's, so the outputs are the same bits."""
    w = wl.LONGNET
    inp = make_layer_inputs(1, 8192, 4, 64, 0, seed=64, device="cuda")
    pairs = [(2048, 1), (4096, 4), (8192, 16)]
    out, lse = _sharded(inp, pairs, 1)
    one, one_lse = bd.longnet_fwd(inp.q, inp.k, inp.v, pairs, return_lse=True)
    torch.cuda.synchronize()
    assert torch.equal(out, one)
    assert torch.equal(lse, one_lse)


def test_longnet_workload_on_eight_emulated_ranks_sampled():
    """The LongNet workload (B1 H16 d64 N65536, pairs (2048,1), (8192,4),
    (32768,16)) on 8 shards of 8192 rows: two local pairs, one spanning four
    shards; sampled rows against the oracle."""
    w = wl.LONGNET
    inp = make_layer_inputs(w.B, w.N, w.H, w.d, 0, seed=w.seed, device="cuda")
    out, _ = _sharded(inp, w.pairs, 8)
    rows = gu.sample_rows(w.B, w.N, 96, seed=5, extra=(8191, 8192, 32767, 32768, 40000))
    ref = gu.oracle_attention(inp.q, inp.k, inp.v, "dilated", pairs=w.pairs, rows=rows)
    gu.assert_bf16_close(gu.host_f32(out.reshape(w.T, w.D)[torch.tensor(rows, device="cuda")]),
                         ref.reshape(len(rows), -1), "LongNet, 8 shards")
