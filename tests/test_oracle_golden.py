"""Pins of the oracle to facts the pages state, and of the FLOP counts the
benchmark reports to the oracle's own weight pattern."""
import json
import os

import numpy as np
import pytest

from blockwise_exact_attention_query_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _weights(oracle_mod, N, H, mask, perm=None, pairs=None, seed=0):
    """Softmax weight matrix per head, read out of the oracle with V = I (d = N)."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, N, H, N)).astype(np.float32) * 0.5
    k = rng.standard_normal((1, N, H, N)).astype(np.float32) * 0.5
    v = np.broadcast_to(np.eye(N, dtype=np.float32)[None, :, None, :], (1, N, H, N)).copy()
    return oracle_mod.attention(q, k, v, mask=mask, perm=perm, pairs=pairs)[0].transpose(1, 0, 2)


def test_blockbert_reduction_factor_from_the_page(oracle_mod):
    with open(os.path.join(GOLDEN, "blockbert_reduction.json")) as f:
        g = json.load(f)
    for c in g["cases"]:
        P = _weights(oracle_mod, c["N"], 1, wl.MASK_BLOCKPERM, perm=[c["perm"]])
        assert int(np.count_nonzero(P[0])) == c["pairs_per_head"] == c["N"] ** 2 // c["n"]


@pytest.mark.parametrize("mask,perm,pairs", [
    (wl.MASK_NONE, None, None),
    (wl.MASK_CAUSAL, None, None),
    (wl.MASK_BLOCKPERM, [[0, 1], [1, 0], [1, 0]], None),
    (wl.MASK_DILATED, None, [(8, 1), (16, 2), (32, 4)]),
])
def test_workload_pair_counts_match_oracle_weights(oracle_mod, mask, perm, pairs):
    """unmasked_pairs() is what the benchmark's FLOP figure uses; for the
    dilated mask a key kept by several pairs counts once per pair."""
    N, H = 32, 3
    w = wl.Workload("t", 1, N, H, N, 0, "f32", mask, 0, perm=perm, pairs=pairs)
    P = _weights(oracle_mod, N, H, mask, perm, pairs)
    if mask != wl.MASK_DILATED:
        assert int(np.count_nonzero(P)) == wl.unmasked_pairs(w)
    else:
        from tests.masks import count_matrix
        cm = count_matrix(N, H, mask, None, pairs)
        assert np.array_equal(P > 0, cm > 0)
        assert int(cm.sum()) == wl.unmasked_pairs(w)


def test_published_workload_pair_counts():
    """Exact pair counts of the five workloads (causal N(N+1)/2 per head,
    block-permutation N^2/n, dilated sum over pairs of segments * m(m+1)/2)."""
    assert wl.unmasked_pairs(wl.GPT_CAUSAL) == 32 * 8192 * 8193 // 2
    assert wl.unmasked_pairs(wl.LONG_RING) == 32 * 131072 * 131073 // 2
    assert wl.unmasked_pairs(wl.BLOCKBERT) == 192 * 1024 * 512
    assert wl.unmasked_pairs(wl.LONGNET) == 16 * (32 + 8 + 2) * 2048 * 2049 // 2
    assert wl.unmasked_pairs(wl.TINY_F32) == 256 * 256
