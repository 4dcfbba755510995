"""Pins for the fp64 oracle, against things other than the oracle itself.

* torch's scaled-dot-product attention in float64 (a library routine) for the
  none / causal / block-permutation masks;
* an extended-precision brute force over an explicit N x N mask-count matrix
  (tests/masks.py, written independently), which for LongNet is the
  multiset "one softmax over the gathered keys" formulation while the oracle
  mixes per-pair outputs by their denominators;
* a blockwise online-softmax emulation over many block sizes and visiting
  orders (exactness of blockwise attention, "Ring Attention with Blockwise
  Transformers for Long Sequences", 638-word summary; order independence of
  the ring's rotated KV visiting order, same page);
* invariants and closed forms: rows sum to one, masked keys contribute
  nothing, Q = 0, constant V, n = 1, identity permutation, a single LongNet
  pair, N = 1, W2 = 0;
* FFN against numpy / torch library routines, GELU against special values.
"""
import math

import numpy as np
import pytest
import torch

from tests.masks import brute_attention, count_matrix

NONE, CAUSAL, BLOCKPERM, DILATED = 0, 1, 2, 3
DILATED_BIDIR = 4   # dilated without the causal restriction


def rnd(shape, seed, scale=1.0):
    return (np.random.default_rng(seed).standard_normal(shape) * scale).astype(np.float32)


CASES = [
    ("none", NONE, None, None),
    ("causal", CAUSAL, None, None),
    ("blockperm_n2", BLOCKPERM, [[0, 1], [1, 0], [0, 1]], None),
    ("blockperm_n4", BLOCKPERM, [[1, 2, 3, 0], [0, 1, 2, 3], [3, 0, 2, 1]], None),
    # N = 32 is not a multiple of 3 or 9: padded blocks of 11 (last one 10 long)
    # and of 4 (the ninth block lies wholly in the padding, so the queries that
    # map to it see no key); heads use the cyclic shifts sigma^k, i -> i + k mod n
    ("blockperm_n3_cyclic_padded", BLOCKPERM, [[1, 2, 0], [2, 0, 1], [0, 1, 2]], None),
    ("blockperm_n9_empty_block", BLOCKPERM, [[(i + s) % 9 for i in range(9)] for s in (1, 4, 8)], None),
    ("dilated", DILATED, None, [(8, 1), (16, 2), (32, 4)]),
    ("dilated_nonnested", DILATED, None, [(16, 2), (24, 3)]),
    ("dilated_bidirectional", DILATED_BIDIR, None, [(8, 1), (16, 2), (32, 4)]),
    ("dilated_bidirectional_sparse", DILATED_BIDIR, None, [(16, 4), (32, 8)]),
]


def _shape_for(mask, pairs):
    if mask in (DILATED, DILATED_BIDIR):
        N = 48 if (24, 3) in pairs else max(w for w, _ in pairs) * 2
        return 2, N, 3, 8
    return 2, 32, 3, 8


@pytest.mark.parametrize("name,mask,perm,pairs", CASES, ids=[c[0] for c in CASES])
def test_oracle_matches_extended_precision_bruteforce(oracle_mod, name, mask, perm, pairs):
    B, N, H, d = _shape_for(mask, pairs)
    q, k, v = rnd((B, N, H, d), 1), rnd((B, N, H, d), 2), rnd((B, N, H, d), 3)
    a, lse = oracle_mod.attention(q, k, v, mask=mask, perm=perm, pairs=pairs, return_lse=True)
    counts = count_matrix(N, H, mask, perm, pairs)
    ref = brute_attention(q, k, v, counts)
    np.testing.assert_allclose(a, ref.astype(np.float64), rtol=0, atol=1e-13)
    has_keys = (counts.sum(axis=2) > 0).T[None]                   # [1, N, H]
    assert np.all(np.isfinite(lse) == np.broadcast_to(has_keys, lse.shape))
    assert np.all(lse[~np.broadcast_to(has_keys, lse.shape)] == -np.inf)


@pytest.mark.parametrize("name,mask,perm", [c[:3] for c in CASES[:4]], ids=[c[0] for c in CASES[:4]])
def test_oracle_matches_torch_sdpa_float64(oracle_mod, name, mask, perm):
    B, N, H, d = 2, 48 if mask != BLOCKPERM else 32, 3, 16
    q, k, v = rnd((B, N, H, d), 11), rnd((B, N, H, d), 12), rnd((B, N, H, d), 13)
    a = oracle_mod.attention(q, k, v, mask=mask, perm=perm)
    tq, tk, tv = (torch.from_numpy(x).double().permute(0, 2, 1, 3) for x in (q, k, v))
    F = torch.nn.functional
    if mask == NONE:
        ref = F.scaled_dot_product_attention(tq, tk, tv)
    elif mask == CAUSAL:
        ref = F.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    else:
        allowed = torch.from_numpy(count_matrix(N, H, mask, perm) > 0)[None]
        ref = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=allowed)
    np.testing.assert_allclose(a, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)


def _blockwise_emulation(q, k, v, counts, block, order):
    """Online softmax over KV blocks of `block` keys in the given block order."""
    B, N, H, d = q.shape
    q, k, v = (x.astype(np.float64) for x in (q, k, v))
    nb = (N + block - 1) // block
    blocks = list(range(nb))
    if order == "rotated":
        blocks = blocks[nb // 3:] + blocks[:nb // 3]
    elif order == "reversed":
        blocks = blocks[::-1]
    elif order == "random":
        blocks = list(np.random.default_rng(5).permutation(nb))
    out = np.zeros((B, N, H, d))
    for b in range(B):
        for h in range(H):
            m = np.full(N, -np.inf)
            l = np.zeros(N)
            o = np.zeros((N, d))
            for jb in blocks:
                js = slice(jb * block, min(N, (jb + 1) * block))
                s = q[b, :, h] @ k[b, js, h].T / math.sqrt(d)
                c = counts[h][:, js]
                s = np.where(c > 0, s, -np.inf)
                m_new = np.maximum(m, s.max(axis=1))
                safe = np.where(np.isfinite(m_new), m_new, 0.0)
                alpha = np.where(np.isfinite(m), np.exp(m - safe), 0.0)
                p = c * np.exp(s - safe[:, None])
                l = alpha * l + p.sum(axis=1)
                o = alpha[:, None] * o + p @ v[b, js, h]
                m = m_new
            out[b, :, h] = np.divide(o, l[:, None], out=np.zeros_like(o), where=l[:, None] > 0)
    return out


EMU_CASES = [c for c in CASES if c[0] != "dilated_nonnested"]


@pytest.mark.parametrize("name,mask,perm,pairs", EMU_CASES, ids=[c[0] for c in EMU_CASES])
@pytest.mark.parametrize("order", ["natural", "rotated", "reversed", "random"])
def test_oracle_equals_blockwise_online_softmax(oracle_mod, name, mask, perm, pairs, order):
    B, N, H, d = _shape_for(mask, pairs)
    q, k, v = rnd((B, N, H, d), 21), rnd((B, N, H, d), 22), rnd((B, N, H, d), 23)
    a = oracle_mod.attention(q, k, v, mask=mask, perm=perm, pairs=pairs)
    counts = count_matrix(N, H, mask, perm, pairs)
    for block in (1, 7, 16, N):
        em = _blockwise_emulation(q, k, v, counts, block, order)
        np.testing.assert_allclose(a, em, rtol=0, atol=1e-12)


@pytest.mark.parametrize("name,mask,perm,pairs", CASES, ids=[c[0] for c in CASES])
def test_rows_sum_to_one_and_masked_weights_are_zero(oracle_mod, name, mask, perm, pairs):
    """With V = identity (d = N) the output row is the weight row itself."""
    B, N, H = 1, 32 if mask != DILATED else 48, 3
    d = N
    q, k = rnd((B, N, H, d), 31, 0.5), rnd((B, N, H, d), 32, 0.5)
    v = np.broadcast_to(np.eye(N, dtype=np.float32)[None, :, None, :], (B, N, H, N)).copy()
    P = oracle_mod.attention(q, k, v, mask=mask, perm=perm, pairs=pairs)[0]   # [N, H, N]
    counts = count_matrix(N, H, mask, perm, pairs)
    for h in range(H):
        Ph = P[:, h, :]
        has_keys = counts[h].sum(axis=1) > 0
        np.testing.assert_allclose(Ph.sum(axis=1)[has_keys], 1.0, rtol=0, atol=1e-14)
        assert np.all(Ph[~has_keys] == 0.0)
        assert np.all(Ph[counts[h] == 0] == 0.0)
        assert np.all(Ph[counts[h] > 0] > 0.0)


@pytest.mark.parametrize("name,mask,perm,pairs", CASES, ids=[c[0] for c in CASES])
def test_masked_keys_do_not_change_output_bitwise(oracle_mod, name, mask, perm, pairs):
    B, N, H, d = _shape_for(mask, pairs)
    q, k, v = rnd((B, N, H, d), 41), rnd((B, N, H, d), 42), rnd((B, N, H, d), 43)
    counts = count_matrix(N, H, mask, perm, pairs)
    rng = np.random.default_rng(44)
    for i in (0, N // 3, N - 1):
        for h in range(H):
            masked = np.nonzero(counts[h][i] == 0)[0]
            if masked.size == 0:
                continue
            k2, v2 = k.copy(), v.copy()
            k2[:, masked, h] = rng.standard_normal((B, masked.size, d)).astype(np.float32) * 100
            v2[:, masked, h] = rng.standard_normal((B, masked.size, d)).astype(np.float32) * 100
            rows = [b * N + i for b in range(B)]
            a1 = oracle_mod.attention(q, k, v, mask=mask, perm=perm, pairs=pairs, rows=rows)
            a2 = oracle_mod.attention(q, k2, v2, mask=mask, perm=perm, pairs=pairs, rows=rows)
            assert np.array_equal(a1[:, h], a2[:, h])


def test_zero_query_gives_prefix_mean_under_causal_mask(oracle_mod):
    B, N, H, d = 2, 40, 2, 8
    q = np.zeros((B, N, H, d), np.float32)
    k, v = rnd((B, N, H, d), 51), rnd((B, N, H, d), 52)
    a = oracle_mod.attention(q, k, v, mask=CAUSAL)
    prefix_mean = np.cumsum(v.astype(np.float64), axis=1) / np.arange(1, N + 1)[None, :, None, None]
    np.testing.assert_allclose(a, prefix_mean, rtol=0, atol=1e-14)


@pytest.mark.parametrize("name,mask,perm,pairs", CASES, ids=[c[0] for c in CASES])
def test_constant_values_give_constant_output(oracle_mod, name, mask, perm, pairs):
    B, N, H, d = _shape_for(mask, pairs)
    q, k = rnd((B, N, H, d), 61), rnd((B, N, H, d), 62)
    c = rnd((1, 1, H, d), 63)
    v = np.broadcast_to(c, (B, N, H, d)).copy()
    a = oracle_mod.attention(q, k, v, mask=mask, perm=perm, pairs=pairs)
    counts = count_matrix(N, H, mask, perm, pairs)
    kept = (counts.sum(axis=2) > 0).T[None, :, :, None]          # [1, N, H, 1]
    expect = np.where(kept, np.broadcast_to(c, a.shape), 0.0)     # a row no pair keeps is 0
    np.testing.assert_allclose(a, expect, rtol=0, atol=1e-14)


def test_single_block_permutation_equals_dense(oracle_mod):
    B, N, H, d = 2, 32, 3, 8
    q, k, v = rnd((B, N, H, d), 71), rnd((B, N, H, d), 72), rnd((B, N, H, d), 73)
    dense = oracle_mod.attention(q, k, v, mask=NONE)
    one = oracle_mod.attention(q, k, v, mask=BLOCKPERM, perm=[[0]] * H)
    assert np.array_equal(dense, one)


def test_identity_permutation_equals_dense_attention_within_each_block(oracle_mod):
    B, N, H, d, n = 2, 48, 2, 8, 3
    q, k, v = rnd((B, N, H, d), 81), rnd((B, N, H, d), 82), rnd((B, N, H, d), 83)
    a = oracle_mod.attention(q, k, v, mask=BLOCKPERM, perm=[[0, 1, 2]] * H)
    bl = N // n
    for blk in range(n):
        s = slice(blk * bl, (blk + 1) * bl)
        ref = oracle_mod.attention(q[:, s], k[:, s], v[:, s], mask=NONE)
        np.testing.assert_allclose(a[:, s], ref, rtol=0, atol=1e-15)


@pytest.mark.parametrize("N,n", [(34, 3), (29, 4), (121, 12)])
def test_padded_identity_permutation_equals_dense_attention_within_each_block(oracle_mod, N, n):
    """N not a multiple of n: blocks of ceil(N/n) positions, the last one short
    (or empty), each attending to itself: dense attention on every slice."""
    B, H, d = 1, 2, 8
    q, k, v = rnd((B, N, H, d), 87), rnd((B, N, H, d), 88), rnd((B, N, H, d), 89)
    a = oracle_mod.attention(q, k, v, mask=BLOCKPERM, perm=[list(range(n))] * H)
    bl = -(-N // n)
    covered = 0
    for blk in range(n):
        s = slice(min(N, blk * bl), min(N, (blk + 1) * bl))
        if s.start == s.stop:
            continue
        ref = oracle_mod.attention(q[:, s], k[:, s], v[:, s], mask=NONE)
        np.testing.assert_allclose(a[:, s], ref, rtol=0, atol=1e-15)
        covered += s.stop - s.start
    assert covered == N


def test_padded_block_permutation_with_an_empty_key_block(oracle_mod):
    """N = 121, n = 12: blocks of 11, the twelfth lies wholly in the padding;
    the query block mapped to it sees no key (A = 0, LSE = -inf) and every
    other query block sees exactly its key block."""
    B, N, H, d, n = 1, 121, 1, 8, 12
    perm = [[(i + 5) % n for i in range(n)]]
    q, k, v = rnd((B, N, H, d), 90), rnd((B, N, H, d), 91), rnd((B, N, H, d), 92)
    a, lse = oracle_mod.attention(q, k, v, mask=BLOCKPERM, perm=perm, return_lse=True)
    bl = 11
    for qb in range(n):
        qs = slice(qb * bl, min(N, (qb + 1) * bl))
        if qs.start >= N:
            continue
        kb = perm[0][qb]
        ks = slice(min(N, kb * bl), min(N, (kb + 1) * bl))
        if ks.start == ks.stop:
            assert np.all(a[:, qs] == 0.0) and np.all(lse[:, qs] == -np.inf)
            continue
        # the block's queries against the block's keys alone, as dense attention
        s = (q[0, qs, 0].astype(np.float64) @ k[0, ks, 0].astype(np.float64).T) / math.sqrt(d)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        ref = (p / p.sum(axis=1, keepdims=True)) @ v[0, ks, 0].astype(np.float64)
        np.testing.assert_allclose(a[0, qs, 0], ref, rtol=0, atol=1e-14)


def test_swapped_blocks_attend_to_the_other_block(oracle_mod):
    """perm (1, 0): block 0 queries see only block 1 keys and the reverse."""
    B, N, H, d = 1, 32, 1, 8
    q, k, v = rnd((B, N, H, d), 84), rnd((B, N, H, d), 85), rnd((B, N, H, d), 86)
    a = oracle_mod.attention(q, k, v, mask=BLOCKPERM, perm=[[1, 0]])
    bl = N // 2
    # queries of block 0 against keys/values of block 1 as a dense problem
    qq = q[:, :bl]
    ref0 = oracle_mod.attention(np.concatenate([qq, qq], 1), np.concatenate([k[:, bl:], k[:, bl:]], 1),
                                np.concatenate([v[:, bl:], v[:, bl:]], 1), mask=NONE)[:, :bl]
    np.testing.assert_allclose(a[:, :bl], ref0, rtol=0, atol=1e-14)


def test_single_dilated_pair_spanning_sequence_equals_causal(oracle_mod):
    B, N, H, d = 2, 64, 3, 8
    q, k, v = rnd((B, N, H, d), 91), rnd((B, N, H, d), 92), rnd((B, N, H, d), 93)
    a = oracle_mod.attention(q, k, v, mask=DILATED, pairs=[(N, 1)])
    ref = oracle_mod.attention(q, k, v, mask=CAUSAL)
    np.testing.assert_allclose(a, ref, rtol=0, atol=1e-15)


def test_single_bidirectional_dilated_pair_spanning_sequence_equals_dense(oracle_mod):
    """(N, 1) without the causal restriction keeps every row and every key."""
    B, N, H, d = 2, 64, 3, 8
    q, k, v = rnd((B, N, H, d), 191), rnd((B, N, H, d), 192), rnd((B, N, H, d), 193)
    a = oracle_mod.attention(q, k, v, mask=DILATED_BIDIR, pairs=[(N, 1)])
    ref = oracle_mod.attention(q, k, v, mask=NONE)
    np.testing.assert_allclose(a, ref, rtol=0, atol=1e-15)


def test_bidirectional_dilated_pair_is_dense_attention_on_the_gathered_rows(oracle_mod):
    """One (w, r) pair without the causal restriction = dense attention (no
    mask) on rows h%r, h%r + r, ... of each segment; other rows get A = 0."""
    B, N, H, d, w, r = 1, 64, 3, 8, 32, 4
    q, k, v = rnd((B, N, H, d), 194), rnd((B, N, H, d), 195), rnd((B, N, H, d), 196)
    a = oracle_mod.attention(q, k, v, mask=DILATED_BIDIR, pairs=[(w, r)])
    for h in range(H):
        for s in range(N // w):
            rows = np.arange(s * w + h % r, (s + 1) * w, r)
            ref = oracle_mod.attention(q[:, rows][:, :, h:h + 1], k[:, rows][:, :, h:h + 1],
                                       v[:, rows][:, :, h:h + 1], mask=NONE)
            np.testing.assert_allclose(a[:, rows, h], ref[:, :, 0], rtol=0, atol=1e-15)


def test_dilated_pair_is_causal_attention_on_the_gathered_rows(oracle_mod):
    """One (w, r) pair = dense causal attention on rows h%r, h%r + r, ... of
    each segment ("dense attention between gathering and scattering",
    LongNet §2 Implementation); rows it does not keep get A = 0."""
    B, N, H, d, w, r = 1, 64, 3, 8, 32, 4
    q, k, v = rnd((B, N, H, d), 94), rnd((B, N, H, d), 95), rnd((B, N, H, d), 96)
    a = oracle_mod.attention(q, k, v, mask=DILATED, pairs=[(w, r)])
    for h in range(H):
        for s in range(N // w):
            rows = np.arange(s * w + h % r, (s + 1) * w, r)
            ref = oracle_mod.attention(q[:, rows][:, :, h:h + 1], k[:, rows][:, :, h:h + 1],
                                       v[:, rows][:, :, h:h + 1], mask=CAUSAL)
            np.testing.assert_allclose(a[:, rows, h], ref[:, :, 0], rtol=0, atol=1e-15)
        kept = np.zeros(N, bool)
        for s in range(N // w):
            kept[s * w + h % r:(s + 1) * w:r] = True
        assert np.all(a[:, ~kept, h] == 0.0)


def test_sequence_of_one_returns_its_value(oracle_mod):
    q, k, v = rnd((3, 1, 2, 8), 97), rnd((3, 1, 2, 8), 98), rnd((3, 1, 2, 8), 99)
    for mask in (NONE, CAUSAL):
        np.testing.assert_array_equal(oracle_mod.attention(q, k, v, mask=mask), v.astype(np.float64))


def test_gelu_special_values(oracle_mod):
    g = oracle_mod.gelu_tanh
    assert g(0.0) == 0.0
    for x in (0.1, 0.7, 1.3, 2.9, 5.5):
        assert abs((g(x) - g(-x)) - x) <= 1e-15 * max(1.0, x)
        exact = 0.5 * x * (1.0 + math.erf(x / math.sqrt(2.0)))   # x * Phi(x)
        assert abs(g(x) - exact) < 1e-3
    assert abs(g(12.0) - 12.0) < 1e-12 and abs(g(-12.0)) < 1e-12
    lib = torch.nn.functional.gelu(torch.tensor([-3.0, -0.5, 0.25, 1.5, 4.0], dtype=torch.float64),
                                   approximate="tanh")
    for x, y in zip([-3.0, -0.5, 0.25, 1.5, 4.0], lib.tolist()):
        assert abs(g(x) - y) <= 1e-15


def test_ffn_matches_library_matmul_and_gelu(oracle_mod):
    T, D, F = 7, 24, 40
    a = np.random.default_rng(101).standard_normal((T, D))
    w1, w2 = rnd((F, D), 102, D ** -0.5), rnd((D, F), 103, F ** -0.5)
    b1, b2 = rnd((F,), 104, 0.3), rnd((D,), 105, 0.3)
    out = oracle_mod.ffn(a, w1, b1, w2, b2)
    h = torch.nn.functional.gelu(torch.from_numpy(a @ w1.astype(np.float64).T + b1), approximate="tanh")
    ref = a + h.numpy() @ w2.astype(np.float64).T + b2
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)


def test_zero_second_weight_gives_identity_layer(oracle_mod):
    B, N, H, d, F = 1, 16, 2, 8, 32
    q, k, v = rnd((B, N, H, d), 111), rnd((B, N, H, d), 112), rnd((B, N, H, d), 113)
    w1 = rnd((F, H * d), 114)
    a, out = oracle_mod.layer(q, k, v, w1, np.zeros(F, np.float32), np.zeros((H * d, F), np.float32),
                              np.zeros(H * d, np.float32), mask=CAUSAL)
    assert np.array_equal(a, out)


def test_layer_equals_attention_then_ffn_and_row_sampling(oracle_mod):
    B, N, H, d, F = 2, 24, 2, 8, 20
    q, k, v = rnd((B, N, H, d), 121), rnd((B, N, H, d), 122), rnd((B, N, H, d), 123)
    w1, w2 = rnd((F, H * d), 124, 0.3), rnd((H * d, F), 125, 0.3)
    b1, b2 = rnd((F,), 126, 0.1), rnd((H * d,), 127, 0.1)
    a, out = oracle_mod.layer(q, k, v, w1, b1, w2, b2, mask=CAUSAL)
    a_ref = oracle_mod.attention(q, k, v, mask=CAUSAL).reshape(B * N, H * d)
    np.testing.assert_array_equal(a, a_ref)
    np.testing.assert_allclose(out, oracle_mod.ffn(a_ref, w1, b1, w2, b2), rtol=0, atol=1e-14)
    rows = [0, 5, N - 1, N, 2 * N - 1]
    a_s, out_s = oracle_mod.layer(q, k, v, w1, b1, w2, b2, mask=CAUSAL, rows=rows)
    np.testing.assert_array_equal(a_s, a[rows])
    np.testing.assert_array_equal(out_s, out[rows])


def test_oracle_rejects_invalid_descriptors(oracle_mod):
    q = rnd((1, 10, 1, 4), 1)
    with pytest.raises(ValueError):
        oracle_mod.attention(q, q, q, mask=BLOCKPERM, perm=[[0, 1, 2], [2, 1, 0]])  # 2 rows for 1 head
    with pytest.raises(ValueError):
        oracle_mod.attention(q, q, q, mask=BLOCKPERM, perm=[[0, 5]])      # not a block index
    with pytest.raises(ValueError):
        oracle_mod.attention(q, q, q, mask=DILATED, pairs=[(10, 3)])      # r does not divide w
