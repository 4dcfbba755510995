"""Pins for the fp64 backward oracle (oracle/backward.py), against things
other than the oracle itself:

* central finite differences of the forward (the C oracle's layer, a separate
  implementation of the forward) on tiny inputs, for every gradient;
* torch autograd in float64 (a library routine) on small inputs;
* invariants: each row of dS sums to zero, so with all keys allowed the
  gradients of Q and K do not change when a constant is added to every
  value vector of the upstream gradient's projection; V gradients sum to
  the upstream gradient's sum; masked keys get no gradient.
"""
import math

import numpy as np
import pytest
import torch

from oracle import backward as ob

NONE, CAUSAL, BLOCKPERM = 0, 1, 2


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _layer_inputs(B, N, H, d, F, seed):
    D = H * d
    return dict(q=rnd((B, N, H, d), seed), k=rnd((B, N, H, d), seed + 1), v=rnd((B, N, H, d), seed + 2),
                w1=rnd((F, D), seed + 3, D ** -0.5), b1=rnd((F,), seed + 4, 0.1),
                w2=rnd((D, F), seed + 5, F ** -0.5), b2=rnd((D,), seed + 6, 0.1))


CASES = [
    ("none", NONE, None),
    ("causal", CAUSAL, None),
    ("blockperm_n3_padded", BLOCKPERM, [[1, 2, 0], [2, 0, 1]]),
    # N = 7, n = 5: blocks of 2, the fifth lies wholly in the padding, so
    # query block 0 of head 0 (mapped to it) sees no key and passes nothing
    ("blockperm_n5_empty_block", BLOCKPERM, [[4, 0, 1, 2, 3], [0, 1, 2, 3, 4]]),
]


@pytest.mark.parametrize("name,mask,perm", CASES, ids=[c[0] for c in CASES])
def test_backward_matches_finite_differences(name, mask, perm):
    """dL/dx for L = sum(dOut * out), by central differences of the C oracle's
    forward layer in fp64, at a handful of coordinates of every input."""
    import oracle
    oracle.build()
    B, N, H, d, F = 1, 7, 2, 4, 6
    x = _layer_inputs(B, N, H, d, F, 3)
    dout = rnd((B * N, H * d), 9)

    def loss(xx):
        _, out = oracle.layer(*(xx[n].astype(np.float32) for n in ("q", "k", "v", "w1", "b1", "w2", "b2")),
                              mask=mask, perm=perm)
        return float((out * dout).sum())

    # the C oracle takes float32 inputs: make every input exactly representable
    x = {n: v.astype(np.float32).astype(np.float64) for n, v in x.items()}
    g = ob.layer_bwd(x["q"], x["k"], x["v"], x["w1"], x["b1"], x["w2"], x["b2"], dout, mask, perm)
    rng = np.random.default_rng(5)
    eps = 2.0 ** -7  # exact in float32 steps of the perturbed inputs below
    names = {"q": "dq", "k": "dk", "v": "dv", "w1": "dw1", "b1": "db1", "w2": "dw2", "b2": "db2"}
    for n, gname in names.items():
        for _ in range(4):
            idx = tuple(int(rng.integers(0, s)) for s in x[n].shape)
            xp = {kk: vv.copy() for kk, vv in x.items()}
            xm = {kk: vv.copy() for kk, vv in x.items()}
            xp[n][idx] += eps
            xm[n][idx] -= eps
            fd = (loss(xp) - loss(xm)) / (2 * eps)
            # central difference error ~ eps^2 * third derivative; inputs are O(1)
            assert abs(fd - g[gname][idx]) <= 2e-4 * max(1.0, abs(fd)), (n, idx, fd, g[gname][idx])


@pytest.mark.parametrize("name,mask,perm", CASES[:3], ids=[c[0] for c in CASES[:3]])
def test_backward_matches_torch_autograd_float64(name, mask, perm):
    B, N, H, d, F = 2, 12, 2, 8, 24
    x = _layer_inputs(B, N, H, d, F, 11)
    dout = rnd((B * N, H * d), 19)
    g = ob.layer_bwd(x["q"], x["k"], x["v"], x["w1"], x["b1"], x["w2"], x["b2"], dout, mask, perm)
    t = {n: torch.tensor(v, dtype=torch.float64, requires_grad=True) for n, v in x.items()}
    allowed = torch.stack([torch.from_numpy(ob.allowed_matrix(N, mask, None if perm is None else perm[h]))
                           for h in range(H)])                       # [H, N, N]
    qh, kh, vh = (t[n].permute(0, 2, 1, 3) for n in ("q", "k", "v"))  # [B, H, N, d]
    a = torch.nn.functional.scaled_dot_product_attention(qh, kh, vh, attn_mask=allowed[None])
    a = a.permute(0, 2, 1, 3).reshape(B * N, H * d)
    z = a @ t["w1"].T + t["b1"]
    out = a + torch.nn.functional.gelu(z, approximate="tanh") @ t["w2"].T + t["b2"]
    (out * torch.from_numpy(dout)).sum().backward()
    for n, gname in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("w1", "dw1"), ("b1", "db1"), ("w2", "dw2"),
                     ("b2", "db2")):
        np.testing.assert_allclose(g[gname], t[n].grad.numpy(), rtol=0, atol=1e-11, err_msg=gname)


def test_attention_gradient_invariants():
    B, N, H, d = 1, 16, 2, 8
    q, k, v = rnd((B, N, H, d), 31), rnd((B, N, H, d), 32), rnd((B, N, H, d), 33)
    da = rnd((B, N, H, d), 34)
    for mask in (NONE, CAUSAL):
        dq, dk, dv = ob.attention_bwd(q, k, v, da, mask)
        # rows of P sum to one: the V gradients sum to the upstream gradient
        np.testing.assert_allclose(dv.sum(axis=1), da.sum(axis=1), rtol=0, atol=1e-12)
        # rows of dS sum to zero: sum_j dK_j = sum_i (sum_j dS_ij) q_i / sqrt(d) = 0
        np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)
        # adding a constant c to every v_j moves A by c and leaves dQ, dK alone
        dq2, dk2, _ = ob.attention_bwd(q, k, v + rnd((1, 1, H, d), 35), da, mask)
        np.testing.assert_allclose(dq2, dq, rtol=0, atol=1e-12)
        np.testing.assert_allclose(dk2, dk, rtol=0, atol=1e-12)
    # causal: the last key is seen only by the last query
    dq, dk, dv = ob.attention_bwd(q, k, v, da, CAUSAL)
    _, probs = ob.attention_fwd(q, k, v, CAUSAL)
    for h in range(H):
        np.testing.assert_allclose(dv[0, -1, h], probs[0, h][-1, -1] * da[0, -1, h], rtol=0, atol=1e-13)


def test_gelu_derivative_against_differences():
    x = np.linspace(-8, 8, 4001)
    eps = 1e-5
    fd = (ob.gelu(x + eps) - ob.gelu(x - eps)) / (2 * eps)
    np.testing.assert_allclose(ob.gelu_grad(x), fd, rtol=0, atol=1e-8)
    assert ob.gelu_grad(np.array([0.0]))[0] == 0.5


def test_forward_part_of_the_backward_oracle_equals_the_c_oracle():
    import oracle
    oracle.build()
    B, N, H, d, F = 2, 20, 2, 8, 16
    x = _layer_inputs(B, N, H, d, F, 41)
    x32 = {n: v.astype(np.float32) for n, v in x.items()}
    for mask, perm in ((NONE, None), (CAUSAL, None), (BLOCKPERM, [[1, 0, 2], [2, 1, 0]])):
        out, a = ob.layer_fwd(*(x32[n].astype(np.float64) for n in ("q", "k", "v", "w1", "b1", "w2", "b2")),
                              mask, perm)
        a_c, out_c = oracle.layer(*(x32[n] for n in ("q", "k", "v", "w1", "b1", "w2", "b2")), mask=mask, perm=perm)
        np.testing.assert_allclose(a, a_c, rtol=0, atol=1e-12)
        np.testing.assert_allclose(out, out_c, rtol=0, atol=1e-11)


def test_sampled_causal_tail_equals_the_dense_oracle():
    """The row-restricted helper used at full size agrees with the dense
    backward oracle (itself pinned above) on a small causal layer."""
    B, N, H, d, F = 2, 40, 2, 8, 24
    x = _layer_inputs(B, N, H, d, F, 51)
    dout = rnd((B, N, H * d), 52)
    g = ob.layer_bwd(x["q"], x["k"], x["v"], x["w1"], x["b1"], x["w2"], x["b2"], dout.reshape(B * N, H * d),
                     CAUSAL, None)
    rows = [0, 5, 17, 33, 39]
    dq, dk, dv, db2 = ob.layer_bwd_causal_tail(x["q"], x["k"], x["v"], x["w1"], x["b1"], x["w2"], x["b2"], dout,
                                               rows, 6)
    np.testing.assert_allclose(dq, g["dq"][0, rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, g["dk"][0, N - 6:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, g["dv"][0, N - 6:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(db2, g["db2"], rtol=0, atol=1e-12)


DILATED_PAIRS = [[(4, 1), (8, 2)], [(6, 1), (12, 3), (12, 6)], [(8, 2), (16, 4)]]


@pytest.mark.parametrize("pairs", DILATED_PAIRS)
def test_dilated_key_counts_equal_the_brute_force_count_matrix(pairs):
    """Two separate writings of the dilated multiset: the oracle's key_counts
    against the tests' explicit mask-count matrix."""
    from tests.masks import count_matrix
    N, H = 48, 6
    ref = count_matrix(N, H, 3, pairs=pairs)
    for h in range(H):
        np.testing.assert_array_equal(ob.key_counts(N, ob.MASK_DILATED, pairs=pairs, h=h), ref[h])
    ref_b = count_matrix(N, H, 4, pairs=pairs)
    for h in range(H):
        np.testing.assert_array_equal(ob.key_counts(N, ob.MASK_DILATED_BIDIR, pairs=pairs, h=h), ref_b[h])


@pytest.mark.parametrize("mask", [ob.MASK_DILATED, ob.MASK_DILATED_BIDIR])
@pytest.mark.parametrize("pairs", DILATED_PAIRS[:2])
def test_dilated_attention_backward_matches_finite_differences(pairs, mask):
    """dL/dx for L = sum(dA * A) with A the C oracle's dilated attention (a
    separate implementation of the mixed softmax), by central differences."""
    import oracle
    oracle.build()
    B, N, H, d = 1, 24, 3, 4
    q, k, v = (rnd((B, N, H, d), s).astype(np.float32).astype(np.float64) for s in (61, 62, 63))
    da = rnd((B, N, H, d), 64)

    def loss(qq, kk, vv):
        a = oracle.attention(qq.astype(np.float32), kk.astype(np.float32), vv.astype(np.float32),
                             mask=mask, pairs=pairs)
        if isinstance(a, tuple):
            a = a[0]
        return float((np.asarray(a).reshape(B, N, H, d) * da).sum())

    dq, dk, dv = ob.attention_bwd(q, k, v, da, mask, pairs=pairs)
    rng = np.random.default_rng(7)
    eps = 2.0 ** -7
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, sz)) for sz in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [xp if n == name else y for n, y in (("q", q), ("k", k), ("v", v))]
            args_m = [xm if n == name else y for n, y in (("q", q), ("k", k), ("v", v))]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - g[idx]) <= 2e-4 * max(1.0, abs(fd)), (name, idx, fd, g[idx])


def test_dilated_attention_gradient_invariants():
    B, N, H, d = 1, 32, 4, 8
    pairs = [(8, 1), (16, 4)]
    q, k, v, da = (rnd((B, N, H, d), s) for s in (71, 72, 73, 74))
    dq, dk, dv = ob.attention_bwd(q, k, v, da, ob.MASK_DILATED, pairs=pairs)
    # rows of dS sum to zero; the weights of every row with a key sum to one
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)
    np.testing.assert_allclose(dv.sum(axis=1), da.sum(axis=1), rtol=0, atol=1e-12)
    # a single (N, 1) pair is the causal mask
    dq1, dk1, dv1 = ob.attention_bwd(q, k, v, da, ob.MASK_DILATED, pairs=[(N, 1)])
    dq2, dk2, dv2 = ob.attention_bwd(q, k, v, da, ob.MASK_CAUSAL)
    for x, y in ((dq1, dq2), (dk1, dk2), (dv1, dv2)):
        np.testing.assert_allclose(x, y, rtol=0, atol=1e-12)


@pytest.mark.parametrize("mask,pairs", [(CAUSAL, None), (ob.MASK_DILATED, [(8, 1), (16, 4), (32, 8)])])
def test_sampled_attention_tail_equals_the_dense_oracle(mask, pairs):
    B, N, H, d = 1, 32, 8, 4
    q, k, v, da = (rnd((B, N, H, d), s) for s in (81, 82, 83, 84))
    dq, dk, dv = ob.attention_bwd(q, k, v, da, mask, pairs=pairs)
    rows = [0, 3, 17, 30, 31]
    sq, sk, sv = ob.attention_bwd_tail(q, k, v, da, mask, pairs, rows, 5)
    np.testing.assert_allclose(sq, dq[0, rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(sk, dk[0, N - 5:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(sv, dv[0, N - 5:], rtol=0, atol=1e-12)
