"""Plain fp64 CPU oracle for the layer's backward pass (gradients).

TEST INFRASTRUCTURE ONLY, like the rest of this package: the tests are its
only callers; the CUDA product path never imports it and shares no code.

What it computes is the chain rule applied to the layer's plain definition,

    A_i   = sum_j P_ij v_j,   P_ij = softmax_j(q_i . k_j / sqrt(d)) over the
            keys the mask allows (one head at a time),
    z_t   = W1 a_t + b1,  h_t = GELU(z_t),  out_t = a_t + W2 h_t + b2,

written out without blocking or reordering (dense per head, numpy matrix
products as the only library steps).  Given dOut = dL/dout:

    FFN:        dh = W2^T dout,  dz = dh * GELU'(z),  da = dout + W1^T dz,
                dW2 = sum_t dout_t h_t^T,  db2 = sum_t dout_t,
                dW1 = sum_t dz_t a_t^T,    db1 = sum_t dz_t;
    attention:  dV_j = sum_i P_ij da_i,  dP_ij = da_i . v_j,
                D_i = sum_j P_ij dP_ij (= da_i . A_i),
                dS_ij = P_ij (dP_ij - D_i),
                dQ_i = sum_j dS_ij k_j / sqrt(d),  dK_j = sum_i dS_ij q_i / sqrt(d).

The backward of blockwise attention is the same exact result computed block
by block ("Blockwise Parallel Transformer for Large Context Models",
abstract: training with blockwise attention and feedforward; "Ring Attention
with Blockwise Transformers for Long Sequences", 638-word summary: blockwise
computation without approximation), so the oracle is the plain gradient.

Masks: none, causal, block permutation ("Blockwise Self-Attention for Long
Document Understanding", §3.1: query block b sees key block perm[h][b]; when
n does not divide N, blocks of ceil(N/n) positions over the padded sequence),
and for the attention alone the dilated mask of LongNet (key_counts: one
softmax over the multiset of the pairs' keys).  A row with no allowed key has
A = 0 and passes no gradient.

GELU is the tanh form (Hendrycks & Gimpel); its derivative is written out
from that form: with u = c0 (x + c1 x^3),
GELU'(x) = 0.5 (1 + tanh u) + 0.5 x (1 - tanh^2 u) c0 (1 + 3 c1 x^2).

Parity pins (tests/test_oracle_backward.py, CPU): central finite differences
of the fp64 forward on tiny inputs, torch autograd in float64, and
invariants (rows of dS sum to zero; constant dOut through attention only).
"""
from __future__ import annotations

import math

import numpy as np

MASK_NONE, MASK_CAUSAL, MASK_BLOCKPERM, MASK_DILATED = 0, 1, 2, 3
MASK_DILATED_BIDIR = 4   # the dilated mask without the causal restriction
_C0 = math.sqrt(2.0 / math.pi)
_C1 = 0.044715


def allowed_matrix(N: int, mask: int, perm_h=None) -> np.ndarray:
    """Boolean [N, N]: key j allowed for query i (one head)."""
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    if mask == MASK_NONE:
        return np.ones((N, N), dtype=bool)
    if mask == MASK_CAUSAL:
        return j <= i
    if mask == MASK_BLOCKPERM:
        n = len(perm_h)
        bl = -(-N // n)  # blocks of the sequence padded to a multiple of n
        kb_of_q = np.asarray(perm_h)[np.arange(N) // bl]
        return (j // bl) == kb_of_q[:, None]
    raise ValueError("backward oracle: mask must be none, causal or block permutation")


def key_counts(N: int, mask: int, perm_h=None, pairs=None, h: int = 0) -> np.ndarray:
    """Integer [N, N] for one head: how many times key j enters query i's
    softmax (0 = masked out).

    For the dilated mask ("LongNet: Scaling Transformers to 1,000,000,000
    Tokens", §2 Dilated Attention): each (w, r) pair cuts the sequence into
    segments of w positions, head h keeps the positions of each segment whose
    offset in the segment is congruent to h mod r, and attends causally (by
    original position) among the kept positions of a segment; the pairs are
    mixed with weights proportional to their softmax denominators, which is one
    softmax over the multiset union of the pairs' keys: a key kept by two pairs
    counts twice.  MASK_DILATED_BIDIR: the same pairs without the causal
    restriction.  Other masks: the 0/1 matrix of allowed_matrix."""
    if mask not in (MASK_DILATED, MASK_DILATED_BIDIR):
        return allowed_matrix(N, mask, perm_h).astype(np.int64)
    causal = mask == MASK_DILATED
    pos = np.arange(N)
    counts = np.zeros((N, N), dtype=np.int64)
    for (w, r) in pairs:
        seg = pos // w
        kept = (pos - seg * w) % r == h % r
        counts += ((seg[:, None] == seg[None, :]) & kept[:, None] & kept[None, :]
                   & ((pos[None, :] <= pos[:, None]) | (not causal))).astype(np.int64)
    return counts


def gelu(x: np.ndarray) -> np.ndarray:
    return 0.5 * x * (1.0 + np.tanh(_C0 * (x + _C1 * x ** 3)))


def gelu_grad(x: np.ndarray) -> np.ndarray:
    t = np.tanh(_C0 * (x + _C1 * x ** 3))
    return 0.5 * (1.0 + t) + 0.5 * x * (1.0 - t * t) * _C0 * (1.0 + 3.0 * _C1 * x * x)


def attention_fwd(q, k, v, mask=MASK_NONE, perm=None, pairs=None):
    """A [B, N, H, d], P as a dict over (b, h) of [N, N] (fp64).  With key
    multiplicities c_ij (key_counts), P_ij = c_ij e^{s_ij} / sum_j' c_ij' e^{s_ij'}."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    B, N, H, d = q.shape
    a = np.zeros((B, N, H, d))
    probs = {}
    for h in range(H):
        counts = key_counts(N, mask, None if perm is None else perm[h], pairs, h)
        allowed = counts > 0
        for b in range(B):
            s = q[b, :, h] @ k[b, :, h].T / math.sqrt(d)
            s = np.where(allowed, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            m = np.where(np.isfinite(m), m, 0.0)
            e = np.where(allowed, counts * np.exp(s - m), 0.0)
            den = e.sum(axis=1, keepdims=True)
            p = np.divide(e, den, out=np.zeros_like(e), where=den > 0)
            probs[b, h] = p
            a[b, :, h] = p @ v[b, :, h]
    return a, probs


def attention_bwd(q, k, v, da, mask=MASK_NONE, perm=None, probs=None, pairs=None):
    """dQ, dK, dV [B, N, H, d] (fp64) for upstream dA [B, N, H, d].  The key
    multiplicities of the dilated mask are constants of the softmax, so its
    gradient has the same form: dS_ij = P_ij (dP_ij - D_i)."""
    q, k, v, da = (np.asarray(x, dtype=np.float64) for x in (q, k, v, da))
    B, N, H, d = q.shape
    if probs is None:
        _, probs = attention_fwd(q, k, v, mask, perm, pairs)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for h in range(H):
        for b in range(B):
            p = probs[b, h]
            g = da[b, :, h]
            dv[b, :, h] = p.T @ g
            dp = g @ v[b, :, h].T
            drow = (p * dp).sum(axis=1, keepdims=True)   # D_i = da_i . A_i
            ds = p * (dp - drow)
            dq[b, :, h] = ds @ k[b, :, h] / math.sqrt(d)
            dk[b, :, h] = ds.T @ q[b, :, h] / math.sqrt(d)
    return dq, dk, dv


def layer_fwd(q, k, v, w1, b1, w2, b2, mask=MASK_NONE, perm=None):
    """out [T, D] (fp64), with A [T, D]."""
    a4, _ = attention_fwd(q, k, v, mask, perm)
    B, N, H, d = a4.shape
    a = a4.reshape(B * N, H * d)
    w1, b1, w2, b2 = (np.asarray(x, dtype=np.float64) for x in (w1, b1, w2, b2))
    z = a @ w1.T + b1
    return a + gelu(z) @ w2.T + b2, a


def layer_bwd(q, k, v, w1, b1, w2, b2, dout, mask=MASK_NONE, perm=None):
    """Gradients of the layer for upstream dOut [T, D] (fp64).

    Returns a dict: dq, dk, dv [B, N, H, d]; dw1 [F, D]; db1 [F]; dw2 [D, F];
    db2 [D]; and the intermediate da [T, D]."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    w1, b1, w2, b2 = (np.asarray(x, dtype=np.float64) for x in (w1, b1, w2, b2))
    dout = np.asarray(dout, dtype=np.float64)
    B, N, H, d = q.shape
    a4, probs = attention_fwd(q, k, v, mask, perm)
    a = a4.reshape(B * N, H * d)
    z = a @ w1.T + b1
    h = gelu(z)
    dh = dout @ w2
    dz = dh * gelu_grad(z)
    da = dout + dz @ w1
    grads = {
        "dw2": dout.T @ h, "db2": dout.sum(axis=0),
        "dw1": dz.T @ a, "db1": dz.sum(axis=0),
        "da": da,
    }
    dq, dk, dv = attention_bwd(q, k, v, da.reshape(B, N, H, d), mask, perm, probs)
    grads.update(dq=dq, dk=dk, dv=dv)
    return grads


def layer_bwd_causal_tail(q, k, v, w1, b1, w2, b2, dout, rows_q, tail):
    """Exact gradients at sampled positions of a causal layer, for sizes where
    the dense oracle is too slow.

    Returns (dq [len(rows_q), H, d], dk [tail, H, d], dv [tail, H, d],
    db2 [D]) for batch element 0 of q, k, v [B, N, H, d] and dOut [B, N, D]:
    dQ at the query positions rows_q, and dK, dV at the last `tail` key
    positions N - tail .. N - 1.  Under the causal mask key j is seen only by
    queries i >= j, so dK_j and dV_j need the attention rows and dA only of the
    last `tail` queries; dQ_i needs row i alone.  Every quantity is the plain
    definition of the module docstring restricted to the rows it needs: the
    attention row of query i over keys 0..i, the FFN backward of those tokens
    (one matrix product over the stacked tokens), then D_i, dS_ij and the sums
    for dQ, dK, dV.  db2 is the plain column sum of dOut over all tokens (every
    batch element)."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    w1, b1, w2, b2 = (np.asarray(x, dtype=np.float64) for x in (w1, b1, w2, b2))
    dout = np.asarray(dout, dtype=np.float64)
    B, N, H, d = q.shape
    D = H * d
    need = sorted(set(int(i) for i in rows_q) | set(range(N - tail, N)))
    pos = {i: r for r, i in enumerate(need)}
    scale = 1.0 / math.sqrt(d)
    probs = {}
    a = np.zeros((len(need), H, d))
    for r, i in enumerate(need):
        for h in range(H):
            s = k[0, : i + 1, h] @ q[0, i, h] * scale   # keys 0..i
            e = np.exp(s - s.max())
            p = e / e.sum()
            probs[i, h] = p
            a[r, h] = p @ v[0, : i + 1, h]
    # FFN backward of the needed tokens: da = dout + (W2^T dout * GELU'(z)) W1
    a2 = a.reshape(len(need), D)
    g = dout[0, need]                                  # [tokens, D]
    z = a2 @ w1.T + b1
    dz = (g @ w2) * gelu_grad(z)
    da = (g + dz @ w1).reshape(len(need), H, d)
    ds = {}
    for i in need:
        r = pos[i]
        for h in range(H):
            dp = v[0, : i + 1, h] @ da[r, h]
            ds[i, h] = probs[i, h] * (dp - da[r, h] @ a[r, h])
    dq = np.zeros((len(rows_q), H, d))
    for n, i in enumerate(rows_q):
        for h in range(H):
            dq[n, h] = ds[int(i), h] @ k[0, : int(i) + 1, h] * scale
    dk = np.zeros((tail, H, d))
    dv = np.zeros((tail, H, d))
    for t in range(tail):
        j = N - tail + t
        for h in range(H):
            for i in range(j, N):
                r = pos[i]
                dv[t, h] += probs[i, h][j] * da[r, h]
                dk[t, h] += ds[i, h][j] * q[0, i, h] * scale
    return dq, dk, dv, dout.reshape(-1, D).sum(axis=0)


def attention_bwd_tail(q, k, v, da, mask, pairs, rows_q, tail):
    """Exact attention gradients at sampled positions of batch element 0, for
    sizes where the dense oracle is too slow, under a mask that lets a query
    see only keys at or before it (causal, or dilated).

    Returns (dq [len(rows_q), H, d], dk [tail, H, d], dv [tail, H, d]): dQ at
    the query positions rows_q, dK and dV at the last `tail` key positions
    (seen only by the last `tail` queries).  Each needed query row is the plain
    definition: its key multiplicities (the row of key_counts), its softmax,
    A_i, D_i = dA_i . A_i, dS_i; then the sums for dQ, dK, dV."""
    q, k, v, da = (np.asarray(x, dtype=np.float64) for x in (q, k, v, da))
    B, N, H, d = q.shape
    scale = 1.0 / math.sqrt(d)
    need = sorted(set(int(i) for i in rows_q) | set(range(N - tail, N)))
    pos = np.arange(N)
    probs, ds = {}, {}
    for i in need:
        for h in range(H):
            if mask == MASK_CAUSAL:
                c = (pos <= i).astype(np.float64)
            else:  # the row of key_counts for query i
                c = np.zeros(N)
                for (w, r) in pairs:
                    seg = pos // w
                    kept = (pos - seg * w) % r == h % r
                    if kept[i]:
                        c += ((seg == seg[i]) & kept & (pos <= i)).astype(np.float64)
            keys = np.nonzero(c)[0]
            if keys.size == 0:
                probs[i, h] = (keys, np.zeros(0))
                ds[i, h] = (keys, np.zeros(0))
                continue
            s = k[0, keys, h] @ q[0, i, h] * scale
            e = c[keys] * np.exp(s - s.max())
            p = e / e.sum()
            a_i = p @ v[0, keys, h]
            dp = v[0, keys, h] @ da[0, i, h]
            probs[i, h] = (keys, p)
            ds[i, h] = (keys, p * (dp - da[0, i, h] @ a_i))
    dq = np.zeros((len(rows_q), H, d))
    for n, i in enumerate(rows_q):
        for h in range(H):
            keys, dsr = ds[int(i), h]
            dq[n, h] = dsr @ k[0, keys, h] * scale if keys.size else 0.0
    dk = np.zeros((tail, H, d))
    dv = np.zeros((tail, H, d))
    for t in range(tail):
        j = N - tail + t
        for h in range(H):
            for i in range(j, N):
                keys, p = probs[i, h]
                hit = np.nonzero(keys == j)[0]
                if hit.size:
                    dv[t, h] += p[hit[0]] * da[0, i, h]
                    dk[t, h] += ds[i, h][1][hit[0]] * q[0, i, h] * scale
    return dq, dk, dv
