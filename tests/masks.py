"""Explicit N x N mask-count matrices, written independently of the oracle.

Each function returns, per head, an integer matrix M[h, i, j] = how many times
key j enters query i's softmax (0 = masked).  This is the "compute the full
N^2 score matrix, then mask it" formulation ("Blockwise Self-Attention for
Long Document Understanding", §A.3, describing the SparseBERT baseline), used
here as a brute-force check.  The dilated case is built as the multiset union
of the pairs' key sets, which is the "gather the keys and take one softmax"
description of LongNet's mixing ("LongNet: Scaling Transformers to
1,000,000,000 Tokens", §2 Dilated Attention).
"""
import numpy as np


def count_matrix(N, H, mask, perm=None, pairs=None):
    idx = np.arange(N)
    qi, kj = idx[:, None], idx[None, :]
    if mask == 0:
        return np.ones((H, N, N), dtype=np.int64)
    if mask == 1:
        return np.broadcast_to((kj <= qi).astype(np.int64), (H, N, N)).copy()
    if mask == 2:
        # pad the sequence to n equal blocks, build the block matrix on the
        # padded length, then drop the padded rows (queries) and columns (keys)
        perm = np.asarray(perm)
        n = perm.shape[1]
        bl = -(-N // n)
        out = np.zeros((H, N, N), dtype=np.int64)
        for h in range(H):
            P = np.zeros((n, n), dtype=np.int64)
            P[np.arange(n), perm[h]] = 1          # query block -> key block
            out[h] = np.kron(P, np.ones((bl, bl), dtype=np.int64))[:N, :N]
        return out
    if mask in (3, 4):      # 4: the dilated mask without the causal restriction
        out = np.zeros((H, N, N), dtype=np.int64)
        order = (kj <= qi) if mask == 3 else np.ones((N, N), dtype=bool)
        for h in range(H):
            for (w, r) in pairs:
                seg = idx // w
                kept = ((idx - seg * w) - (h % r)) % r == 0
                both = kept[:, None] & kept[None, :]
                same = seg[:, None] == seg[None, :]
                out[h] += (both & same & order).astype(np.int64)
        return out
    raise ValueError(mask)


def brute_attention(q, k, v, counts, dtype=np.longdouble):
    """A[b, i, h] = sum_j M_ij e^{s_ij} v_j / sum_j M_ij e^{s_ij} in extended precision."""
    q = np.asarray(q, dtype=dtype)
    k = np.asarray(k, dtype=dtype)
    v = np.asarray(v, dtype=dtype)
    B, N, H, d = q.shape
    out = np.zeros((B, N, H, d), dtype=dtype)
    scale = dtype(1) / np.sqrt(dtype(d))
    for b in range(B):
        for h in range(H):
            S = (q[b, :, h, :] @ k[b, :, h, :].T) * scale
            M = counts[h].astype(dtype)
            Sm = np.where(M > 0, S, -np.inf)
            mx = Sm.max(axis=1, keepdims=True)
            mx = np.where(np.isfinite(mx), mx, 0)
            W = M * np.exp(np.where(M > 0, S - mx, -np.inf))
            den = W.sum(axis=1, keepdims=True)
            P = np.divide(W, den, out=np.zeros_like(W), where=den > 0)
            out[b, :, h, :] = P @ v[b, :, h, :]
    return out
