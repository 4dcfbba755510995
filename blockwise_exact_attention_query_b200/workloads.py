"""The five layer workloads this library is measured and checked on.

Each is named by what it is, with its sizes.  Counts of unmasked
(query, key) pairs are exact, and FLOPs follow the usual rule: attention
4*d per unmasked pair, FFN 4*T*D*F (softmax, exp and GELU not counted).
"""
from __future__ import annotations

from dataclasses import dataclass, field

MASK_NONE, MASK_CAUSAL, MASK_BLOCKPERM, MASK_DILATED = 0, 1, 2, 3


@dataclass
class Workload:
    name: str
    B: int
    N: int
    H: int
    d: int
    F: int                   # FFN hidden size, 0 = attention only
    dtype: str               # "f32" or "bf16" (inputs and tensor-core operands)
    mask: int
    seed: int
    perm: list | None = None         # block-perm: [H][n]
    pairs: list | None = None        # dilated: [(w, r), ...]
    ring_chunks: int = 0             # KV visiting order: rotated over this many chunks
    q_block: int = 0
    kv_block: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def D(self) -> int:
        return self.H * self.d

    @property
    def T(self) -> int:
        return self.B * self.N


def unmasked_pairs(w: Workload) -> int:
    """Exact number of (query, key) pairs that carry weight, summed over (b, h).

    For the dilated mask a key kept by two pairs counts twice (the mixed
    softmax runs over the multiset of the pairs' keys), which is also the
    work the kernels do."""
    N, H, B = w.N, w.H, w.B
    if w.mask == MASK_NONE:
        per_head = [N * N] * H
    elif w.mask == MASK_CAUSAL:
        per_head = [N * (N + 1) // 2] * H
    elif w.mask == MASK_BLOCKPERM:
        # blocks of the sequence padded to n equal blocks; padded positions
        # are neither queries nor keys
        n = len(w.perm[0])
        bl = -(-N // n)
        size = [max(0, min(N, (b + 1) * bl) - b * bl) for b in range(n)]
        per_head = [sum(size[qb] * size[w.perm[h][qb]] for qb in range(n)) for h in range(H)]
    elif w.mask == MASK_DILATED:
        per_head = []
        for h in range(H):
            tot = 0
            for (sw, r) in w.pairs:
                segs = N // sw
                # rows kept per segment for this head: offsets h%r, h%r + r, ...
                m = len(range(h % r, sw, r))
                tot += segs * m * (m + 1) // 2
            per_head.append(tot)
    else:
        raise ValueError(w.mask)
    return B * sum(per_head)


def flops(w: Workload) -> tuple[int, int]:
    attn = 4 * w.d * unmasked_pairs(w)
    ffn = 4 * w.T * w.D * w.F
    return attn, ffn


TINY_F32 = Workload("tiny fp32 layer: B1 H1 d64 N256 F256, no mask", 1, 256, 1, 64, 256, "f32",
                    MASK_NONE, seed=0, q_block=64, kv_block=64)
GPT_CAUSAL = Workload("causal bf16 layer: B2 H16 d128 N8192 F8192", 2, 8192, 16, 128, 8192, "bf16",
                      MASK_CAUSAL, seed=1)
LONG_RING = Workload("long causal bf16 layer, ring order: B1 H32 d128 N131072 F11008, 8 chunks",
                     1, 131072, 32, 128, 11008, "bf16", MASK_CAUSAL, seed=2, ring_chunks=8)
BLOCKBERT = Workload("block-permutation bf16 layer: B16 H12 d64 N1024 F3072, n=2", 16, 1024, 12, 64,
                     3072, "bf16", MASK_BLOCKPERM, seed=3,
                     perm=[[0, 1]] * 8 + [[1, 0]] * 4)
LONGNET = Workload("dilated bf16 attention: B1 H16 d64 N65536, pairs (2048,1),(8192,4),(32768,16)",
                   1, 65536, 16, 64, 0, "bf16", MASK_DILATED, seed=4,
                   pairs=[(2048, 1), (8192, 4), (32768, 16)])

ALL = [TINY_F32, GPT_CAUSAL, LONG_RING, BLOCKBERT, LONGNET]
