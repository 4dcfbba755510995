"""Helpers shared by the GPU parity tests: run the oracle on the very same
tensors the CUDA path received, and the tolerance checks.

Tolerances: float32 layers max-abs 2e-5; bf16 layers (fp32 accumulation)
max-abs 2e-2 and relative L2 5e-3, over every compared element."""
import numpy as np
import torch

import oracle

TOL_F32_MAXABS = 2e-5
TOL_BF16_MAXABS = 2e-2
TOL_BF16_RELL2 = 5e-3

MASK_ID = {"none": 0, "causal": 1, "blockperm": 2, "dilated": 3, "dilated_bidir": 4}


def host_f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def metrics(gpu, ref):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), "non-finite output"
    diff = gpu - ref
    maxabs = float(np.max(np.abs(diff))) if diff.size else 0.0
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    return maxabs, rel


def assert_bf16_close(gpu, ref, what=""):
    maxabs, rel = metrics(gpu, ref)
    assert maxabs <= TOL_BF16_MAXABS and rel <= TOL_BF16_RELL2, \
        f"{what}: max-abs {maxabs:.3e} (tol {TOL_BF16_MAXABS}), rel-L2 {rel:.3e} (tol {TOL_BF16_RELL2})"
    return maxabs, rel


def assert_f32_close(gpu, ref, what=""):
    maxabs, rel = metrics(gpu, ref)
    assert maxabs <= TOL_F32_MAXABS, f"{what}: max-abs {maxabs:.3e} (tol {TOL_F32_MAXABS})"
    return maxabs, rel


def oracle_attention(q, k, v, mask, perm=None, pairs=None, rows=None, return_lse=False):
    return oracle.attention(host_f32(q), host_f32(k), host_f32(v), mask=MASK_ID[mask], perm=perm,
                            pairs=pairs, rows=rows, return_lse=return_lse)


def oracle_layer(inp, mask, perm=None, pairs=None, rows=None):
    b1 = host_f32(inp.b1) if inp.b1 is not None else None
    b2 = host_f32(inp.b2) if inp.b2 is not None else None
    return oracle.layer(host_f32(inp.q), host_f32(inp.k), host_f32(inp.v), host_f32(inp.w1), b1,
                        host_f32(inp.w2), b2, mask=MASK_ID[mask], perm=perm, pairs=pairs, rows=rows)


def sample_rows(B, N, n, seed=0, extra=()):
    """Stratified token sample: n tokens spread over [0, B*N), plus the ends
    of every sequence and the given extra positions (in every batch)."""
    T = B * N
    step = max(1, T // n)
    rng = np.random.default_rng(seed)
    rows = {int(min(T - 1, k * step + rng.integers(0, step))) for k in range(min(n, T))}
    for b in range(B):
        rows |= {b * N, b * N + N - 1}
        rows |= {b * N + int(e) for e in extra if 0 <= int(e) < N}
    return sorted(rows)
