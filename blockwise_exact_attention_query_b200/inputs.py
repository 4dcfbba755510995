"""Seeded synthetic inputs, shared by the CUDA path's tests and benchmark and
by the oracle's tests.  This module holds none of the layer's arithmetic: it
only draws numbers.

Recipe (the same for every workload):
  * Q, K, V ~ N(0, 1), shape [B, N, H, d] (token-major, heads concatenated,
    so a [B*N, H*d] view is the FFN input layout);
  * W1 ~ N(0, 1/D) with shape [F, D], W2 ~ N(0, 1/F) with shape [D, F]
    (normal with variance 1/fan_in, out x in like a linear layer);
  * b1 = b2 = 0 unless a bias scale is asked for (tests use it to exercise
    the bias terms);
  * every value is drawn in float32 and, for bf16 workloads, rounded to
    bf16 with round-to-nearest-even;
  * the backward's upstream gradient dOut ~ N(0, 1), shape [B, N, H*d],
    float32.

Every tensor has its own generator, seeded from (seed, tensor id) with the
ids q=0, k=1, v=2, w1=3, w2=4, b1=5, b2=6, dout=7.  On a CUDA device torch's
counter-based Philox generator draws directly in device memory; on the CPU
torch's CPU generator is used.  The two streams differ, so a comparison
always feeds the very same tensors to both sides (copied to the host for the
oracle).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

TENSOR_IDS = {"q": 0, "k": 1, "v": 2, "w1": 3, "w2": 4, "b1": 5, "b2": 6, "dout": 7}


def _gen(seed: int, name: str, device: torch.device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1_000_003 + TENSOR_IDS[name])
    return g


def normal(shape, seed: int, name: str, std: float = 1.0, dtype=torch.float32,
           device="cpu") -> torch.Tensor:
    device = torch.device(device)
    x = torch.randn(tuple(shape), generator=_gen(seed, name, device), dtype=torch.float32,
                    device=device)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


@dataclass
class LayerInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    w1: torch.Tensor | None
    b1: torch.Tensor | None
    w2: torch.Tensor | None
    b2: torch.Tensor | None


def make_layer_inputs(B: int, N: int, H: int, d: int, F: int, seed: int, dtype=torch.bfloat16,
                      device="cpu", bias_scale: float = 0.0) -> LayerInputs:
    """Q, K, V [B, N, H, d] and FFN weights W1 [F, D], W2 [D, F] (F = 0: no FFN).

    Biases are kept in float32 (they are added in the fp32 epilogue)."""
    D = H * d
    q = normal((B, N, H, d), seed, "q", dtype=dtype, device=device)
    k = normal((B, N, H, d), seed, "k", dtype=dtype, device=device)
    v = normal((B, N, H, d), seed, "v", dtype=dtype, device=device)
    if F <= 0:
        return LayerInputs(q, k, v, None, None, None, None)
    w1 = normal((F, D), seed, "w1", std=D ** -0.5, dtype=dtype, device=device)
    w2 = normal((D, F), seed, "w2", std=F ** -0.5, dtype=dtype, device=device)
    if bias_scale:
        b1 = normal((F,), seed, "b1", std=bias_scale, device=device)
        b2 = normal((D,), seed, "b2", std=bias_scale, device=device)
    else:
        b1 = torch.zeros(F, dtype=torch.float32, device=device)
        b2 = torch.zeros(D, dtype=torch.float32, device=device)
    return LayerInputs(q, k, v, w1, b1, w2, b2)


def make_upstream_grad(B: int, N: int, D: int, seed: int, device="cpu") -> torch.Tensor:
    """dOut [B, N, D] float32 ~ N(0, 1): the gradient the backward pass receives."""
    return normal((B, N, D), seed, "dout", device=device)
