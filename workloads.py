"""Seeded synthetic inputs for the QLoRA linear layer workloads.

This module only draws random tensors with the shapes and distributions of
the workloads; it contains none of the layer's arithmetic. Both the CPU
oracle's tests and the CUDA library's tests and benchmark take their inputs
from here, so the two sides always see identical bits.

Recipe (per workload; torch CPU generator seeded once, draws in this order):
  1. W0  fp32 [N, K]  ~ N(0, sigma^2)   (plus outliers where stated)
  2. A   bf16 [r, K]  ~ U(-1/sqrt(K), 1/sqrt(K))   (Kaiming-uniform, the
                                                     nn.Linear default bound)
  3. B   bf16 [N, r]  ~ N(0, 0.01^2)    (nonzero so the LoRA branch is live)
  4. x   bf16 [M, K]  ~ N(0, 1)
  5. dY  bf16 [M, N]  ~ N(0, 1)
bf16 tensors are drawn in fp32 and rounded once (round to nearest even).
Outliers: round(frac * N * K) distinct positions chosen uniformly without
replacement from a second generator seeded with seed + 7919, multiplied by
`outlier_scale`.

The workloads stand in for real LLaMA-13B / Llama-2-70B projection weights,
which are not available here; the pages use those models' shapes.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Optional

import torch


@dataclass(frozen=True)
class LayerWorkload:
    name: str
    N: int                 # output features (rows of W0)
    K: int                 # input features (columns of W0)
    M: int                 # tokens
    r: int
    alpha: float
    sigma: float
    double_quant: bool
    seed: int
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0
    forward_only: bool = False
    layers: int = 1        # independent projections (adapter stack)

    def with_(self, **kw) -> "LayerWorkload":
        return replace(self, **kw)


WORKLOADS = {
    # single 1024x1024 layer, no double quant, 16 tokens, rank 8
    "single_1024": LayerWorkload("single_1024", 1024, 1024, 16, 8, 16.0, 0.02, False, 1001),
    # LLaMA-13B attention projection, batch 4 x seq 512 tokens
    "llama13b_attn_5120": LayerWorkload("llama13b_attn_5120", 5120, 5120, 2048, 16, 32.0, 0.02,
                                        True, 1002),
    # decode-shaped MLP up-projection with 0.1% outliers x20, forward only
    "decode_mlp_up_13824x5120": LayerWorkload("decode_mlp_up_13824x5120", 13824, 5120, 16, 16,
                                              32.0, 0.02, True, 1003, outlier_frac=0.001,
                                              outlier_scale=20.0, forward_only=True),
    # LLaMA-13B adapter stack: 40 layers x {Q,K,V,O}, batch 8 x seq 512
    "llama13b_stack_40x4": LayerWorkload("llama13b_stack_40x4", 5120, 5120, 4096, 16, 32.0, 0.02,
                                         True, 4000, layers=160),
    # Llama-2-70B MLP projection, batch 16 x seq 512
    "llama2_70b_mlp_28672x8192": LayerWorkload("llama2_70b_mlp_28672x8192", 28672, 8192, 8192, 64,
                                               16.0, 0.015, True, 1005),
}


def stack_seed(layer: int, proj: int) -> int:
    """Seed of projection `proj` (0..3 = Q,K,V,O) of layer `layer` in the stack."""
    return 4000 + 4 * layer + proj


def make_weight(w: LayerWorkload, seed: Optional[int] = None) -> torch.Tensor:
    g = torch.Generator(device="cpu").manual_seed(w.seed if seed is None else seed)
    return _draw_weight(w, g, w.seed if seed is None else seed)


def _draw_weight(w: LayerWorkload, g: torch.Generator, seed: int) -> torch.Tensor:
    W0 = torch.randn(w.N, w.K, generator=g, dtype=torch.float32) * w.sigma
    if w.outlier_frac > 0.0:
        count = int(round(w.outlier_frac * w.N * w.K))
        go = torch.Generator(device="cpu").manual_seed(seed + 7919)
        pos = torch.randperm(w.N * w.K, generator=go)[:count]
        flat = W0.view(-1)
        flat[pos] = flat[pos] * w.outlier_scale
    return W0


def make_inputs(w: LayerWorkload, M: Optional[int] = None, seed: Optional[int] = None,
                with_dy: bool = True) -> dict:
    """All inputs of one projection, drawn in the documented order."""
    seed = w.seed if seed is None else seed
    M = w.M if M is None else M
    g = torch.Generator(device="cpu").manual_seed(seed)
    W0 = _draw_weight(w, g, seed)
    bound = 1.0 / (w.K ** 0.5)
    A = (torch.rand(w.r, w.K, generator=g, dtype=torch.float32) * (2 * bound) - bound)
    B = torch.randn(w.N, w.r, generator=g, dtype=torch.float32) * 0.01
    x = torch.randn(M, w.K, generator=g, dtype=torch.float32)
    out = {
        "W0": W0,
        "A": A.to(torch.bfloat16),
        "B": B.to(torch.bfloat16),
        "x": x.to(torch.bfloat16),
    }
    if with_dy and not w.forward_only:
        out["dY"] = torch.randn(M, w.N, generator=g, dtype=torch.float32).to(torch.bfloat16)
    return out


def bf16_bits(t: torch.Tensor):
    """uint16 numpy view of a bf16 CPU tensor's bit patterns."""
    import numpy as np
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
