"""Seeded synthetic inputs for the SVDQuant W4A4 linear layer.

This module only draws random numbers and names the workload shapes.  It
holds none of the method's arithmetic (no smoothing, no SVD, no
quantization), so both the CPU oracle and the CUDA path can take their
inputs from here without sharing any computation.

The pages' workloads are FLUX.1-style diffusion transformers run on real
prompts ("svdq-int4-flux.1-dev" model card, SVDQuant overview figure; the
"SVDQuant: Absorbing Outliers by Low-Rank Components for 4-Bit Diffusion
Models" abstract).  Neither the trained weights nor the calibration dataset
are available, so these generators stand in for them with FLUX-shaped
matrices that carry the outlier structure the method is about: a few input
channels of the activation are much larger than the rest (x20), and the
same input channels of the weight are also larger (x5).

Recipe (one torch CPU generator per workload, draws in this order):
  outlier channel indices = randperm(K)[:n_out]
  X    = randn(M, K), x20 on the outlier columns, rounded to bf16
  W    = randn(K, N) * 0.02, x5 on the outlier rows, rounded to bf16
  bias = randn(N) * 0.01, rounded to bf16
  (LoRA) A = randn(K, l) * 0.01, B = randn(l, N) * 0.01, both bf16
n_out = 8 for the small case, round(0.005 * K) otherwise.

All arrays are returned as float32 numpy arrays holding bf16-representable
values, with the weight in the math orientation W[k, n] (K x N); the C-ABI
takes the transpose, in nn.Linear order [N][K].
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch


def _bf16(t: torch.Tensor) -> np.ndarray:
    """Round a float32 tensor to bf16 (torch's round-to-nearest-even) and
    hand it back as float32 numpy values."""
    return t.to(torch.bfloat16).to(torch.float32).numpy()


@dataclass
class Layer:
    """One synthetic linear layer: activation, weight, bias and optional LoRA."""
    name: str
    fmt: str            # "nvfp4" or "int4"
    M: int
    K: int
    N: int
    rank: int
    X: np.ndarray       # (M, K) float32, bf16 values
    W: np.ndarray       # (K, N) float32, bf16 values
    bias: np.ndarray    # (N,) float32, bf16 values
    gelu: bool = False
    lora_A: Optional[np.ndarray] = None   # (K, l)
    lora_B: Optional[np.ndarray] = None   # (l, N)
    seed: int = 0
    outlier_channels: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))


def n_outliers(K: int) -> int:
    return int(round(0.005 * K))


def draw_layer(name: str, fmt: str, M: int, K: int, N: int, rank: int, seed: int,
               n_out: Optional[int] = None, gelu: bool = False, lora_rank: int = 0,
               gen: Optional[torch.Generator] = None) -> Layer:
    """Draw one layer with the outlier recipe above."""
    g = gen if gen is not None else torch.Generator("cpu").manual_seed(seed)
    if n_out is None:
        n_out = n_outliers(K)
    idx = torch.randperm(K, generator=g)[:n_out]
    X = torch.randn(M, K, generator=g)
    X[:, idx] *= 20.0
    W = torch.randn(K, N, generator=g) * 0.02
    W[idx, :] *= 5.0
    b = torch.randn(N, generator=g) * 0.01
    A = B = None
    if lora_rank:
        A = _bf16(torch.randn(K, lora_rank, generator=g) * 0.01)
        B = _bf16(torch.randn(lora_rank, N, generator=g) * 0.01)
    return Layer(name=name, fmt=fmt, M=M, K=K, N=N, rank=rank, X=_bf16(X), W=_bf16(W),
                 bias=_bf16(b), gelu=gelu, lora_A=A, lora_B=B, seed=seed,
                 outlier_channels=np.sort(idx.numpy()))


def draw_weight_only(K: int, N: int, n_out: int, gen: torch.Generator):
    """Weight and bias of a layer whose activation comes from another layer
    (the second linear of an MLP): outlier rows x5, no activation outliers."""
    idx = torch.randperm(K, generator=gen)[:n_out]
    W = torch.randn(K, N, generator=gen) * 0.02
    W[idx, :] *= 5.0
    b = torch.randn(N, generator=gen) * 0.01
    return _bf16(W), _bf16(b), np.sort(idx.numpy())


# ---------------------------------------------------------------------------
# The five workloads.  Shapes follow FLUX.1's 3072-wide transformer: the fused
# QKV projection (N = 3 * 3072) and the MLP pair (3072 -> 12288 -> 3072), at
# 4608 tokens (4096 image + 512 text).  NVFP4 uses group 16 at rank 32 (the
# quantization_config example of the Diffusers "Native loading" section).
# ---------------------------------------------------------------------------

SMALL = dict(name="nvfp4_small_M128_K1024_N1024_r32", fmt="nvfp4", M=128, K=1024, N=1024,
             rank=32, seed=0, n_out=8)
QKV = dict(name="nvfp4_qkv_M4608_K3072_N9216_r32", fmt="nvfp4", M=4608, K=3072, N=9216,
           rank=32, seed=1)
INT4_QKV = dict(name="int4_qkv_M4608_K3072_N9216_r32", fmt="int4", M=4608, K=3072, N=9216,
                rank=32, seed=3)


def small() -> Layer:
    return draw_layer(**SMALL)


def qkv() -> Layer:
    return draw_layer(**QKV)


def int4_qkv() -> Layer:
    return draw_layer(**INT4_QKV)


def mlp_pair(M: int = 4608):
    """FLUX-like MLP: fc1 3072 -> 12288 with GELU, fc2 12288 -> 3072.

    fc2's activation is fc1's output, so only fc2's weight and bias are drawn
    here; its weight gets round(0.005 * 12288) = 61 outlier rows.
    Returns (fc1 Layer, (W2, b2, outlier rows of W2))."""
    g = torch.Generator("cpu").manual_seed(2)
    fc1 = draw_layer("nvfp4_mlp_fc1_M%d_K3072_N12288_r32_gelu" % M, "nvfp4", M, 3072, 12288,
                     32, seed=2, gelu=True, gen=g)
    fc2 = draw_weight_only(12288, 3072, n_outliers(12288), g)
    return fc1, fc2


LORA_SWEEP_M = (256, 1024, 4096, 16384)
LORA_SWEEP_R = (16, 32, 64, 128)
LORA_RANK = 16


def lora_sweep_base(M_max: int = 16384) -> Layer:
    """One activation at the largest M (smaller M use its first rows), one
    3072 x 3072 weight, and one rank-16 LoRA; the SVD is taken once at the
    largest rank and smaller ranks use its leading factors."""
    return draw_layer("nvfp4_lora_sweep_K3072_N3072", "nvfp4", M_max, 3072, 3072, 128, seed=4,
                      lora_rank=LORA_RANK)


def dyadic_layer(M: int, K: int, N: int, rank: int, seed: int) -> dict:
    """Inputs whose products and partial sums are exact in fp32 in any order:
    integers in [-8, 8] scaled by 2^-4.  Used to check the low-rank
    down-projection bit for bit."""
    g = torch.Generator("cpu").manual_seed(seed)
    X = torch.randint(-8, 9, (M, K), generator=g).float() / 16.0
    L1 = torch.randint(-8, 9, (K, rank), generator=g).float() / 16.0
    return dict(X=X.numpy(), L1f=L1.numpy())


# ---------------------------------------------------------------------------
# AWQ W4A16 (the Diffusers blog's awq_w4a16 kernel family): the adaptive-norm
# modulation projection of a FLUX-style block, Linear(3072 -> 6 * 3072), fed
# with SiLU of the conditioning embedding, one row per image.
# Recipe (one torch CPU generator, draws in this order):
#   X = silu(randn(M, K)) rounded to bf16;  W = randn(K, N) * 0.02 -> bf16;
#   bias = randn(N) * 0.01 -> bf16;  s = exp(uniform(-1, 1, K)) (float32),
#   the AWQ per-input-channel scale, drawn only when asked for.
# ---------------------------------------------------------------------------

@dataclass
class AwqLayer:
    name: str
    M: int
    K: int
    N: int
    X: np.ndarray       # (M, K) float32, bf16 values
    W: np.ndarray       # (K, N) float32, bf16 values
    bias: np.ndarray    # (N,) float32, bf16 values
    s: Optional[np.ndarray] = None   # (K,) float32 or None
    seed: int = 0


AWQ_ADALN = dict(name="awq_w4a16_adaln_M1_K3072_N18432", M=1, K=3072, N=18432, seed=5)


def draw_awq_layer(name: str, M: int, K: int, N: int, seed: int, with_scale: bool = False) -> AwqLayer:
    g = torch.Generator("cpu").manual_seed(seed)
    X = torch.nn.functional.silu(torch.randn(M, K, generator=g))
    W = torch.randn(K, N, generator=g) * 0.02
    b = torch.randn(N, generator=g) * 0.01
    s = torch.exp(torch.rand(K, generator=g) * 2.0 - 1.0).numpy().astype(np.float32) if with_scale else None
    return AwqLayer(name=name, M=M, K=K, N=N, X=_bf16(X), W=_bf16(W), bias=_bf16(b), s=s, seed=seed)


def awq_adaln(M: int = 1) -> AwqLayer:
    d = dict(AWQ_ADALN)
    d["M"] = M
    if M != 1:
        d["name"] = "awq_w4a16_adaln_M%d_K3072_N18432" % M
    return draw_awq_layer(**d)


def awq_qkv() -> AwqLayer:
    """The QKV workload's activation, weight and bias as an AWQ W4A16 layer
    (no AWQ scale): the W4A16 side of the W4A4-over-W4A16 comparison on the
    same shape (M=4608, K=3072, N=9216)."""
    L = qkv()
    return AwqLayer(name="awq_w4a16_qkv_M4608_K3072_N9216", M=L.M, K=L.K, N=L.N, X=L.X, W=L.W, bias=L.bias,
                    s=None, seed=L.seed)
