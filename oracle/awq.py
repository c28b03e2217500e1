"""Plain CPU oracle of the AWQ W4A16 linear layer (float64 numpy).

TEST INFRASTRUCTURE ONLY: only tests/, __graft_entry__.smoke() and the CPU
baseline leg of bench.py may import this module.  It shares no code with
the CUDA path.

What the layer is (the pages): the Diffusers blog "Integrating Nunchaku 4-bit
diffusion inference into Diffusers", section "Introducing Nunchaku Lite",
names two kernel families; besides svdq_w4a4, awq_w4a16 keeps 4-bit weights
with 16-bit activations for the adaptive-normalization and modulation
projections (FLUX's adanorm_single / adanorm_zero, Qwen-Image's modulation
layers), which are memory-bound and sensitive to precision.  The section
"Native loading in Diffusers" gives its quantization_config: precision int4,
group_size 64, targets such as adaLN_modulation.1.

Readings where the pages are silent (each one is a choice of this build):
  * AWQ's activation-aware scaling is the per-input-channel factor s_k of
    the AWQ method: W' = diag(s) W and X' = X diag(s)^-1, so X' W' = X W
    (the same algebra as SVDQuant's smoothing).  Choosing s is an offline
    calibration on real activations, outside the layer; s is an input here
    (all ones when absent).  X' = fl32(x * fl32(1/s_k)), W' = fl32(w * s_k).
  * Groups of 64 run along K (the contraction), per output feature n.
  * The 4-bit code is asymmetric, AWQ's usual zero-point form: per group
    lo = min w', hi = max w', d = fp16_satfinite(fl32(max(fl32(hi - lo),
    1e-5) / 15)) (the stored binary16 scale, used as float32 for both
    quantization and dequantization), zero = clamp(rint(fl32(-lo / d)),
    0, 15), code = clamp(rint(fl32(w' / d)) + zero, 0, 15); rint is round
    half to even, divisions are IEEE float32.
  * Dequantized weight: w^ = (code - zero) d, exact in float32.
  * Y = X' W^ + b in float64, rounded once to bf16.
  * The tensor-core form (large batches, forward_16bit): the product runs
    on 16-bit operands, as W4A16 GEMMs do; X'16 = bf16(X') (X itself when
    s = 1) and w^16 = bf16((code - zero) d) (one rounding of the exact
    product); Y = bf16(X'16 W^16 + b), float64 in between.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

from . import formats as F

GROUP = 64
MAX_CODE = 15
MIN_RANGE = np.float32(1e-5)
FP16_MAX = 65504.0


@dataclass
class AwqWeights:
    K: int
    N: int
    inv_s: np.ndarray   # (K,) float32: fl32(1/s)
    s: np.ndarray       # (K,) float32
    code: np.ndarray    # (K, N) uint8 in [0, 15]
    scale: np.ndarray   # (K/64, N) float32 holding binary16 values
    zero: np.ndarray    # (K/64, N) uint8 in [0, 15]
    bias: np.ndarray    # (N,) float64


def fp16_satfinite(v) -> np.ndarray:
    """float32 -> binary16 (round to nearest even), saturating at +-65504
    instead of overflowing; returned as float32 values."""
    v = np.asarray(v, dtype=np.float32)
    h = np.clip(v, -FP16_MAX, FP16_MAX).astype(np.float16)
    # a value above 65504 that clipping brought to 65504 stays there; one in
    # (65504, 65520) would round up to infinity without the clip
    return h.astype(np.float32)


def scaled_weight(W, s) -> np.ndarray:
    """W' = fl32(w * s_k), row k scaled by the AWQ factor of input channel k."""
    W = np.asarray(W, np.float32)
    return (W * np.asarray(s, np.float32)[:, None]).astype(np.float32)


def quantize_groups(Wp) -> tuple:
    """The zero-point quantizer over groups of 64 along K of W' (K, N).
    Returns (code (K, N) uint8, scale (K/64, N) float32, zero (K/64, N) uint8)."""
    Wp = np.asarray(Wp, np.float32)
    K, N = Wp.shape
    assert K % GROUP == 0
    G = Wp.reshape(K // GROUP, GROUP, N)
    lo = G.min(axis=1)
    hi = G.max(axis=1)
    rng = np.maximum((hi - lo).astype(np.float32), MIN_RANGE)
    d = fp16_satfinite((rng / np.float32(MAX_CODE)).astype(np.float32))
    zero = np.clip(np.rint((-lo / d).astype(np.float32)), 0, MAX_CODE)
    q = np.rint((G / d[:, None, :]).astype(np.float32)) + zero[:, None, :]
    code = np.clip(q, 0, MAX_CODE).astype(np.uint8).reshape(K, N)
    return code, d.astype(np.float32), zero.astype(np.uint8)


def prepare(W, bias, s: Optional[np.ndarray] = None) -> AwqWeights:
    """Offline weight preparation: AWQ scaling, then the 4-bit group code."""
    W = np.asarray(W, np.float32)
    K, N = W.shape
    s = np.ones(K, np.float32) if s is None else np.asarray(s, np.float32)
    code, scale, zero = quantize_groups(scaled_weight(W, s))
    inv_s = (np.float32(1.0) / s).astype(np.float32)
    return AwqWeights(K=K, N=N, inv_s=inv_s, s=s, code=code, scale=scale, zero=zero,
                      bias=np.asarray(bias, np.float64))


def dequantize(aw: AwqWeights) -> np.ndarray:
    """W^ (K, N) float64: (code - zero) d per group, exact."""
    z = np.repeat(aw.zero.astype(np.float64), GROUP, axis=0)
    d = np.repeat(aw.scale.astype(np.float64), GROUP, axis=0)
    return (aw.code.astype(np.float64) - z) * d


def scaled_activation(aw: AwqWeights, X) -> np.ndarray:
    """X' = fl32(x * fl32(1/s_k))."""
    return (np.asarray(X, np.float32) * aw.inv_s[None, :]).astype(np.float32)


def dequantize_16bit(aw: AwqWeights) -> np.ndarray:
    """W^16 (K, N) float64 holding bf16 values: (code - zero) d rounded once."""
    return F.bf16_round(dequantize(aw))


def forward_16bit(aw: AwqWeights, X) -> dict:
    """The tensor-core form: Y = bf16(bf16(X') W^16 + b), float64 in between."""
    Xp16 = F.bf16_round(scaled_activation(aw, X).astype(np.float64))
    y = Xp16 @ dequantize_16bit(aw) + aw.bias[None, :]
    return dict(Xp16=Xp16, W16=dequantize_16bit(aw), Y=F.bf16_round(y))


def forward(aw: AwqWeights, X) -> dict:
    """Y = bf16(X' W^ + b) for X (M, K); float64 in between."""
    Xp = scaled_activation(aw, X).astype(np.float64)
    y = Xp @ dequantize(aw) + aw.bias[None, :]
    return dict(Xp=Xp, Y=F.bf16_round(y))
