"""Plain CPU oracle of the SVDQuant W4A4 linear layer (float64 numpy).

TEST INFRASTRUCTURE ONLY: only tests/, __graft_entry__.smoke() and the CPU
baseline leg of bench.py may import this module.  It shares no code with
the CUDA path.

What the layer computes (the pages):
  * Stage 2 of the SVDQuant overview figure ("svdq-int4-flux.1-dev" model
    card): outliers migrate from the activation to the weight,
    X^ = X diag(lambda)^-1, W^ = diag(lambda) W, so X^ W^ = X W.
  * Stage 3 of the same figure: an SVD splits W^ into a 16-bit low-rank
    branch L1 L2 and a residual R = W^ - L1 L2 that is quantized to 4 bits.
  * The "SVDQuant: ..." abstract: the low-rank branch runs at high precision,
    the 4-bit branch takes the residual; LoRAs attach to the low-rank branch
    without re-quantizing R; formats INT4 and NVFP4.
  * Diffusers blog, "Native loading in Diffusers": nvfp4 uses group_size 16
    at rank 32.
  So  Y = X^ L1 L2 + Q(X^) Q(R) + b.

Readings where the pages are silent (each one is a choice of this build):
  * lambda_k = max_m|X[m,k]|^a / max_n|W[k,n]|^(1-a), a = 0.5, computed in
    float64 and rounded once to float32; lambda_k = 1 where either max is 0.
    1/lambda is the correctly rounded float32 reciprocal.
  * SVD split of Sigma: L1 = U_r Sigma_r, L2 = V_r^T; each right singular
    vector is signed so its largest-magnitude entry is positive (lowest index
    wins a tie).
  * lambda^-1 is folded into the first factor: L1f = bf16(diag(lambda)^-1
    U_r Sigma_r) (one rounding from float64), L2 = bf16(V_r^T).  X L1f equals
    X^ L1 in exact arithmetic, and a LoRA's A factor then applies to the raw
    X unchanged.
  * R[k,n] = fp32(lambda_k W[k,n] - lambda_k sum_{i<r} L1f[k,i] L2[i,n]),
    float64, i ascending, separate multiply and add, one final rounding.
    The rounded factors are used, so low-rank + residual rebuild W^.
  * Groups run along K (the contraction), per activation row and per weight
    output column.
  * NVFP4 tensor scales: the activation's s_tX is a static calibration,
    fp32(amax(|X^|) / 2688) (2688 = 6 * 448; 1 if the amax is 0); the
    residual's is s_tR = fl32(2^k / s_tX) with k the smallest integer such
    that 2^k >= s_tX amax(|R|) / 2688, so s_tR >= amax(|R|) / 2688 and
    s_tX s_tR is a power of two (see weight_tensor_scale).
    Per block of 16: a = max|v|, sb = E4M3(a / fp32(6 s_t)),
    d = fp32(f32(sb) s_t), inv = fp32(1/d) (0 if d = 0),
    code = E2M1(fp32(v inv)).  The activation tensor scale is static (an
    offline calibration: amax of X^ / 2688) or, per call, the batch's own
    (dynamic_act_scale: the batch's amax paired with s_tR to a power of two).
  * INT4: per block of 64: sb = fp16(fp32(a / 7)), d = f32(sb),
    inv = fp32(1/d) (0 if d = 0), code = clamp(rint(fp32(v inv)), -8, 7).
  * The low-rank down-projection output LR is rounded to bf16 (it is the
    16-bit branch's intermediate); the output Y is rounded to bf16.
  * The fused GELU of the blog's "Introducing Nunchaku Lite" section is the
    tanh form 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3))).
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Optional

import numpy as np

from . import formats as F

NVFP4_GROUP = 16
INT4_GROUP = 64
NVFP4_TENSOR_DIVISOR = np.float32(6.0 * 448.0)   # 2688


# ============================================================ smoothing (Stage 2)
def smoothing_factors(X, W, alpha: float = 0.5) -> np.ndarray:
    """Per-input-channel migration strength lambda (float32, length K).

    X: (M, K) activation used for calibration; W: (K, N) math weight."""
    ax = np.max(np.abs(np.asarray(X, np.float64)), axis=0)
    aw = np.max(np.abs(np.asarray(W, np.float64)), axis=1)
    if alpha == 0.5:
        num, den = np.sqrt(ax), np.sqrt(aw)
    else:
        num, den = ax ** alpha, aw ** (1.0 - alpha)
    with np.errstate(divide="ignore", invalid="ignore"):
        lam = num / den
    lam = np.where((ax == 0) | (aw == 0), 1.0, lam)
    return lam.astype(np.float32)


def inverse_lambda(lam) -> np.ndarray:
    lam = np.asarray(lam, np.float32)
    return (np.float32(1.0) / lam).astype(np.float32)


def smooth_activation(X, inv_lam) -> np.ndarray:
    """X^ = X diag(lambda)^-1 as one float32 multiply per element."""
    return (np.asarray(X, np.float32) * np.asarray(inv_lam, np.float32)[None, :]).astype(np.float32)


def act_tensor_scale(X, inv_lam) -> np.float32:
    """Static NVFP4 activation tensor scale: amax(|X^|) / 2688 in float32."""
    a = np.float32(np.max(np.abs(smooth_activation(X, inv_lam)))) if np.size(X) else np.float32(0)
    return np.float32(1.0) if a == 0 else np.float32(a / NVFP4_TENSOR_DIVISOR)


# ============================================================ SVD split (Stage 3)
def svd_split(W, lam, rank: int):
    """Truncated SVD of W^ = diag(lambda) W in float64, before any rounding.

    Returns (U_r (K, r), sigma (all singular values), Vt_r (r, N), W^), with
    each right singular vector signed so its largest-|.| entry is positive
    (first index wins a tie) and the matching left vector flipped with it."""
    W = np.asarray(W, np.float64)
    lam64 = np.asarray(lam, np.float32).astype(np.float64)
    What = lam64[:, None] * W                       # exact: 24-bit x 8-bit significands
    U, S_all, Vt = np.linalg.svd(What, full_matrices=False)
    U, Vt = U[:, :rank], Vt[:rank]
    piv = np.argmax(np.abs(Vt), axis=1)
    sgn = np.where(Vt[np.arange(Vt.shape[0]), piv] < 0, -1.0, 1.0)
    return U * sgn[None, :], S_all, Vt * sgn[:, None], What


def svd_factors(W, lam, rank: int):
    """The 16-bit low-rank factors with lambda^-1 folded into the first.

    Returns (L1f, L2, sigma): L1f = bf16(diag(lambda)^-1 U_r Sigma_r) (K, r)
    and L2 = bf16(V_r^T) (r, N) as float64 arrays of bf16 values, and all
    singular values of W^."""
    U, S_all, Vt, _ = svd_split(W, lam, rank)
    lam64 = np.asarray(lam, np.float32).astype(np.float64)
    L1 = U * S_all[None, :rank]
    L1f = F.bf16_round(L1 / lam64[:, None])
    L2 = F.bf16_round(Vt)
    return L1f, L2, S_all


def residual(W, lam, L1f, L2) -> np.ndarray:
    """R = lambda o W - lambda o (L1f L2) in float64 with i ascending, no fused
    multiply-add, rounded once to float32.  Returns (K, N) float32."""
    W = np.asarray(W, np.float64)
    lam64 = np.asarray(lam, np.float32).astype(np.float64)[:, None]
    L1f = np.asarray(L1f, np.float64)
    L2 = np.asarray(L2, np.float64)
    S = np.zeros_like(W)
    for i in range(L1f.shape[1]):
        S = S + L1f[:, i:i + 1] * L2[i:i + 1, :]
    return (lam64 * W - lam64 * S).astype(np.float32)


def tensor_scale(V) -> np.float32:
    a = np.float32(np.max(np.abs(np.asarray(V, np.float32)))) if np.size(V) else np.float32(0)
    return np.float32(1.0) if a == 0 else np.float32(a / NVFP4_TENSOR_DIVISOR)


def weight_tensor_scale(R, s_tX):
    """NVFP4 tensor scale of the residual, paired with the activation's.

    k is the smallest integer with 2^k >= s_tX amax(|R|) / 2688 (float64;
    amax 0 counts as 2688), and s_tR = fl32(2^k / s_tX).  Then s_tR is at
    least amax / 2688 up to one float32 rounding, so no block scale needs
    more than E4M3's 448, and the product alpha = s_tX s_tR that the 4-bit
    product is multiplied by is 2^k up to that rounding: the 16-bit branch
    can carry 1/alpha exactly.  Returns (s_tR, k)."""
    a = float(np.max(np.abs(np.asarray(R, np.float32)))) if np.size(R) else 0.0
    x = (a if a > 0 else 2688.0) * float(np.float32(s_tX)) / 2688.0
    m, e = np.frexp(x)
    k = int(e - 1) if m == 0.5 else int(e)
    return np.float32(np.float32(np.ldexp(1.0, k)) / np.float32(s_tX)), k


# ============================================================ 4-bit group quantization
def quantize_nvfp4(V, s_t):
    """Rows of V (rows, K) in groups of 16 along K.

    Returns codes (rows, K) uint8 4-bit E2M1 codes and scales (rows, K/16)
    uint8 E4M3 codes."""
    V = np.asarray(V, np.float32)
    rows, K = V.shape
    G = V.reshape(rows, K // NVFP4_GROUP, NVFP4_GROUP)
    a = np.max(np.abs(G), axis=2).astype(np.float32)
    s_t = np.float32(s_t)
    six_st = np.float32(np.float32(6.0) * s_t)
    sb_code = F.e4m3_encode_satfinite((a / six_st).astype(np.float32))
    sb = F.e4m3_decode(sb_code).astype(np.float32)
    d = (sb * s_t).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(d == 0, np.float32(0), np.float32(1.0) / d).astype(np.float32)
    q = F.e2m1_encode((G * inv[:, :, None]).astype(np.float32))
    return q.reshape(rows, K), sb_code


def quantize_int4(V):
    """Rows of V (rows, K) in groups of 64 along K.

    Returns codes (rows, K) int8 in [-8, 7] and scales (rows, K/64) float16."""
    V = np.asarray(V, np.float32)
    rows, K = V.shape
    G = V.reshape(rows, K // INT4_GROUP, INT4_GROUP)
    a = np.max(np.abs(G), axis=2).astype(np.float32)
    sb = F.to_fp16((a / np.float32(7.0)).astype(np.float32))
    d = sb.astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(d == 0, np.float32(0), np.float32(1.0) / d).astype(np.float32)
    q = F.int4_encode((G * inv[:, :, None]).astype(np.float32))
    return q.reshape(rows, K), sb


def dequantize_nvfp4(codes, scales) -> np.ndarray:
    """codes (rows, K), E4M3 scales (rows, K/16) -> float64 e2m1 * scale
    (without the tensor scale)."""
    vals = F.e2m1_decode(codes)
    sc = F.e4m3_decode(scales)
    return vals * np.repeat(sc, NVFP4_GROUP, axis=1)


def dequantize_int4(codes, scales) -> np.ndarray:
    return np.asarray(codes, np.float64) * np.repeat(np.asarray(scales, np.float64), INT4_GROUP, axis=1)


# ============================================================ the two branches
def lowrank_down(X, L1f_all, round_bf16: bool = True) -> np.ndarray:
    """LR = X L1f (float64 sum), rounded to bf16 (the 16-bit intermediate)."""
    lr = np.asarray(X, np.float64) @ np.asarray(L1f_all, np.float64)
    return F.bf16_round(lr) if round_bf16 else lr


def lowrank_up(LR, L2_all) -> np.ndarray:
    return np.asarray(LR, np.float64) @ np.asarray(L2_all, np.float64)


def gelu_tanh(y) -> np.ndarray:
    y = np.asarray(y, np.float64)
    return 0.5 * y * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (y + 0.044715 * y ** 3)))


# ============================================================ whole layer
@dataclass
class PreparedWeights:
    fmt: str
    K: int
    N: int
    rank: int
    lam: np.ndarray          # (K,) float32
    inv_lam: np.ndarray      # (K,) float32
    L1f: np.ndarray          # (K, r_tot) bf16 values, SVD factor then LoRA A
    L2: np.ndarray           # (r_tot, N) bf16 values, SVD factor then LoRA B
    R: np.ndarray            # (K, N) float32 residual
    qR: np.ndarray           # (N, K) codes (uint8 e2m1 or int8 int4)
    sR: np.ndarray           # (N, K/g) scales (uint8 e4m3 or float16)
    s_tR: np.float32         # NVFP4 weight tensor scale (1 for INT4)
    s_tX: np.float32         # NVFP4 static activation tensor scale (1 for INT4)
    bias: np.ndarray         # (N,) bf16 values
    sigma: Optional[np.ndarray] = None
    alpha_log2: int = 0      # log2 of the power of two that s_tX s_tR rounds to


def prepare(fmt: str, W, lam, L1f, L2, bias, act_scale=None, lora_A=None, lora_B=None,
            sigma=None) -> PreparedWeights:
    """Offline weight preparation: residual, its 4-bit quantization, and the
    low-rank factors with an optional LoRA appended (the LoRA does not touch
    R: SVDQuant abstract, 'without re-quantization')."""
    W = np.asarray(W, np.float32)
    K, N = W.shape
    lam = np.asarray(lam, np.float32)
    R = residual(W, lam, L1f, L2)
    if fmt == "nvfp4":
        s_tX = np.float32(act_scale)
        s_tR, alpha_log2 = weight_tensor_scale(R, s_tX)
        qR, sR = quantize_nvfp4(R.T.copy(), s_tR)
    elif fmt == "int4":
        s_tR = np.float32(1.0)
        s_tX = np.float32(1.0)
        alpha_log2 = 0
        qR, sR = quantize_int4(R.T.copy())
    else:
        raise ValueError(fmt)
    L1f_all = np.asarray(L1f, np.float64)
    L2_all = np.asarray(L2, np.float64)
    if lora_A is not None:
        L1f_all = np.concatenate([L1f_all, np.asarray(lora_A, np.float64)], axis=1)
        L2_all = np.concatenate([L2_all, np.asarray(lora_B, np.float64)], axis=0)
    return PreparedWeights(fmt=fmt, K=K, N=N, rank=np.asarray(L1f).shape[1], lam=lam,
                           inv_lam=inverse_lambda(lam), L1f=L1f_all, L2=L2_all, R=R, qR=qR, sR=sR,
                           s_tR=s_tR, s_tX=s_tX, bias=np.asarray(bias, np.float64), sigma=sigma,
                           alpha_log2=alpha_log2)


def quantize_activation(pw: PreparedWeights, X):
    """Kernel-1 half of the layer: X^ and its 4-bit codes and scales."""
    Xh = smooth_activation(X, pw.inv_lam)
    if pw.fmt == "nvfp4":
        return quantize_nvfp4(Xh, pw.s_tX)
    return quantize_int4(Xh)


def dynamic_act_scale(pw: PreparedWeights, X):
    """Per-call NVFP4 activation tensor scale (a reading: the pages fix only
    the FP32 tensor scale, not how it is chosen).  The batch's own
    a = amax(|X^|) takes the place of the calibration value, paired with the
    residual's tensor scale the way weight_tensor_scale pairs it the other
    way round: j is the smallest integer with 2^j >= s_tR a / 2688 (float64;
    a = 0 counts as 2688) and s_tX = fl32(2^j / s_tR), so no block scale needs
    more than 448 and s_tX s_tR is the power of two 2^j.  Returns (s_tX, j)."""
    Xh = smooth_activation(X, pw.inv_lam)
    a = float(np.max(np.abs(Xh))) if np.size(Xh) else 0.0
    x = (a if a > 0 else NVFP4_TENSOR_DIVISOR) * float(np.float32(pw.s_tR)) / float(NVFP4_TENSOR_DIVISOR)
    m, e = np.frexp(x)
    j = int(e - 1) if m == 0.5 else int(e)
    return np.float32(np.float32(np.ldexp(1.0, j)) / np.float32(pw.s_tR)), j


def with_act_scale(pw: PreparedWeights, s_tX) -> PreparedWeights:
    """The same prepared layer with another NVFP4 activation tensor scale."""
    return replace(pw, s_tX=np.float32(s_tX))


def main_product(pw: PreparedWeights, qX, sX) -> np.ndarray:
    """Q(X^) Q(R) in float64 from the codes and scales."""
    if pw.fmt == "nvfp4":
        alpha = np.float64(pw.s_tX) * np.float64(pw.s_tR)
        return alpha * (dequantize_nvfp4(qX, sX) @ dequantize_nvfp4(pw.qR, pw.sR).T)
    return dequantize_int4(qX, sX) @ dequantize_int4(pw.qR, pw.sR).T


def epilogue(y, bias, gelu: bool) -> np.ndarray:
    y = np.asarray(y, np.float64) + np.asarray(bias, np.float64)[None, :]
    if gelu:
        y = gelu_tanh(y)
    return F.bf16_round(y)


def forward(pw: PreparedWeights, X, gelu: bool = False, quantize: bool = True, dynamic: bool = False):
    """Y for activation X (M, K).  Returns dict with the intermediates.

    dynamic=True (NVFP4) quantizes X^ with its own tensor scale
    (dynamic_act_scale) instead of the calibrated one.

    quantize=False replaces every rounding of the layer's data path (the two
    4-bit quantizers, the bf16 LR and the bf16 output) by the identity, which
    leaves X^ R + X L1f L2 + b: equal to X W + b up to float32 rounding."""
    X = np.asarray(X, np.float32)
    if dynamic and pw.fmt == "nvfp4":
        pw = with_act_scale(pw, dynamic_act_scale(pw, X)[0])
    if quantize:
        qX, sX = quantize_activation(pw, X)
        LR = lowrank_down(X, pw.L1f)
        y = main_product(pw, qX, sX) + lowrank_up(LR, pw.L2)
        return dict(qX=qX, sX=sX, LR=LR, Y=epilogue(y, pw.bias, gelu))
    Xh = smooth_activation(X, pw.inv_lam).astype(np.float64)
    LR = lowrank_down(X, pw.L1f, round_bf16=False)
    y = Xh @ pw.R.astype(np.float64) + lowrank_up(LR, pw.L2) + pw.bias[None, :]
    if gelu:
        y = gelu_tanh(y)
    return dict(LR=LR, Y=y)


def calibrate_and_prepare(fmt: str, X, W, bias, rank: int, lora_A=None, lora_B=None,
                          alpha: float = 0.5) -> PreparedWeights:
    """The offline pipeline in the pages' order: smoothing factors from the
    calibration activation, SVD of W^, residual quantization."""
    lam = smoothing_factors(X, W, alpha)
    L1f, L2, sigma = svd_factors(W, lam, rank)
    act_scale = act_tensor_scale(X, inverse_lambda(lam)) if fmt == "nvfp4" else None
    return prepare(fmt, W, lam, L1f, L2, bias, act_scale, lora_A, lora_B, sigma=sigma)
