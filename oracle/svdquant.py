"""SVDQuant prepare / forward / LoRA attach, restated plainly (test infrastructure).

Only tests, the smoke check and the benchmark's CPU baseline may import this.

Layout convention: W is [K, N] (Y = X W + b, as in the migration identity of
the msModelSlim entry, section 2.3 eq. 1). That page writes the SVD factors
in PyTorch's [out, in] notation, U [out_dim, rank], V [in_dim, rank]; with
W = [K, N] = [in, out] they become L1 = V_r ([K, r], the input-side factor the
branch multiplies first: X diag(s)^-1 V) and L2 = (U_r S_r)^T ([r, N], the
singular values on the output side, as in (U S)). The low-rank branch is kept
in bfloat16 ("high precision (such as FP16)", section 2.4).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

from .formats import (
    F32,
    bf16_round,
    dequantize,
    nvfp4_tensor_scale,
    quantize_int4_g64,
    quantize_nvfp4_g16,
)

S_MIN = F32(1e-5)


def group_size(fmt: str) -> int:
    return {"int4_g64": 64, "nvfp4_g16": 16}[fmt]


@dataclass
class Prepared:
    """Canonical prepared layer: every array in the layout the tests compare."""

    fmt: str
    K: int
    N: int
    rank: int
    alpha: float
    s: np.ndarray  # float32 [K]
    inv_s: np.ndarray  # float32 [K]
    L1: np.ndarray  # float64 holding bf16 values [K, r]
    L2: np.ndarray  # float64 holding bf16 values [r, N]
    R: np.ndarray  # float32 [K, N] residual
    w_codes: np.ndarray  # [N, K]: int8 (INT4) or uint8 E2M1 codes (NVFP4)
    w_scales: np.ndarray  # [N, K/G]: float32 (INT4) or uint8 E4M3 (NVFP4)
    g_w: np.float32  # NVFP4 tensor scale of R (1 for INT4)
    g_x: np.float32  # NVFP4 static activation tensor scale (1 for INT4)
    bias: np.ndarray  # float64 holding bf16 values [N]
    sigma: np.ndarray = field(default=None)  # float64 singular values of W_hat (all of them)


def calibrate_absmax(X: np.ndarray) -> np.ndarray:
    """A_scale: per-input-channel absolute maximum of calibration activations
    (msModelSlim entry, section 2.3, the A_scale definition under eq. 2)."""
    return np.max(np.abs(np.asarray(X, dtype=np.float64)), axis=0).astype(F32)


def weight_absmax(W: np.ndarray) -> np.ndarray:
    """W_scale: the weight statistic of eq. 2, read as the absolute maximum per
    input channel k (a row of W [K, N]) - the channel that diag(s) scales."""
    return np.max(np.abs(np.asarray(W, dtype=np.float64)), axis=1).astype(F32)


def smoothing_factors(a: np.ndarray, w: np.ndarray, alpha: float, s_min: float = float(S_MIN), smooth: bool = True):
    """Eq. 2 of section 2.3: s = A_scale^alpha / W_scale^(1 - alpha), s >= s_min.

    Computed in float64 (sqrt(a) / sqrt(w) when alpha = 0.5, which is exact
    up to one rounding per operation), rounded once to float32, clamped below
    at s_min; a channel whose activation or weight statistic is 0 keeps s = 1.
    inv_s = 1 / s in float32. With smooth=False (the ablation without
    migration) s = 1 for every channel.
    """
    if not smooth:
        ones = np.ones(np.asarray(a).shape, dtype=F32)
        return ones, ones.copy()
    alpha = float(F32(alpha))  # alpha is a float32 parameter of the layer
    a64 = np.asarray(a, dtype=np.float64)
    w64 = np.asarray(w, dtype=np.float64)
    dead = (a64 == 0) | (w64 == 0)
    a_safe = np.where(dead, 1.0, a64)
    w_safe = np.where(dead, 1.0, w64)
    if alpha == 0.5:
        s = np.sqrt(a_safe) / np.sqrt(w_safe)
    else:
        s = np.power(a_safe, alpha) / np.power(w_safe, 1.0 - alpha)
    s = np.where(dead, 1.0, s)
    s32 = np.maximum(s.astype(F32), F32(s_min)).astype(F32)
    inv_s = (F32(1.0) / s32).astype(F32)
    return s32, inv_s


def migrate_weight(W: np.ndarray, s: np.ndarray) -> np.ndarray:
    """diag(s) W of eq. 1, rounded to float32: W_hat[k, n] = fp32(s_k * W[k, n])."""
    return (np.asarray(s, dtype=F32)[:, None] * np.asarray(W, dtype=F32)).astype(F32)


def svd_factors(W_hat: np.ndarray, rank: int, round_bf16: bool = True):
    """Rank-r truncated SVD of the migrated weight (section 2.2; eq. 3).

    numpy.linalg.svd (LAPACK, float64) gives W_hat = U diag(sigma) V^T with
    sigma descending. L1 = U_r [K, r], L2 = diag(sigma_r) V_r^T [r, N]: the
    singular values go with the output-side factor, as in (U S). Each column
    of L1 is signed so that its largest-magnitude entry is positive (the
    product L1 L2 does not change). With round_bf16 the factors are rounded
    to bfloat16, the precision the branch runs in.
    Returns (L1, L2, sigma) in float64.
    """
    U, sigma, Vt = np.linalg.svd(np.asarray(W_hat, dtype=np.float64), full_matrices=False)
    L1 = U[:, :rank].copy()
    L2 = sigma[:rank, None] * Vt[:rank, :]
    for j in range(L1.shape[1]):
        if L1[np.argmax(np.abs(L1[:, j])), j] < 0:
            L1[:, j] = -L1[:, j]
            L2[j, :] = -L2[j, :]
    if round_bf16:
        L1 = bf16_round(L1)
        L2 = bf16_round(L2)
    return L1, L2, sigma


def residual(W_hat: np.ndarray, L1: np.ndarray, L2: np.ndarray) -> np.ndarray:
    """R = W_hat - L1 L2 (section 2.2, W = L + R), in float64, one rank term
    at a time in the order j = 0 .. r-1, then rounded once to float32."""
    acc = np.asarray(W_hat, dtype=np.float64).copy()
    for j in range(L1.shape[1]):
        acc -= np.outer(L1[:, j], L2[j, :])
    return acc.astype(F32)


def quantize_rows(v: np.ndarray, fmt: str, g: Optional[np.float32] = None):
    """Q(.) of eq. 4 applied along the last axis (groups along K)."""
    if fmt == "int4_g64":
        return quantize_int4_g64(v)
    if fmt == "nvfp4_g16":
        return quantize_nvfp4_g16(v, g)
    raise ValueError(fmt)


def static_activation_scale(a: np.ndarray, inv_s: np.ndarray) -> np.float32:
    """NVFP4 tensor scale of the smoothed activations, fixed at prepare time
    from the calibration statistic: g_x = max_k fp32(a_k * inv_s_k) / 2688.
    (The largest |x_hat| of any calibration row is at most this, because
    rounding is monotone.)"""
    xs = (np.asarray(a, dtype=F32) * np.asarray(inv_s, dtype=F32)).astype(F32)
    return nvfp4_tensor_scale(float(np.max(xs)) if xs.size else 0.0)


def prepare_from_factors(W, bias, act_absmax, fmt: str, alpha: float, L1, L2, sigma=None,
                         s_min: float = float(S_MIN), smooth: bool = True) -> Prepared:
    """Offline steps with given (bfloat16) SVD factors: statistics, eq. 2,
    migration (eq. 1), residual R = W_hat - L1 L2 and its 4-bit quantization.
    Rank 0 (L1 [K, 0], L2 [0, N]) is the smoothing-only case: R = W_hat."""
    W = np.asarray(W, dtype=np.float64)
    K, N = W.shape
    w_stat = weight_absmax(W)
    s, inv_s = smoothing_factors(act_absmax, w_stat, alpha, s_min, smooth)
    W_hat = migrate_weight(W, s)
    L1 = np.asarray(L1, dtype=np.float64)
    L2 = np.asarray(L2, dtype=np.float64)
    R = residual(W_hat, L1, L2)
    RT = np.ascontiguousarray(R.T)  # [N, K]: groups of K for each output column
    if fmt == "nvfp4_g16":
        g_w = nvfp4_tensor_scale(float(np.max(np.abs(R))) if R.size else 0.0)
        g_x = static_activation_scale(act_absmax, inv_s)
    else:
        g_w = F32(1.0)
        g_x = F32(1.0)
    codes, scales = quantize_rows(RT, fmt, g_w)
    b = np.zeros(N) if bias is None else np.asarray(bias, dtype=np.float64)
    return Prepared(fmt, K, N, L1.shape[1], alpha, s, inv_s, L1, L2, R, codes, scales, g_w, g_x, b, sigma)


def prepare(W, bias, act_absmax, fmt: str, alpha: float, rank: int, s_min: float = float(S_MIN),
            smooth: bool = True) -> Prepared:
    """The three offline stages of section 2.1 in order: migrate (eq. 1, 2),
    decompose (eq. 3, rank-r truncated SVD), quantize the residual.
    rank = 0 skips the decomposition (smoothing only, the SmoothQuant special
    case the entry's related terms name); smooth=False skips the migration."""
    W = np.asarray(W, dtype=np.float64)
    s, _ = smoothing_factors(act_absmax, weight_absmax(W), alpha, s_min, smooth)
    W_hat = migrate_weight(W, s)
    L1, L2, sigma = svd_factors(W_hat, rank)
    return prepare_from_factors(W, bias, act_absmax, fmt, alpha, L1, L2, sigma, s_min, smooth)


def smooth_activations(X, inv_s) -> np.ndarray:
    """X diag(s)^-1 of eq. 1, one float32 rounding: x_hat = fp32(x * inv_s_k)."""
    return (np.asarray(X, dtype=F32) * np.asarray(inv_s, dtype=F32)[None, :]).astype(F32)


def dequantized_weight(p: Prepared) -> np.ndarray:
    """Q(R) as float64 values [N, K] (computed once per prepared layer)."""
    cached = getattr(p, "_wq", None)
    if cached is None or cached[0] is not p.w_codes:
        cached = (p.w_codes, dequantize(p.w_codes, p.w_scales, p.fmt, p.g_w))
        object.__setattr__(p, "_wq", cached)
    return cached[1]


@dataclass
class ForwardResult:
    Y: np.ndarray  # float64 [M, N], not rounded
    x_codes: np.ndarray  # [M, K]
    x_scales: np.ndarray  # [M, K/G]
    T: np.ndarray  # float64 [M, r]: x_hat L1
    main: np.ndarray  # float64 [M, N]: Q(x_hat) Q(R)


def forward(p: Prepared, X) -> ForwardResult:
    """Eq. 4 of section 2.3 plus the bias:
    Y = Q(X diag(s)^-1) Q(R) + (X diag(s)^-1 L1) L2 + b, all sums in float64.

    The 4-bit product is the plain product of the dequantized operands: for
    INT4, sum_g sx[m,g] sw[n,g] sum_{k in g} qx qw; for NVFP4 the block
    scales and both tensor scales multiply the E2M1 values likewise.
    """
    x_hat = smooth_activations(X, p.inv_s)
    x_codes, x_scales = quantize_rows(x_hat, p.fmt, p.g_x)
    xq = dequantize(x_codes, x_scales, p.fmt, p.g_x)
    main = xq @ dequantized_weight(p).T
    T = x_hat.astype(np.float64) @ p.L1
    Y = main + T @ p.L2 + p.bias[None, :]
    return ForwardResult(Y, x_codes, x_scales, T, main)


def forward_unquantized(p: Prepared, X) -> np.ndarray:
    """The dual path with Q(.) the identity: x_hat R + (x_hat L1) L2 + b.
    Section 2.4 ("mathematical equivalence") says this equals X W + b."""
    x_hat = smooth_activations(X, p.inv_s).astype(np.float64)
    return x_hat @ p.R.astype(np.float64) + (x_hat @ p.L1) @ p.L2 + p.bias[None, :]


def attach_lora(p: Prepared, A, B, scale: float) -> Prepared:
    """Adds a LoRA X A B * scale to the low-rank branch without touching R
    (abstract: off-the-shelf LoRAs without re-quantization).

    The branch sees x_hat = X diag(s)^-1, so X A = x_hat (diag(s) A):
    L1' = [L1 | bf16(diag(s) A)], L2' = [L2 ; bf16(scale B)] (each product is
    exact in float64 and rounded once to bfloat16)."""
    sA, sB = lora_factors(p, A, B, scale)
    L1 = np.concatenate([p.L1, sA], axis=1)
    L2 = np.concatenate([p.L2, sB], axis=0)
    return dataclasses.replace(p, L1=L1, L2=L2, rank=L1.shape[1])


def lora_factors(p: Prepared, A, B, scale: float):
    """An adapter's branch factors: F = bf16(diag(s) A) [K, r_l] and
    G = bf16(scale B) [r_l, N] (the branch sees x_hat = X diag(s)^-1)."""
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    F = bf16_round(p.s.astype(np.float64)[:, None] * A)
    G = bf16_round(np.float64(F32(scale)) * B)
    return F, G


def forward_selected(p: Prepared, adapters: dict, X, row_mask) -> np.ndarray:
    """Per-row adapter selection: row m of the output is the layer's output
    plus, for every adapter slot a set in row_mask[m], that adapter's branch
    product (x_hat F_a) G_a. `adapters` maps slot -> (F, G) from lora_factors;
    p is the layer without adapters. All sums in float64."""
    x_hat = smooth_activations(X, p.inv_s).astype(np.float64)
    Y = forward(p, X).Y.copy()
    mask = np.asarray(row_mask, dtype=np.int64)
    for slot, (F, G) in adapters.items():
        sel = ((mask >> slot) & 1).astype(bool)
        if np.any(sel):
            Y[sel] += (x_hat[sel] @ F) @ G
    return Y


# ---------------------------------------------------------------------------
# the 4-bit weight-only baseline (W4A16) of the abstract's speed comparison
# ---------------------------------------------------------------------------

@dataclass
class WeightOnly:
    """W quantized alone (no smoothing, no branch): INT4 group 64 per output column."""

    K: int
    N: int
    codes: np.ndarray  # int8 [N, K]
    scales: np.ndarray  # float32 [N, K/64]
    bias: np.ndarray  # float64 holding bf16 values [N]


def prepare_weight_only(W, bias) -> WeightOnly:
    """The weight-only baseline's offline step: the same symmetric INT4 group-64
    quantizer as the W4A4 layer, applied to W itself, per output column."""
    W = np.asarray(W, dtype=np.float64)
    K, N = W.shape
    codes, scales = quantize_int4_g64(np.ascontiguousarray(W.T).astype(F32))
    b = np.zeros(N) if bias is None else np.asarray(bias, dtype=np.float64)
    return WeightOnly(K, N, codes, scales, b)


def dequantize_weight_only(p: WeightOnly) -> np.ndarray:
    """w[n, k] = bf16(fp32(q[n, k] * scale[n, k / 64])): the bf16 operand the
    activations meet (one float32 rounding of the product, then bf16)."""
    q = p.codes.astype(F32).reshape(p.N, p.K // 64, 64)
    prod = (q * p.scales.astype(F32)[:, :, None]).astype(F32)
    return bf16_round(prod.reshape(p.N, p.K).astype(np.float64))


def forward_weight_only(p: WeightOnly, X) -> np.ndarray:
    """Y = X w^T + b in float64 with X in bf16 (the activations stay 16-bit)."""
    return np.asarray(X, dtype=np.float64) @ dequantize_weight_only(p).T + p.bias[None, :]


# ---------------------------------------------------------------------------
# the MLP block: up layer, GELU, down layer
# ---------------------------------------------------------------------------

def gelu_erf(x) -> np.ndarray:
    """GELU(x) = x * Phi(x) = 0.5 x (1 + erf(x / sqrt 2)) in float64 (the exact
    form; scipy's erf is the library step)."""
    from scipy.special import erf
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


@dataclass
class MlpResult:
    y_up: np.ndarray  # float64 holding bf16 values [M, N_up]: the up layer's stored output
    h: np.ndarray  # float64 holding bf16 values [M, N_up]: GELU(y_up), the down layer's input
    down: ForwardResult  # the down layer's forward on h


def mlp_forward(p_up: Prepared, p_down: Prepared, X) -> MlpResult:
    """An MLP block of two SVDQuant layers: Y = down(GELU(up(X))). Each tensor
    between the layers is held in bf16, as a plain composition of the layers
    would store it: the up layer's output is rounded to bf16, GELU is applied
    to that and rounded to bf16, and the down layer runs on the result."""
    y_up = bf16_round(forward(p_up, X).Y)
    h = bf16_round(gelu_erf(y_up))
    return MlpResult(y_up, h, forward(p_down, h))
