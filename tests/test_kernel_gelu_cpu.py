"""The fused MLP epilogue's GELU, emulated on the CPU over every bf16 input.

The up GEMM of the MLP block applies GELU (the erf form; "SVDQuant", abstract:
the block's activation between its two linear layers) to the bf16 up output in
float32: with u = |y| sqrt(log2(e) / 2), erfc(|y| / sqrt 2) / 2 = 2^(-u^2) q(u)
for a fitted polynomial q. This test reads the polynomial, the scale of u and
its clamp from the kernel source and replays the kernel's arithmetic in
float32 (each packed multiply-add rounded once), so that a change to the
constants is checked before it reaches a GPU. It pins two properties the GPU
MLP tests rely on:

- the error bound the interval checks of the down layer's codes assume,
  |GELU_kernel(y) - GELU(y)| <= 1e-6 |y| + 2^-21 |GELU(y)|, with the
  exponential exact and with it off by 2^-22 relative either way (a margin
  for the hardware's approximate exp2);
- the sign: GELU(y) has the sign of y for every y (zeros included), so a
  value that quantizes to a zero code gets the oracle's signed zero. A fit
  whose polynomial changes sign inside the clamp breaks this for negative y
  while still meeting the error bound.
"""
import os
import re

import numpy as np
from scipy.special import erfc

F32 = np.float32
E_GELU_Y = 1e-6
E_GELU_G = 2.0 ** -21
SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "rank_gemm_quantize_b200", "csrc", "gemm_nvfp4.cu")


def _kernel_constants():
    src = open(SRC).read()
    body = src[src.index("uint32_t gelu_bf16x2"):src.index("return pack_bf16x2(g.x, g.y);")]
    num = r"([-0-9.e+]+)f"
    lead = F32(float(re.search(r"float2 q = make_float2\(" + num, body).group(1)))
    rest = [F32(float(m)) for m in re.findall(r"__ffma2_rn\(q, u, make_float2\(" + num, body)]
    scale = F32(float(re.search(r"float2 u = __fmul2_rn\([^;]*make_float2\(" + num, body, re.S).group(1)))
    clamp = F32(float(re.search(r"u\.x = fminf\(u\.x, " + num, body).group(1)))
    return [lead] + rest, scale, clamp


def _fma(a, b, c):
    # float32 operands: the float64 product is exact; one rounding of the sum to float32
    return (np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.asarray(c, np.float64)).astype(F32)


def _all_bf16():
    bits = np.arange(65536, dtype=np.uint32)
    y = (bits << 16).view(F32)
    return y[np.isfinite(y)]


def _kernel_gelu(y, exp_rel=0.0):
    coeffs, scale, clamp = _kernel_constants()
    u = np.minimum((np.abs(y) * scale).astype(F32), clamp)
    q = np.full_like(u, coeffs[0])
    for c in coeffs[1:]:
        q = _fma(q, u, c)
    uu = (u * u).astype(F32)
    e = (np.exp2(-uu.astype(np.float64)) * (1.0 + exp_rel)).astype(F32)
    hc = (e * q).astype(F32)  # erfc(x) / 2
    om = _fma(hc, F32(-1), F32(1))  # 1 - erfc(x) / 2
    t = np.where(np.signbit(y), hc, om)
    return (y * t).astype(F32), q


def _gelu_exact(y):
    yd = np.asarray(y, np.float64)
    half_erfc = 0.5 * erfc(np.abs(yd) / np.sqrt(2.0))
    return yd * np.where(yd >= 0, 1.0 - half_erfc, half_erfc)


def test_kernel_gelu_error_bound():
    y = _all_bf16()
    exact = _gelu_exact(y)
    bound = E_GELU_Y * np.abs(y.astype(np.float64)) + E_GELU_G * np.abs(exact)
    for exp_rel in (0.0, 2.0 ** -22, -(2.0 ** -22)):
        g, _ = _kernel_gelu(y, exp_rel)
        excess = np.abs(g.astype(np.float64) - exact) - bound
        assert excess.max() <= 0.0, (exp_rel, float(excess.max()), float(y[np.argmax(excess)]))


def test_kernel_gelu_keeps_the_sign():
    y = _all_bf16()
    g, q = _kernel_gelu(y)
    assert np.all(q > 0), "q(u) changes sign inside the clamp"
    assert np.array_equal(np.signbit(g), np.signbit(y))
    # -0 stays -0, +0 stays +0
    g0, _ = _kernel_gelu(np.array([0.0, -0.0], dtype=F32))
    assert not np.signbit(g0[0]) and np.signbit(g0[1]) and np.all(g0 == 0)


def test_emulation_catches_a_sign_changing_fit():
    """The check above is not vacuous: a polynomial that meets the error bound
    but turns negative before the clamp (a fit that ignores the far range)
    makes GELU of large negative y positive."""
    coeffs, scale, clamp = _kernel_constants()
    y = _all_bf16()
    u = np.minimum((np.abs(y) * scale).astype(F32), clamp)
    q = np.full_like(u, coeffs[0])
    for c in coeffs[1:]:
        q = _fma(q, u, c)
    q_bad = np.where(u > F32(5), -q, q).astype(F32)  # negative near the clamp, where 2^(-u^2) hides it
    uu = (u * u).astype(F32)
    hc = (np.exp2(-uu.astype(np.float64)).astype(F32) * q_bad).astype(F32)
    t = np.where(np.signbit(y), hc, _fma(hc, F32(-1), F32(1)))
    g = (y * t).astype(F32)
    assert np.any(np.signbit(g) != np.signbit(y))
    exact = _gelu_exact(y)
    bound = E_GELU_Y * np.abs(y.astype(np.float64)) + E_GELU_G * np.abs(exact)
    assert np.all(np.abs(g.astype(np.float64) - exact) <= bound)  # while the error bound still holds
