"""Number formats and group quantizers of the oracle (test infrastructure).

Only tests, the smoke check and the benchmark's CPU baseline may import this.

The SVDQuant pages say only that weights and activations are quantized to
4 bits per group (abstract of arXiv 2411.05007; "Linear Quantization" as the
companion term of the msModelSlim entry, section 3). The concrete formats
follow published definitions:

* E2M1 (FP4): OCP Microscaling Formats (MX) v1.0, section 5.3.3 - one sign
  bit, two exponent bits (bias 1), one mantissa bit; magnitudes
  {0, 0.5, 1, 1.5, 2, 3, 4, 6}; no infinities or NaN.
* E4M3 (FP8): "FP8 Formats for Deep Learning" (Micikevicius et al. 2022),
  table 1 - one sign bit, four exponent bits (bias 7), three mantissa bits,
  subnormals, no infinities, S.1111.111 is NaN, largest finite 448.
* bfloat16: 8 exponent bits, 7 stored mantissa bits (8 significant bits).

Conversions round to nearest, ties to even, and saturate to the largest
finite magnitude ("satfinite"). Signs are kept, so a negative value that
rounds to zero encodes as negative zero (E2M1 code 0x8) - a reading; the
pages are silent on it.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32


def _e2m1_magnitudes() -> np.ndarray:
    vals = []
    for code in range(8):
        e, m = code >> 1, code & 1
        if e == 0:
            vals.append(m * 0.5)  # subnormal: m/2 * 2^(1-1)
        else:
            vals.append((1.0 + m / 2.0) * 2.0 ** (e - 1))
    return np.array(vals, dtype=np.float64)


def _e4m3_magnitudes() -> np.ndarray:
    vals = []
    for code in range(127):  # 0x7F (S.1111.111) is NaN and excluded
        e, m = code >> 3, code & 7
        if e == 0:
            vals.append(m / 8.0 * 2.0 ** -6)
        else:
            vals.append((1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(vals, dtype=np.float64)


E2M1_VALUES = _e2m1_magnitudes()  # index = 3-bit magnitude code
E4M3_VALUES = _e4m3_magnitudes()  # index = 7-bit magnitude code
E2M1_MAX = float(E2M1_VALUES[-1])  # 6
E4M3_MAX = float(E4M3_VALUES[-1])  # 448


def _encode_magnitude(mag: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Nearest entry of an ascending table, ties to the even code, saturating."""
    mag = np.asarray(mag, dtype=np.float64)
    hi = np.searchsorted(table, mag, side="left")
    hi = np.clip(hi, 0, len(table) - 1)
    lo = np.clip(hi - 1, 0, len(table) - 1)
    d_lo = np.abs(mag - table[lo])
    d_hi = np.abs(table[hi] - mag)
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(mag >= table[-1], len(table) - 1, code)
    return code.astype(np.int64)


def e2m1_encode(x) -> np.ndarray:
    """float32/float64 values -> 4-bit E2M1 codes (uint8, sign in bit 3)."""
    x = np.asarray(x, dtype=np.float64)
    code = _encode_magnitude(np.abs(x), E2M1_VALUES)
    sign = np.signbit(x).astype(np.int64) << 3
    return (code | sign).astype(np.uint8)


def e2m1_decode(code) -> np.ndarray:
    code = np.asarray(code, dtype=np.int64)
    mag = E2M1_VALUES[code & 7]
    return np.where(code & 8, -mag, mag)


def e4m3_encode(x) -> np.ndarray:
    """Values -> E4M3 bytes (uint8), round to nearest even, satfinite."""
    x = np.asarray(x, dtype=np.float64)
    code = _encode_magnitude(np.abs(x), E4M3_VALUES)
    sign = np.signbit(x).astype(np.int64) << 7
    return (code | sign).astype(np.uint8)


def e4m3_decode(code) -> np.ndarray:
    code = np.asarray(code, dtype=np.int64)
    mag = E4M3_VALUES[np.minimum(code & 0x7F, 126)]
    mag = np.where((code & 0x7F) == 0x7F, np.nan, mag)
    return np.where(code & 0x80, -mag, mag)


def bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value (ties to even).

    Done directly from float64 (no intermediate float32, hence no double
    rounding): a value in [2^(e-1), 2^e) has 8 significant bits, so its unit
    in the last place is 2^(e-8); below the smallest normal 2^-126 the unit
    stays 2^-133 (subnormals).
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    ulp_exp = np.maximum(e - 8, -133)
    r = np.rint(np.ldexp(x, -ulp_exp))
    out = np.ldexp(r, ulp_exp)
    big = np.abs(out) > 3.3895313892515355e38
    return np.where(big, np.copysign(np.inf, x), out)


# ---------------------------------------------------------------------------
# group quantizers (one row = one vector along K; groups of G consecutive k)
# ---------------------------------------------------------------------------

def quantize_int4_g64(v: np.ndarray):
    """Symmetric INT4 per group of 64 along the last axis.

    scale = amax / 7 (float32), codes q = clamp(rint(v * (7 / amax)), -8, 7)
    with round half to even, and scale = 0, q = 0 for an all-zero group.
    Codes stay in [-7, 7] in practice; -8 is a guard only.
    Returns (codes int8 [..., K], scales float32 [..., K/64]).
    """
    v = np.asarray(v, dtype=F32)
    *lead, K = v.shape
    if K % 64:
        raise ValueError("K must be a multiple of 64")
    g = v.reshape(*lead, K // 64, 64)
    amax = np.max(np.abs(g), axis=-1)
    zero = amax == 0
    safe = np.where(zero, F32(1), amax).astype(F32)
    scale = np.where(zero, F32(0), safe / F32(7.0)).astype(F32)
    inv = (F32(7.0) / safe).astype(F32)
    prod = (g * inv[..., None]).astype(F32)
    q = np.clip(np.rint(prod), -8, 7)
    q = np.where(zero[..., None], 0, q)
    return q.astype(np.int8).reshape(*lead, K), scale


def nvfp4_tensor_scale(amax_tensor: float) -> np.float32:
    """Per-tensor NVFP4 scale g = amax / (6 * 448) in float32 (1 for amax = 0)."""
    a = F32(amax_tensor)
    if a == 0:
        return F32(1.0)
    return F32(a / F32(2688.0))


def quantize_nvfp4_g16(v: np.ndarray, g: np.float32):
    """NVFP4 per group of 16 along the last axis with tensor scale g.

    sb = E4M3(amax_blk / (6 g)); eff = decode(sb) * g; q = E2M1(v * (1/eff));
    all-zero codes for a block whose eff is 0.
    Returns (codes uint8 E2M1 [..., K], scale bytes uint8 E4M3 [..., K/16]).
    """
    v = np.asarray(v, dtype=F32)
    *lead, K = v.shape
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    g = F32(g)
    blk = v.reshape(*lead, K // 16, 16)
    amax = np.max(np.abs(blk), axis=-1).astype(F32)
    denom = F32(F32(6.0) * g)
    sb = e4m3_encode((amax / denom).astype(F32))
    eff = (e4m3_decode(sb).astype(F32) * g).astype(F32)
    zero = eff == 0
    inv = (F32(1.0) / np.where(zero, F32(1), eff)).astype(F32)
    prod = (blk * inv[..., None]).astype(F32)
    q = e2m1_encode(prod)
    q = np.where(zero[..., None], np.uint8(0), q)
    return q.astype(np.uint8).reshape(*lead, K), sb


def dequantize(codes: np.ndarray, scales: np.ndarray, fmt: str, g: float = 1.0) -> np.ndarray:
    """Codes and group scales -> float64 values (exact products)."""
    *lead, K = codes.shape
    if fmt == "int4_g64":
        G = 64
        vals = codes.astype(np.float64)
        s = scales.astype(np.float64)
    elif fmt == "nvfp4_g16":
        G = 16
        vals = e2m1_decode(codes)
        s = e4m3_decode(scales) * np.float64(F32(g))
    else:
        raise ValueError(fmt)
    out = vals.reshape(*lead, K // G, G) * s[..., None]
    return out.reshape(*lead, K)


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte: element 2j in bits 3:0, element 2j+1 in bits 7:4."""
    c = (np.asarray(codes).astype(np.int64) & 0xF).astype(np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray, signed: bool) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    lo = p & 0xF
    hi = p >> 4
    out = np.stack([lo, hi], axis=-1).reshape(*p.shape[:-1], p.shape[-1] * 2)
    if signed:
        out = np.where(out >= 8, out.astype(np.int16) - 16, out).astype(np.int8)
    return out
