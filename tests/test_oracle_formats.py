"""Pins of the oracle's number formats and group quantizers (CPU only).

Each check compares the oracle with something other than itself: the
published value tables (tests/golden), brute force over every code, torch's
own float32 -> bfloat16 conversion, and hand-worked examples.
"""
import numpy as np
import pytest
import torch

from oracle import formats as F

F32 = np.float32


def _e2m1_brute(x):
    """Nearest E2M1 value by scanning all 16 codes; ties to the even code."""
    best = None
    for code in range(16):
        mag = [0, 0.5, 1, 1.5, 2, 3, 4, 6][code & 7]
        val = -mag if code & 8 else mag
        if (code & 8) != (8 if np.signbit(x) else 0):
            continue
        d = abs(float(x) - val)
        key = (d, code & 1)
        if best is None or key < best[0]:
            best = (key, code)
    # saturation: beyond 6 the largest magnitude
    if abs(x) >= 6:
        return 0xF if np.signbit(x) else 0x7
    return best[1]


def test_e2m1_table_matches_spec(golden):
    for code, val in golden("e2m1_values.txt"):
        c = int(code, 16)
        assert F.e2m1_decode(c) == float(val)
        assert F.e2m1_encode(float(val)) == c or float(val) == 0.0


def test_e4m3_table_matches_spec(golden):
    for code, val in golden("e4m3_values.txt"):
        c = int(code, 16)
        d = F.e4m3_decode(c)
        assert d == float(val) and np.signbit(d) == np.signbit(float(val))
        assert F.e4m3_encode(float(val)) == c
    assert F.E4M3_MAX == 448.0
    assert np.isnan(F.e4m3_decode(0x7F)) and np.isnan(F.e4m3_decode(0xFF))
    # 126 nonzero finite positive values plus zero
    assert len(F.E4M3_VALUES) == 127 and np.all(np.diff(F.E4M3_VALUES) > 0)


def test_e2m1_encode_brute_force():
    rng = np.random.default_rng(1)
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    xs = list(rng.uniform(-8, 8, 3000).astype(F32))
    for m in mids + [0.0, 6.0, 7.0, 1e9]:
        for s in (1.0, -1.0):
            xs += [F32(s * m), np.nextafter(F32(s * m), F32(0)), np.nextafter(F32(s * m), F32(s * 100))]
    xs = np.array(xs, dtype=F32)
    enc = F.e2m1_encode(xs)
    for x, c in zip(xs, enc):
        assert c == _e2m1_brute(x), (x, c)


def test_e4m3_encode_brute_force():
    rng = np.random.default_rng(2)
    pos = F.E4M3_VALUES
    mids = (pos[:-1] + pos[1:]) / 2
    xs = np.concatenate([
        rng.uniform(0, 500, 4000), np.exp(rng.uniform(-14, 6, 4000)), mids,
        np.nextafter(mids, 0), np.nextafter(mids, 1e9), pos,
    ]).astype(F32)
    enc = F.e4m3_encode(xs)
    allv = np.array([F.e4m3_decode(c) for c in range(127)])
    for x, c in zip(xs, enc):
        if x >= 448:
            assert c == 0x7E
            continue
        d = np.abs(allv - float(x))
        cands = np.flatnonzero(d == d.min())
        want = cands[0] if len(cands) == 1 else [k for k in cands if k % 2 == 0][0]
        assert c == want, (x, c, want)
    # round trip of every finite value
    assert np.all(F.e4m3_decode(F.e4m3_encode(pos)) == pos)


def test_bf16_round_matches_torch_for_float32_inputs():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                        rng.standard_normal(1000) * 1e-39]).astype(F32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = F.bf16_round(x.astype(np.float64))
    assert np.array_equal(got, want)


def test_bf16_round_has_no_double_rounding():
    # 1 + 2^-8 + 2^-30 is just above the midpoint between 1 and 1 + 2^-7.
    # Through float32 it would become the midpoint 1 + 2^-8 and tie to 1.
    x = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert F.bf16_round(x) == 1.0 + 2.0 ** -7
    assert F.bf16_round(1.0 + 2.0 ** -8) == 1.0  # exact tie -> even
    assert F.bf16_round(1.0 + 3 * 2.0 ** -8) == 1.0 + 2 * 2.0 ** -7  # tie -> even (up)


def _int4_brute(v_row):
    amax = np.max(np.abs(v_row)).astype(F32)
    if amax == 0:
        return np.zeros(64, np.int8), F32(0)
    inv = F32(F32(7.0) / amax)
    out = []
    for v in v_row:
        t = float(F32(F32(v) * inv))
        best = min(range(-8, 8), key=lambda q: (abs(t - q), q % 2))
        out.append(best)
    return np.array(out, np.int8), F32(amax / F32(7.0))


def test_int4_quantizer_brute_force():
    rng = np.random.default_rng(4)
    v = (rng.standard_normal((40, 256)) * rng.uniform(0.01, 100, (40, 1))).astype(F32)
    v[3, :64] = 0.0  # an all-zero group
    v[5, 70] = 1e4  # a dominant outlier
    codes, scales = F.quantize_int4_g64(v)
    for i in range(v.shape[0]):
        for g in range(4):
            q, s = _int4_brute(v[i, 64 * g:64 * (g + 1)])
            assert np.array_equal(codes[i, 64 * g:64 * (g + 1)], q)
            assert scales[i, g] == s
    # reconstruction error at most half a step (plus float32 rounding)
    dq = F.dequantize(codes, scales, "int4_g64")
    step = np.repeat(scales, 64, axis=1).astype(np.float64)
    assert np.all(np.abs(dq - v) <= 0.5 * step * (1 + 1e-6) + 1e-30)


def test_int4_worked_example(golden):
    rows = golden("int4_g64_worked.txt")
    groups = []
    for r in rows:
        if r[0] == "group":
            groups.append((float(r[3]), float(r[5]), []))
        else:
            groups[-1][2].append((float(r[0]), int(r[1])))
    for amax, scale, pairs in groups:
        v = np.zeros(64, F32)
        want = np.zeros(64, np.int8)
        for i, (x, q) in enumerate(pairs):
            v[i] = x
            want[i] = q
        codes, scales = F.quantize_int4_g64(v[None, :])
        assert np.array_equal(codes[0], want)
        assert scales[0, 0] == F32(scale)


def test_nvfp4_worked_example(golden):
    rows = golden("nvfp4_g16_worked.txt")
    blocks = []
    for r in rows:
        if r[0] == "block":
            blocks.append((float(r[3]), int(r[5], 16), []))
        else:
            blocks[-1][2].append((float(r[0]), int(r[1], 16)))
    for g, sb, pairs in blocks:
        v = np.zeros(16, F32)
        want = np.zeros(16, np.uint8)
        for i, (x, c) in enumerate(pairs):
            v[i] = x
            want[i] = c
        codes, scales = F.quantize_nvfp4_g16(v[None, :], F32(g))
        assert scales[0, 0] == sb
        assert np.array_equal(codes[0], want), (codes[0], want)


def test_nvfp4_error_bound_and_tensor_scale():
    rng = np.random.default_rng(5)
    v = (rng.standard_normal((64, 512)) * 3).astype(F32)
    v[0, 0] = 250.0
    g = F.nvfp4_tensor_scale(float(np.max(np.abs(v))))
    assert g == F32(F32(250.0) / F32(2688.0))
    codes, sb = F.quantize_nvfp4_g16(v, g)
    dq = F.dequantize(codes, sb, "nvfp4_g16", g)
    eff = np.repeat(F.e4m3_decode(sb) * float(g), 16, axis=1)
    # |error| at most half the widest E2M1 spacing (2, between 4 and 6) times eff,
    # and the block maximum is within a relative 2^-4 (E4M3 scale rounding) of 6 * eff
    assert np.all(np.abs(dq - v) <= eff * 1.0 + 1e-12)
    amax = np.max(np.abs(v.reshape(64, 32, 16)), axis=-1)
    assert np.all(amax <= F.e4m3_decode(sb) * float(g) * 6 * (1 + 2 ** -4) + 1e-12)
    assert F.nvfp4_tensor_scale(0.0) == 1.0


def test_nvfp4_zero_scale_block_gives_zero_codes():
    g = F32(1.0)
    v = np.zeros((1, 16), F32)
    v[0, 0] = 1e-6  # amax / 6 rounds to E4M3 zero
    codes, sb = F.quantize_nvfp4_g16(v, g)
    assert sb[0, 0] == 0 and np.all(codes == 0)


def test_nibble_packing_round_trip():
    rng = np.random.default_rng(6)
    q = rng.integers(-8, 8, (7, 64)).astype(np.int8)
    p = F.pack_nibbles(q)
    assert p.shape == (7, 32)
    assert np.all((p[:, 0] & 0xF) == (q[:, 0] & 0xF)) and np.all((p[:, 0] >> 4) == (q[:, 1] & 0xF))
    assert np.array_equal(F.unpack_nibbles(p, signed=True), q)
