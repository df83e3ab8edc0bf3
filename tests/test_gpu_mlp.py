"""The fused MLP block Y = down(GELU(up(X))) against the oracle, on a B200.

The up layer's GEMM epilogue computes GELU and the down layer's smoothing and
NVFP4 quantization itself ("SVDQuant", abstract: the low-rank branch fused
into the low-bit kernels to cut redundant memory access; here across the
block's two layers). The oracle runs the plain composition: the up layer in
float64, its output rounded to bf16, exact-erf GELU rounded to bf16, the
down layer.

The two sides reach h = bf16(GELU(bf16(y))) along different roundings: the
kernel accumulates in float32, carries the up layer's branch input T as a
bf16 pair (T + T_lo, about 16 significant bits) and evaluates erf in float32.
Where y or GELU(y) lies close to a bf16 rounding boundary, h may
legitimately come out one bf16 step apart. So the down layer's codes and
scales are checked against intervals: a bound on the kernel's deviation in y
(from the sums of absolute terms of each product) gives, per element, the
bf16 values y and then h can take; through the smoothing and the group
maximum that gives the range of valid E4M3 scales of each group, and, given
the kernel's scale, the range of valid E2M1 codes of each element. Where the
range holds one value (almost every group and element) the comparison is
exact, bit for bit; elsewhere the kernel's value must lie inside it. T and Y
are compared within the single layer's 2e-3 / 4e-3 normwise bounds.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import formats as F
from oracle import svdquant as S
from parity import T_TOL, Y_TOL, bf16_tensor, f64, rel

pytestmark = pytest.mark.gpu

F32 = np.float32
GELU_ARGMIN = -0.7517915246935645  # GELU is decreasing left of this point, increasing right of it
# |GELU_kernel(y) - GELU(y)| <= E_GELU_Y |y| + E_GELU_G |GELU(y)|: the kernel's erf is within
# about 5e-7 of the exact one (absolute), then float32 products
E_GELU_Y = 1e-6
E_GELU_G = 2.0 ** -21


def _up_output_bound(p, X, fr):
    """Per element, a bound on |y_kernel - y_oracle| for the up layer's output
    before its bf16 rounding: T as a float32 accumulation over K held as a
    bf16 pair (2^-16 relative), float32 accumulation of the 4-bit and branch
    products, the tensor-scale product and the bias; each term with a factor
    of at least 2 to spare."""
    x_hat = S.smooth_activations(X, p.inv_s).astype(np.float64)
    xq = F.dequantize(fr.x_codes, fr.x_scales, p.fmt, p.g_x)
    wq = S.dequantized_weight(p)
    absT = np.abs(fr.T)
    e_T = 2.0 ** -15 * (absT + np.abs(x_hat) @ np.abs(p.L1))
    return (e_T @ np.abs(p.L2)
            + 2.0 ** -15 * (np.abs(xq) @ np.abs(wq).T + absT @ np.abs(p.L2))
            + 2.0 ** -20 * (np.abs(fr.Y) + np.abs(p.bias)[None, :]))


def _h_interval(y, e_y):
    """The bf16 values h = bf16(GELU(bf16(y'))) can take for |y' - y| <= e_y
    and a kernel GELU within the stated error: [h_lo, h_hi]."""
    y_lo, y_hi = F.bf16_round(y - e_y), F.bf16_round(y + e_y)
    g_a, g_b = S.gelu_erf(y_lo), S.gelu_erf(y_hi)
    g_min = np.minimum(g_a, g_b)
    inside = (y_lo < GELU_ARGMIN) & (y_hi > GELU_ARGMIN)
    g_min = np.where(inside, np.minimum(g_min, S.gelu_erf(np.float64(GELU_ARGMIN))), g_min)
    g_max = np.maximum(g_a, g_b)
    e_g = E_GELU_Y * np.maximum(np.abs(y_lo), np.abs(y_hi)) + E_GELU_G * np.maximum(np.abs(g_a), np.abs(g_b))
    return F.bf16_round(g_min - e_g), F.bf16_round(g_max + e_g)


def _check_down_quantization(h_lo, h_hi, p_dn, q_gpu, sc_gpu, q_ref, sc_ref):
    """The kernel's scales and codes of the down layer lie in the ranges that
    [h_lo, h_hi] allows; exact where a range holds one value. Returns the
    decided fractions (scales, codes)."""
    R = h_lo.shape[0]
    inv = np.asarray(p_dn.inv_s, dtype=F32)[None, :]
    x_lo = (h_lo.astype(F32) * inv).astype(F32).reshape(R, -1, 16)
    x_hi = (h_hi.astype(F32) * inv).astype(F32).reshape(R, -1, 16)
    straddle = (x_lo <= 0) & (x_hi >= 0)
    a_lo = np.where(straddle, F32(0), np.minimum(np.abs(x_lo), np.abs(x_hi))).max(axis=-1)
    a_hi = np.maximum(np.abs(x_lo), np.abs(x_hi)).max(axis=-1)
    g = F32(p_dn.g_x)
    denom = F32(F32(6.0) * g)
    sb_lo = F.e4m3_encode((a_lo.astype(F32) / denom).astype(F32)).astype(int)
    sb_hi = F.e4m3_encode((a_hi.astype(F32) / denom).astype(F32)).astype(int)
    assert np.all((sb_lo <= sc_ref) & (sc_ref <= sb_hi)), "the oracle's own scales fall outside the ranges"
    sc = sc_gpu.astype(int)
    bad = ~((sb_lo <= sc) & (sc <= sb_hi))
    assert not bad.any(), f"{bad.sum()} of {bad.size} group scales outside their valid range"
    one = sb_lo == sb_hi
    assert np.array_equal(sc[one], sc_ref[one].astype(int))
    # codes, given the kernel's scale of each group
    eff = (F.e4m3_decode(sc_gpu).astype(F32) * g).astype(F32)
    zero = eff == 0
    inv_e = (F32(1.0) / np.where(zero, F32(1), eff)).astype(F32)[..., None]
    c_lo = np.where(zero[..., None], 0, F.e2m1_encode((x_lo * inv_e).astype(F32)))
    c_hi = np.where(zero[..., None], 0, F.e2m1_encode((x_hi * inv_e).astype(F32)))
    v_lo, v_hi, v = F.e2m1_decode(c_lo), F.e2m1_decode(c_hi), F.e2m1_decode(q_gpu)
    bad = ~((v_lo <= v) & (v <= v_hi))
    assert not bad.any(), f"{bad.sum()} of {bad.size} codes outside their valid range"
    c_one = (c_lo == c_hi) & one[..., None]
    assert np.array_equal(q_gpu[c_one], c_lo[c_one].astype(q_gpu.dtype))
    assert np.array_equal(q_gpu[c_one], q_ref[c_one])  # there the oracle's code is the only valid one
    return one.mean(), c_one.mean()


def _block(M, K, N, Kd_out, seed, up_rank=32):
    rng = np.random.Generator(np.random.PCG64(seed))
    up = workloads.custom(M, K, N, up_rank, workloads.NVFP4_G16, seed=seed)
    Wd = F.bf16_round(rng.normal(0, 0.02, (N, Kd_out)))
    bd = F.bf16_round(rng.normal(0, 0.01, Kd_out))
    return up, Wd, bd


def _run(up, Wd, bd, rows=None, down_rank=32):
    import rank_gemm_quantize_b200 as rq
    X, Wu, bu = workloads.to_f64(up.X), workloads.to_f64(up.W), workloads.to_f64(up.bias)
    a_u = S.calibrate_absmax(X)
    p_up = S.prepare(Wu, bu, a_u, up.fmt, 0.5, up.rank)
    # the down layer is calibrated on the oracle's h of the whole batch (both sides use this statistic)
    y_up_all = F.bf16_round(S.forward(p_up, X).Y)
    h_all = F.bf16_round(S.gelu_erf(y_up_all))
    a_d = S.calibrate_absmax(h_all)
    p_dn = S.prepare(Wd, bd, a_d, up.fmt, 0.5, down_rank)
    g_up = rq.Layer.prepare(up.W.cuda(), up.bias.cuda(), torch.from_numpy(a_u).cuda(), up.fmt, up.rank,
                            factors=(bf16_tensor(p_up.L1), bf16_tensor(p_up.L2)))
    g_dn = rq.Layer.prepare(bf16_tensor(Wd), bf16_tensor(bd), torch.from_numpy(a_d).cuda(), up.fmt, down_rank,
                            factors=(bf16_tensor(p_dn.L1), bf16_tensor(p_dn.L2)))
    try:
        blk = rq.MlpBlock(g_up, g_dn)
        ws = blk.workspace(up.M)
        Y = blk.forward(up.X.cuda(), workspace=ws)
        torch.cuda.synchronize()
        off = blk.workspace_layout(up.M)
        M_pad = (up.M + 127) // 128 * 128
        Kd = Wd.shape[0]
        wsn = ws.cpu().numpy()
        codes = wsn[off[0]:off[0] + M_pad * Kd // 2].reshape(M_pad, Kd // 2)
        atoms = wsn[off[1]:off[1] + M_pad // 128 * (Kd // 64) * 512]
        T = wsn[off[2]:off[2] + M_pad * 32 * 2].view(np.uint16).reshape(M_pad, 32)
        T = (T.astype(np.uint32) << 16).view(np.float32).astype(np.float64) / np.float64(np.float32(g_dn.info().t_scale))
        y = f64(Y)
        assert g_up.device_status() == 0 and g_dn.device_status() == 0
    finally:
        g_up.close()
        g_dn.close()
    r = np.arange(up.M) if rows is None else rows
    res = S.mlp_forward(p_up, p_dn, X[r])
    fr_up = S.forward(p_up, X[r])
    h_lo, h_hi = _h_interval(fr_up.Y, _up_output_bound(p_up, X[r], fr_up))
    assert np.all((h_lo <= res.h) & (res.h <= h_hi))
    q = F.unpack_nibbles(codes[r], signed=False)
    m = np.asarray(r)[:, None]
    i = np.arange(Kd // 16)[None, :]
    sc = atoms[((m // 128) * (Kd // 64) + i // 4) * 512 + (m % 32) * 16 + ((m // 32) % 4) * 4 + i % 4]
    qg = q.reshape(len(r), -1, 16)
    wg = res.down.x_codes.reshape(len(r), -1, 16)
    s_one, c_one = _check_down_quantization(h_lo, h_hi, p_dn, qg, sc, wg, res.down.x_scales)
    # the bound is worst-case, so the exact comparison covers most but not all of the tensor
    # (scales 99-99.5 %, codes 91-97 % on the small shapes and 73 % on the FLUX block) ...
    if sc.size >= 1000:
        assert s_one > 0.95 and c_one > 0.6, (s_one, c_one)
    # ... while the kernel's typical deviation is far smaller: nearly every scale and code is the
    # oracle's own (over 99.99 % when T is a bf16 pair and everything else is exact)
    assert (sc != res.down.x_scales).sum() <= max(1, 0.005 * sc.size)
    assert (qg != wg).sum() <= max(1, 0.005 * qg.size)
    assert rel(T[r][:, :down_rank], res.down.T) <= T_TOL
    assert np.all(T[r][:, down_rank:] == 0)  # the branch's padding columns
    assert rel(y[r], res.down.Y) <= Y_TOL
    return s_one, c_one


@pytest.mark.parametrize("M,K,N,Kd_out,seed", [(200, 512, 512, 256, 121), (384, 256, 1024, 512, 122)])
def test_fused_mlp_block_small(M, K, N, Kd_out, seed):
    up, Wd, bd = _block(M, K, N, Kd_out, seed)
    _run(up, Wd, bd)


@pytest.mark.parametrize("M,K,N,Kd_out,seed,up_rank,down_rank", [
    (1, 256, 512, 256, 126, 32, 32),      # a single row
    (300, 384, 768, 512, 127, 32, 32),    # ragged M (not a multiple of 128 or 256), three column blocks
    (256, 256, 512, 256, 128, 0, 32),     # up layer of rank 0: no branch, no T low part
    (256, 512, 512, 256, 129, 16, 8),     # narrower branches on both layers
])
def test_fused_mlp_block_edge_shapes(M, K, N, Kd_out, seed, up_rank, down_rank):
    up, Wd, bd = _block(M, K, N, Kd_out, seed, up_rank=up_rank)
    _run(up, Wd, bd, down_rank=down_rank)


def test_fused_mlp_block_flux_shape():
    """The FLUX MLP block at full size (4608 x 3072 -> 12288 -> 3072), checked
    on a seeded sample of 512 rows (every layer is row-local)."""
    up = workloads.config(3)[0]
    rng = np.random.Generator(np.random.PCG64(123))
    Wd = F.bf16_round(rng.normal(0, 0.02, (12288, 3072)))
    bd = F.bf16_round(rng.normal(0, 0.01, 3072))
    rows = np.sort(np.random.Generator(np.random.PCG64(124)).choice(up.M, 512, replace=False))
    _run(up, Wd, bd, rows)


def test_fused_mlp_refuses_unsupported_pairs():
    import rank_gemm_quantize_b200 as rq
    a = workloads.custom(128, 256, 256, 8, workloads.INT4_G64, seed=125)
    g1 = rq.Layer.prepare(a.W.cuda(), a.bias.cuda(), torch.ones(256, device="cuda"), a.fmt, 8)
    g2 = rq.Layer.prepare(a.W.cuda(), a.bias.cuda(), torch.ones(256, device="cuda"), a.fmt, 8)
    try:
        with pytest.raises(rq.SvdqError) as e:
            rq.MlpBlock(g1, g2).workspace_size(128)
        assert e.value.status == rq.Status.UNSUPPORTED
    finally:
        g1.close()
        g2.close()
