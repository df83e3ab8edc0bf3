"""The fused MLP block Y = down(GELU(up(X))) against the oracle, on a B200.

The up layer's GEMM epilogue computes GELU and the down layer's smoothing and
NVFP4 quantization itself ("SVDQuant", abstract: the low-rank branch fused
into the low-bit kernels to cut redundant memory access; here across the
block's two layers). The oracle runs the plain composition: the up layer in
float64, its output rounded to bf16, exact-erf GELU rounded to bf16, the
down layer.

The two sides compute the up layer's output in different precisions (float32
tensor-core accumulation vs float64) and GELU with different erf routines, so
h = bf16(GELU(bf16(y))) can legitimately differ by one bf16 unit where a value
sits on a rounding boundary. The down layer's codes and scales are therefore
compared bit for bit on every quantization group whose sixteen h values are
decided: the oracle's float64 y lies farther than a margin from a bf16
rounding boundary, and so does its exact GELU value. Every other group is
checked for validity (scale within one E4M3 step, codes within one E2M1
step). T and Y are compared within the usual 2e-3 / 4e-3 normwise bounds.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import formats as F
from oracle import svdquant as S
from parity import T_TOL, Y_TOL, bf16_tensor, f64, rel

pytestmark = pytest.mark.gpu

Y_MARGIN = 2e-5    # relative: float32 accumulation of the up GEMM against float64
G_MARGIN = 2e-6    # relative: float32 erf-GELU against the exact one


def _far_from_bf16_boundary(x, margin):
    """|x| is farther than margin * |x| from the midpoint between its two
    neighbouring bf16 values (so any estimate within that margin rounds alike)."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    ulp = np.ldexp(1.0, np.maximum(e - 8, -133))
    frac = np.abs(x) / ulp - np.floor(np.abs(x) / ulp)
    dist = np.abs(frac - 0.5) * ulp
    return dist > margin * np.abs(x) + 1e-30


def _block(M, K, N, Kd_out, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    up = workloads.custom(M, K, N, 32, workloads.NVFP4_G16, seed=seed)
    Wd = F.bf16_round(rng.normal(0, 0.02, (N, Kd_out)))
    bd = F.bf16_round(rng.normal(0, 0.01, Kd_out))
    return up, Wd, bd


def _run(up, Wd, bd, rows=None):
    import rank_gemm_quantize_b200 as rq
    X, Wu, bu = workloads.to_f64(up.X), workloads.to_f64(up.W), workloads.to_f64(up.bias)
    a_u = S.calibrate_absmax(X)
    p_up = S.prepare(Wu, bu, a_u, up.fmt, 0.5, up.rank)
    # the down layer is calibrated on the oracle's h of the whole batch (both sides use this statistic)
    y_up_all = F.bf16_round(S.forward(p_up, X).Y)
    h_all = F.bf16_round(S.gelu_erf(y_up_all))
    a_d = S.calibrate_absmax(h_all)
    p_dn = S.prepare(Wd, bd, a_d, up.fmt, 0.5, 32)
    g_up = rq.Layer.prepare(up.W.cuda(), up.bias.cuda(), torch.from_numpy(a_u).cuda(), up.fmt, up.rank,
                            factors=(bf16_tensor(p_up.L1), bf16_tensor(p_up.L2)))
    g_dn = rq.Layer.prepare(bf16_tensor(Wd), bf16_tensor(bd), torch.from_numpy(a_d).cuda(), up.fmt, 32,
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
    # y_up of the oracle before rounding, for the decidability margin
    y_exact = S.forward(p_up, X[r]).Y
    decided_y = _far_from_bf16_boundary(y_exact, Y_MARGIN)
    decided_g = _far_from_bf16_boundary(S.gelu_erf(res.y_up), G_MARGIN)
    decided = (decided_y & decided_g).reshape(len(r), -1, 16).all(axis=-1)  # per group of 16
    q = F.unpack_nibbles(codes[r], signed=False)
    m = np.asarray(r)[:, None]
    i = np.arange(Kd // 16)[None, :]
    sc = atoms[((m // 128) * (Kd // 64) + i // 4) * 512 + (m % 32) * 16 + ((m // 32) % 4) * 4 + i % 4]
    want_q, want_s = res.down.x_codes, res.down.x_scales
    qg = q.reshape(len(r), -1, 16)
    wg = want_q.reshape(len(r), -1, 16)
    assert decided.mean() > 0.9, decided.mean()
    assert np.array_equal(sc[decided], want_s[decided])
    assert np.array_equal(qg[decided], wg[decided])
    # undecided groups: valid neighbours of the oracle's result
    und = ~decided
    assert np.all(np.abs(sc[und].astype(int) - want_s[und].astype(int)) <= 1)
    mag = lambda c: F.e2m1_decode(c)
    assert np.all(np.abs(mag(qg[und]) - mag(wg[und])) <= 2.0 + 1e-12)  # adjacent E2M1 values (or a scale step)
    assert rel(T[r], res.down.T) <= T_TOL
    assert rel(y[r], res.down.Y) <= Y_TOL
    return decided.mean()


@pytest.mark.parametrize("M,K,N,Kd_out,seed", [(200, 512, 512, 256, 121), (384, 256, 1024, 512, 122)])
def test_fused_mlp_block_small(M, K, N, Kd_out, seed):
    up, Wd, bd = _block(M, K, N, Kd_out, seed)
    _run(up, Wd, bd)


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
