"""The K = N = 3072 sweep (M 256 ... 16384, rank 16 ... 128, both formats, and a
rank-32 LoRA on top) through the C ABI against the oracle (needs a B200).

Every activation code and scale is compared in full. Y is compared on every
row up to M = 4096, and on a seeded sample of 1024 rows at M = 16384 (the
oracle's float64 forward is row-local, so a row sample is checked exactly as
the whole batch would be).
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import svdquant as S
from parity import T_TOL, Y_TOL, bf16_tensor, f64, gpu_activations, rel

pytestmark = pytest.mark.gpu

CASES = [  # (M, rank, format)
    (256, 16, workloads.NVFP4_G16),
    (1024, 64, workloads.INT4_G64),
    (4096, 128, workloads.NVFP4_G16),
    (4096, 32, workloads.INT4_G64),
    (16384, 32, workloads.NVFP4_G16),
]


def _prepare(layer):
    import rank_gemm_quantize_b200 as rq
    X = workloads.to_f64(layer.X)
    a = S.calibrate_absmax(X)
    p = S.prepare(workloads.to_f64(layer.W), workloads.to_f64(layer.bias), a, layer.fmt, layer.alpha, layer.rank)
    g = rq.Layer.prepare(layer.W.cuda(), layer.bias.cuda(), torch.from_numpy(a).cuda(), layer.fmt, layer.rank,
                         alpha=layer.alpha, factors=(bf16_tensor(p.L1), bf16_tensor(p.L2)))
    return X, p, g


def _rows(M):
    if M <= 4096:
        return np.arange(M)
    return np.sort(np.random.Generator(np.random.PCG64(4242)).choice(M, 1024, replace=False))


@pytest.mark.parametrize("M,rank,fmt", CASES)
def test_sweep_point_matches_oracle(M, rank, fmt):
    layer = workloads.config(4, M=M, rank=rank, fmt=fmt)[0]
    X, p, g = _prepare(layer)
    try:
        Xd = layer.X.cuda()
        q, sc, T, pad_ok = gpu_activations(g, Xd, fmt, M, layer.K)
        assert pad_ok
        codes, scales = S.quantize_rows(S.smooth_activations(X, p.inv_s), fmt, p.g_x)
        assert np.array_equal(q, codes)
        if fmt == workloads.INT4_G64:
            assert np.array_equal(sc.view(np.uint32), scales.view(np.uint32))
        else:
            assert np.array_equal(sc, scales)
        rows = _rows(M)
        r = S.forward(p, X[rows])
        assert rel(T[rows, :rank], r.T) <= T_TOL
        Y = g.forward(Xd)
        torch.cuda.synchronize()
        assert rel(f64(Y)[rows], r.Y) <= Y_TOL
        assert g.device_status() == 0
    finally:
        g.close()


@pytest.mark.parametrize("fmt", workloads.FORMATS)
def test_sweep_with_rank32_lora(fmt):
    """Rank 32 plus a rank-32 LoRA concatenated into the branch (A, B ~ N(0, 0.01),
    scale 1): the residual codes are untouched and Y follows the oracle."""
    layer = workloads.config(4, M=1024, rank=32, fmt=fmt, lora=True)[0]
    X, p, g = _prepare(layer)
    try:
        before = g.export()
        g.attach_lora(layer.lora_A.cuda(), layer.lora_B.cuda(), layer.lora_scale)
        after = g.export()
        assert np.array_equal(before["codes_packed"], after["codes_packed"])
        q = S.attach_lora(p, workloads.to_f64(layer.lora_A), workloads.to_f64(layer.lora_B), layer.lora_scale)
        assert after["rank"] == 64
        Y = g.forward(layer.X.cuda())
        torch.cuda.synchronize()
        assert rel(f64(Y), S.forward(q, X).Y) <= Y_TOL
    finally:
        g.close()
