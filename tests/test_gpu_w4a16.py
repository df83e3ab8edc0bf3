"""The 4-bit weight-only baseline kernel (W4A16) against the oracle, on a B200.

The baseline the SVDQuant abstract measures its speedup against: weights
quantized alone with the INT4 group-64 quantizer, bf16 activations. Codes and
scales are compared bit for bit; Y normwise within 4e-3 (bf16 output) on
ragged shapes, a zero-input case, and the FLUX MLP-up shape at full size on a
row sample (the forward is row-local).
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import formats as F
from oracle import svdquant as S
from parity import Y_TOL, f64, rel

pytestmark = pytest.mark.gpu


def _check(layer, rows=None):
    import rank_gemm_quantize_b200 as rq
    X, W, b = workloads.to_f64(layer.X), workloads.to_f64(layer.W), workloads.to_f64(layer.bias)
    p = S.prepare_weight_only(W, b)
    g = rq.WeightOnlyLayer(layer.W.cuda(), layer.bias.cuda())
    try:
        codes, scales = g.export()
        assert np.array_equal(codes, F.pack_nibbles(p.codes))
        assert np.array_equal(scales.view(np.uint32), np.ascontiguousarray(p.scales.T).view(np.uint32))
        Y = g.forward(layer.X.cuda())
        torch.cuda.synchronize()
        y = f64(Y)
        r = np.arange(layer.M) if rows is None else rows
        assert np.all(np.isfinite(y[r]))
        assert rel(y[r], S.forward_weight_only(p, X[r])) <= Y_TOL
        return y
    finally:
        g.close()


@pytest.mark.parametrize("M,K,N,seed", [(129, 384, 144, 111), (256, 512, 512, 112), (1, 256, 272, 113)])
def test_weight_only_matches_oracle(M, K, N, seed):
    _check(workloads.custom(M, K, N, 1, workloads.INT4_G64, seed=seed))


def test_weight_only_zero_input_gives_the_bias():
    layer = workloads.custom(130, 256, 128, 1, workloads.INT4_G64, seed=114)
    layer.X = torch.zeros_like(layer.X)
    y = _check(layer)
    assert np.array_equal(y, np.broadcast_to(workloads.to_f64(layer.bias), y.shape))


def test_weight_only_full_size_mlp_up():
    layer = workloads.config(3)[0]  # 4608 x 3072 -> 12288
    rows = np.sort(np.random.Generator(np.random.PCG64(115)).choice(layer.M, 512, replace=False))
    _check(layer, rows)
