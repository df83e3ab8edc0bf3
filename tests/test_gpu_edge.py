"""The method's edge cases on a B200, element by element against the oracle.

* Saturation. The NVFP4 activation tensor scale g_x is fixed at prepare time
  from the calibration statistic (static scale, reading C5 of the design
  notes), and s comes from the same statistic (msModelSlim SVDQuant entry,
  section 2.3 eq. 2). A runtime batch larger than its calibration therefore
  drives amax / (6 g_x) above 448, where the E4M3 group scale saturates, and
  the scaled values above 6, where the E2M1 codes saturate (satfinite, the
  rounding both sides use). Here the calibration is taken on X / 4 and the
  layer then runs X.
* All-zero structure. Zero rows, an all-zero 64-element group (INT4 amax = 0:
  scale 0, codes 0), all-zero 16-element groups (NVFP4 block scale 0, so the
  effective scale is 0 and the codes are 0), zero input channels (A_scale = 0)
  and a zero weight row (W_scale = 0), both of which keep s = 1 (section 2.3,
  eq. 2 with the s_min reading).

Codes and scales bit-exact, T within 2e-3 and Y within 4e-3 normwise, as in
the other parity tests; each test also asserts that its edge case occurred.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import svdquant as S
from parity import Case, T_TOL, Y_TOL, f64, gpu_activations, gpu_prepare, oracle_case, rel

pytestmark = pytest.mark.gpu


def _check(case):
    g = gpu_prepare(case)
    try:
        L = case.layer
        ex = g.export()
        assert np.array_equal(ex["s"].view(np.uint32), case.p.s.view(np.uint32))
        q, sc, T, pad_ok = gpu_activations(g, L.X.cuda(), L.fmt, L.M, L.K)
        assert pad_ok
        assert np.array_equal(q, case.r.x_codes), f"{np.sum(q != case.r.x_codes)} codes differ"
        if L.fmt == workloads.INT4_G64:
            assert np.array_equal(sc.view(np.uint32), case.r.x_scales.view(np.uint32))
        else:
            assert np.array_equal(sc, case.r.x_scales)
        assert rel(T[:, :L.rank], case.r.T) <= T_TOL
        Y = g.forward(L.X.cuda())
        torch.cuda.synchronize()
        y = f64(Y)
        assert np.all(np.isfinite(y))
        assert rel(y, case.r.Y) <= Y_TOL
        assert g.device_status() == 0
        return q, sc, T, y
    finally:
        g.close()


@pytest.mark.parametrize("fmt", workloads.FORMATS)
def test_runtime_batch_beyond_its_calibration_saturates_like_the_oracle(fmt):
    layer = workloads.custom(256, 1024, 512, 32, fmt, seed=95)
    X, W, b = workloads.to_f64(layer.X), workloads.to_f64(layer.W), workloads.to_f64(layer.bias)
    a = S.calibrate_absmax(0.25 * X)  # a power-of-two scaling: exact
    p = S.prepare(W, b, a, fmt, layer.alpha, layer.rank)
    case = Case(layer, X, W, b, a, p, S.forward(p, X))
    if fmt == workloads.NVFP4_G16:
        xs = S.smooth_activations(X, p.inv_s).reshape(layer.M, -1, 16)
        ratio = np.max(np.abs(xs), axis=-1) / (6.0 * np.float64(p.g_x))
        assert np.count_nonzero(ratio > 448.0) > 100, "no group scale saturates"
        assert np.count_nonzero(case.r.x_scales == 0x7E) > 100  # E4M3 448, the largest finite
        mags = case.r.x_codes & 7
        assert np.count_nonzero(mags == 7) > 1000  # E2M1 6, the largest finite
    _check(case)


def _zero_structured(fmt, seed):
    layer = workloads.custom(300, 1024, 512, 32, fmt, seed=seed)
    X = layer.X.clone()
    X[5] = 0
    X[130] = 0                     # all-zero rows, in two different 128-row blocks
    X[7, 128:192] = 0              # one all-zero 64-element group (= four 16-element groups)
    X[9, 48:64] = 0                # one all-zero 16-element group inside a non-zero 64-group
    X[:, 200:211] = 0              # zero input channels: A_scale = 0 there
    W = layer.W.clone()
    W[300] = 0                     # a zero weight row: W_scale = 0 there
    layer.X, layer.W = X, W
    return layer


@pytest.mark.parametrize("fmt", workloads.FORMATS)
def test_all_zero_rows_groups_and_channels(fmt):
    case = oracle_case(_zero_structured(fmt, seed=96 if fmt == workloads.INT4_G64 else 97))
    p, r = case.p, case.r
    assert np.all(p.s[200:211] == 1.0) and p.s[300] == 1.0  # s = 1 where a statistic is 0
    assert np.all(r.x_codes[5] == 0) and np.all(r.x_codes[130] == 0)
    if fmt == workloads.INT4_G64:
        assert r.x_scales[7, 2] == 0 and r.x_scales[5].max() == 0
    else:
        assert np.all(r.x_scales[7, 8:12] == 0) and r.x_scales[9, 3] == 0
    q, sc, T, y = _check(case)
    assert np.all(T[5] == 0) and np.all(T[130] == 0)  # the branch of a zero row is exactly zero
    # a zero row's output is the bias alone, rounded to bf16
    assert np.array_equal(y[5], p.bias) and np.array_equal(y[130], p.bias)
