"""Pins of the oracle's SVDQuant steps (CPU only).

Each step is checked against what the pages and the mathematics fix:
closed-form values of the smoothing factor (eq. 2), the migration identity
(eq. 1), Eckart-Young and the residual energy (eqs. 5-6) with an SVD built
from known factors and with an independent one-sided Jacobi SVD, the dual-path
equivalence with quantization disabled (section 2.4), and a brute-force
re-computation of a tiny layer with plain Python loops.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import formats as F
from oracle import svdquant as S
import workloads

F32 = np.float32


# --------------------------------------------------------------------- eq. 2

def test_smoothing_factor_closed_forms():
    s, inv = S.smoothing_factors(np.array([4.0, 9.0, 1e-20, 0.0, 5.0]), np.array([1.0, 4.0, 1.0, 3.0, 0.0]), 0.5)
    assert s[0] == 2.0 and s[1] == 1.5
    assert s[2] == S.S_MIN  # sqrt(1e-20) = 1e-10 clamped at s_min
    assert s[3] == 1.0 and s[4] == 1.0  # dead channels keep s = 1
    assert inv[1] == F32(1.0) / F32(1.5)
    s1, _ = S.smoothing_factors(np.array([3.0, 0.25]), np.array([7.0, 2.0]), 1.0)
    assert np.array_equal(s1, np.array([3.0, 0.25], F32))  # alpha = 1: s = A_scale
    s0, _ = S.smoothing_factors(np.array([3.0, 0.25]), np.array([8.0, 2.0]), 0.0)
    assert np.array_equal(s0, np.array([0.125, 0.5], F32))  # alpha = 0: s = 1 / W_scale
    s3, _ = S.smoothing_factors(np.array([16.0]), np.array([2.0]), 0.75)
    assert s3[0] == F32(16.0 ** 0.75 / 2.0 ** 0.25)


def test_statistics_axes():
    X = np.array([[1.0, -5.0], [-3.0, 2.0]])
    assert np.array_equal(S.calibrate_absmax(X), np.array([3.0, 5.0], F32))
    W = np.array([[1.0, -7.0, 2.0], [0.5, 0.25, -0.75]])  # [K=2, N=3]
    assert np.array_equal(S.weight_absmax(W), np.array([7.0, 0.75], F32))


# --------------------------------------------------------------------- eq. 1

def test_migration_identity():
    layer = workloads.custom(64, 256, 96, 8, workloads.INT4_G64, seed=11)
    X, W, b = workloads.to_f64(layer.X), workloads.to_f64(layer.W), workloads.to_f64(layer.bias)
    a = S.calibrate_absmax(X)
    s, inv_s = S.smoothing_factors(a, S.weight_absmax(W), 0.5)
    lhs = S.smooth_activations(X, inv_s).astype(np.float64) @ S.migrate_weight(W, s).astype(np.float64)
    rhs = X @ W
    assert np.linalg.norm(lhs - rhs) / np.linalg.norm(rhs) < 1e-6
    # smoothing actually moved the outliers: the smoothed activations' channel maxima are flatter
    xh = S.smooth_activations(X, inv_s)
    assert np.max(np.abs(xh)) / np.median(np.max(np.abs(xh), 0)) < np.max(np.abs(X)) / np.median(np.max(np.abs(X), 0))


# ------------------------------------------------------------- eqs. 3, 5, 6

def _orthonormal(rng, n, k):
    q, r = np.linalg.qr(rng.standard_normal((n, k)))
    return q * np.sign(np.diag(r))


def test_svd_recovers_a_known_decomposition():
    rng = np.random.default_rng(12)
    K, N = 40, 30
    U, V = _orthonormal(rng, K, N), _orthonormal(rng, N, N)
    sigma = np.array([50.0, 20.0, 10.0, 5.0] + list(np.linspace(1.0, 0.01, N - 4)))
    W_hat = (U * sigma) @ V.T
    L1, L2, sig = S.svd_factors(W_hat, 4, round_bf16=False)
    assert np.allclose(sig, sigma, rtol=1e-12, atol=1e-12)
    assert np.allclose(L1 @ L2, (U[:, :4] * sigma[:4]) @ V[:, :4].T, atol=1e-11)
    # each column of L1 is unit-norm and signed so that its largest entry is positive
    assert np.allclose(np.linalg.norm(L1, axis=0), 1.0)
    for j in range(4):
        assert L1[np.argmax(np.abs(L1[:, j])), j] > 0


def _jacobi_singular_values(A, sweeps=60):
    """One-sided Hestenes Jacobi: orthogonalize columns pairwise; the column norms
    are the singular values. Independent of LAPACK."""
    A = np.array(A, dtype=np.float64, copy=True)
    n = A.shape[1]
    for _ in range(sweeps):
        off = 0.0
        for p in range(n - 1):
            for q in range(p + 1, n):
                alpha = A[:, p] @ A[:, p]
                beta = A[:, q] @ A[:, q]
                gamma = A[:, p] @ A[:, q]
                off = max(off, abs(gamma) / math.sqrt(alpha * beta + 1e-300))
                if gamma == 0.0:
                    continue
                zeta = (beta - alpha) / (2.0 * gamma)
                t = math.copysign(1.0, zeta) / (abs(zeta) + math.sqrt(1.0 + zeta * zeta))
                c = 1.0 / math.sqrt(1.0 + t * t)
                s = c * t
                ap, aq = A[:, p].copy(), A[:, q].copy()
                A[:, p] = c * ap - s * aq
                A[:, q] = s * ap + c * aq
        if off < 1e-15:
            break
    return np.sort(np.linalg.norm(A, axis=0))[::-1]


@pytest.mark.parametrize("shape", [(8, 8), (12, 9), (20, 16), (16, 24)])
def test_svd_singular_values_match_independent_jacobi(shape):
    rng = np.random.default_rng(sum(shape))
    W = rng.standard_normal(shape)
    _, _, sig = S.svd_factors(W, 2, round_bf16=False)
    ref = _jacobi_singular_values(W if shape[0] >= shape[1] else W.T)
    assert np.allclose(sig, ref[:len(sig)], rtol=1e-10, atol=1e-12)


def test_eckart_young_residual_energy_and_optimality():
    rng = np.random.default_rng(13)
    W = rng.standard_normal((48, 32)) + 5 * np.outer(rng.standard_normal(48), rng.standard_normal(32))
    prev = np.inf
    for r in range(0, 33, 4):
        L1, L2, sig = S.svd_factors(W, r, round_bf16=False)
        energy = np.linalg.norm(W - L1 @ L2) ** 2
        assert np.isclose(energy, np.sum(sig[r:] ** 2), rtol=1e-10, atol=1e-10)  # eq. 6
        assert energy <= prev + 1e-9  # more rank never increases the residual energy
        prev = energy
    # eq. 5: no other rank-r matrix does better (random ones and perturbations of L_r)
    r = 3
    L1, L2, _ = S.svd_factors(W, r, round_bf16=False)
    best = np.linalg.norm(W - L1 @ L2)
    for _ in range(200):
        P = rng.standard_normal((48, r)) @ rng.standard_normal((r, 32))
        assert np.linalg.norm(W - P) >= best
        Q = (L1 + 1e-3 * rng.standard_normal(L1.shape)) @ (L2 + 1e-3 * rng.standard_normal(L2.shape))
        assert np.linalg.norm(W - Q) >= best - 1e-12


def test_residual_closes_the_split_exactly():
    rng = np.random.default_rng(14)
    W_hat = rng.standard_normal((64, 48)).astype(F32)
    L1, L2, _ = S.svd_factors(W_hat, 6)  # bf16 factors
    R = S.residual(W_hat, L1, L2)
    exact = W_hat.astype(np.float64) - L1 @ L2
    # R is the float32 rounding of W_hat - L1 L2: within half a float32 ulp
    ulp = np.spacing(np.abs(R).astype(F32)).astype(np.float64)
    assert np.all(np.abs(R.astype(np.float64) - exact) <= 0.5 * ulp)
    # the bf16 factors really are bf16 values
    assert np.array_equal(F.bf16_round(L1), L1) and np.array_equal(F.bf16_round(L2), L2)
    # full rank with unrounded factors reconstructs W_hat: R ~ 0
    L1f, L2f, _ = S.svd_factors(W_hat, 48, round_bf16=False)
    assert np.max(np.abs(S.residual(W_hat, L1f, L2f))) < 1e-12 * np.max(np.abs(W_hat)) * 48


# ------------------------------------------------- section 2.4 equivalence

@pytest.mark.parametrize("fmt", workloads.FORMATS)
@pytest.mark.parametrize("rank", [1, 4, 16, 64])
def test_dual_path_without_quantization_equals_xw_plus_b(fmt, rank):
    layer = workloads.custom(32, 128, 64, rank, fmt, seed=20 + rank)
    X, W, b = workloads.to_f64(layer.X), workloads.to_f64(layer.W), workloads.to_f64(layer.bias)
    p = S.prepare(W, b, S.calibrate_absmax(X), fmt, 0.5, rank)
    y = S.forward_unquantized(p, X)
    ref = X @ W + b
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < 2e-6


def test_quantized_layer_beats_plain_w4a4_on_outlier_data():
    """Diagnostic of the method's claim (abstract; section 2.1): with outliers,
    SVDQuant's error is below smoothing-only and below naive W4A4."""
    layer = workloads.custom(128, 512, 256, 32, workloads.INT4_G64, seed=31, n_outliers=6)
    X, W, b = workloads.to_f64(layer.X), workloads.to_f64(layer.W), workloads.to_f64(layer.bias)
    ref = X @ W + b
    a = S.calibrate_absmax(X)
    err = lambda y: np.linalg.norm(y - ref) / np.linalg.norm(ref)
    svdq = err(S.forward(S.prepare(W, b, a, "int4_g64", 0.5, 32), X).Y)
    smooth_only = err(S.forward(S.prepare(W, b, a, "int4_g64", 0.5, 0), X).Y)
    naive = err(S.forward(_naive(W, b), X).Y)
    assert svdq < smooth_only < naive


def _naive(W, b):
    """Plain W4A4 (no smoothing, no branch): s = 1 everywhere, rank 0."""
    K, N = W.shape
    L1 = np.zeros((K, 0))
    L2 = np.zeros((0, N))
    p = S.prepare_from_factors(W, b, np.ones(K), "int4_g64", 1.0, L1, L2)
    # alpha = 1 with A_scale = 1 gives s = 1 exactly
    assert np.all(p.s == 1.0)
    return p


# ----------------------------------------------------------- brute force

def _bf(x):
    return float(F.bf16_round(np.float64(x)))


def _brute_force_layer(X, W, b, a, fmt, rank, L1, L2, smooth=True):
    """Every quantity of a tiny layer recomputed with plain Python loops from
    the definitions (no vectorized oracle code): eq. 2, eq. 1, R = W_hat - L1 L2,
    the group quantizers, the integer / E2M1 group sums, the branch and the bias.
    smooth=False: s = 1 everywhere (no migration)."""
    K, N = W.shape
    M = X.shape[0]
    s, inv_s = [], []
    for k in range(K):
        wk = max(abs(W[k, n]) for n in range(N))
        ak = float(a[k])
        if not smooth:
            s.append(F32(1.0))
            inv_s.append(F32(1.0))
            continue
        if ak == 0 or wk == 0:
            sk = 1.0
        else:
            sk = math.sqrt(ak) / math.sqrt(wk)
        sk = max(float(F32(sk)), float(F32(1e-5)))
        s.append(F32(sk))
        inv_s.append(F32(F32(1.0) / F32(sk)))
    W_hat = [[F32(s[k] * F32(W[k, n])) for n in range(N)] for k in range(K)]
    R = [[0.0] * N for _ in range(K)]
    for k in range(K):
        for n in range(N):
            acc = float(W_hat[k][n])
            for j in range(rank):
                acc -= L1[k, j] * L2[j, n]
            R[k][n] = F32(acc)
    x_hat = [[F32(F32(X[m, k]) * inv_s[k]) for k in range(K)] for m in range(M)]
    G = 64 if fmt == "int4_g64" else 16

    def quant_vec(vec, g):
        codes, scales = [], []
        for g0 in range(0, K, G):
            blk = vec[g0:g0 + G]
            amax = F32(max(abs(float(v)) for v in blk))
            if fmt == "int4_g64":
                if amax == 0:
                    scales.append(0.0)
                    codes += [0] * G
                    continue
                inv = F32(F32(7.0) / amax)
                scales.append(float(F32(amax / F32(7.0))))
                for v in blk:
                    t = float(F32(v * inv))
                    codes.append(min(range(-8, 8), key=lambda q: (abs(t - q), q % 2)))
            else:
                sb = int(F.e4m3_encode(F32(amax / F32(F32(6.0) * g))))
                eff = F32(F32(F.e4m3_decode(sb)) * g)
                scales.append(float(F.e4m3_decode(sb)) * float(g))
                for v in blk:
                    if eff == 0:
                        codes.append(0.0)
                        continue
                    t = float(F32(v * F32(F32(1.0) / eff)))
                    codes.append(float(F.e2m1_decode(_e2m1_nearest(t))))
        return codes, scales

    if fmt == "nvfp4_g16":
        amax_R = max(abs(float(R[k][n])) for k in range(K) for n in range(N))
        g_w = F32(F32(amax_R) / F32(2688.0)) if amax_R else F32(1.0)
        g_x = F32(max(float(F32(F32(a[k]) * inv_s[k])) for k in range(K)) / F32(2688.0))
    else:
        g_w = g_x = F32(1.0)
    wq = [quant_vec([R[k][n] for k in range(K)], g_w) for n in range(N)]
    Y = np.zeros((M, N))
    for m in range(M):
        xc, xs = quant_vec(x_hat[m], g_x)
        T = [sum(float(x_hat[m][k]) * L1[k, j] for k in range(K)) for j in range(rank)]
        for n in range(N):
            wc, ws = wq[n]
            main = 0.0
            for gi in range(K // G):
                if fmt == "int4_g64":
                    isum = sum(int(xc[gi * G + i]) * int(wc[gi * G + i]) for i in range(G))  # exact integer
                    main += xs[gi] * ws[gi] * isum
                else:
                    fsum = sum(xc[gi * G + i] * wc[gi * G + i] for i in range(G))  # exact in float64
                    main += xs[gi] * ws[gi] * fsum
            Y[m, n] = main + sum(T[j] * L2[j, n] for j in range(rank)) + b[n]
    return Y


def _e2m1_nearest(t):
    best = None
    for code in range(16):
        val = float(F.e2m1_decode(code))
        if (code >= 8) != bool(np.signbit(t)):
            continue
        key = (abs(t - val), code & 1)
        if best is None or key < best[0]:
            best = (key, code)
    if abs(t) >= 6:
        return 0xF if np.signbit(t) else 0x7
    return best[1]


@pytest.mark.parametrize("fmt", workloads.FORMATS)
def test_tiny_layer_brute_force(fmt):
    layer = workloads.custom(3, 128, 8, 2, fmt, seed=41, n_outliers=2)
    X, W, b = workloads.to_f64(layer.X), workloads.to_f64(layer.W), workloads.to_f64(layer.bias)
    a = S.calibrate_absmax(X)
    p = S.prepare(W, b, a, fmt, 0.5, 2)
    y = S.forward(p, X).Y
    yb = _brute_force_layer(X, W, b, a, fmt, 2, p.L1, p.L2)
    assert np.allclose(y, yb, rtol=1e-12, atol=1e-12)


def test_brute_force_catches_a_planted_mistake():
    """A dropped bias or a sign flip in the branch must break the brute-force pin."""
    layer = workloads.custom(3, 128, 8, 2, "int4_g64", seed=42, n_outliers=2)
    X, W, b = workloads.to_f64(layer.X), workloads.to_f64(layer.W), workloads.to_f64(layer.bias)
    a = S.calibrate_absmax(X)
    p = S.prepare(W, b, a, "int4_g64", 0.5, 2)
    good = _brute_force_layer(X, W, b, a, "int4_g64", 2, p.L1, p.L2)
    r = S.forward(p, X)
    assert not np.allclose(r.main + r.T @ p.L2, good, rtol=1e-9)  # bias dropped
    assert not np.allclose(r.main - r.T @ p.L2 + b, good, rtol=1e-9)  # branch sign flipped
    assert not np.allclose(r.main + (r.T @ p.L2).T.T[::-1] + b, good, rtol=1e-9)  # rows mixed


# ------------------------------------------------------------------ LoRA

def test_lora_attach_changes_only_the_branch():
    layer = workloads.custom(16, 128, 64, 4, "int4_g64", seed=51, lora_rank=8)
    X, W, b = workloads.to_f64(layer.X), workloads.to_f64(layer.W), workloads.to_f64(layer.bias)
    A, B = workloads.to_f64(layer.lora_A), workloads.to_f64(layer.lora_B)
    p = S.prepare(W, b, S.calibrate_absmax(X), "int4_g64", 0.5, 4)
    q = S.attach_lora(p, A, B, 0.5)
    assert np.array_equal(q.w_codes, p.w_codes) and np.array_equal(q.w_scales, p.w_scales)
    assert q.L1.shape == (128, 12) and q.L2.shape == (12, 64)
    y0, y1 = S.forward(p, X).Y, S.forward(q, X).Y
    delta = y1 - y0
    x_hat = S.smooth_activations(X, p.inv_s).astype(np.float64)
    assert np.allclose(delta, (x_hat @ q.L1[:, 4:]) @ q.L2[4:, :], rtol=1e-10, atol=1e-14)
    # and, up to bf16 rounding of diag(s) A and scale B, it is the LoRA term scale * X A B
    ref = 0.5 * X @ A @ B
    assert np.linalg.norm(delta - ref) / np.linalg.norm(ref) < 1e-2



# ------------------------------------------------- ablations of the method

@pytest.mark.parametrize("fmt", workloads.FORMATS)
@pytest.mark.parametrize("rank,smooth", [(0, True), (2, False), (0, False)])
def test_tiny_ablation_layers_brute_force(fmt, rank, smooth):
    """Rank 0 (smoothing only: the SmoothQuant special case of the entry's
    related terms) and no smoothing (s = 1) recomputed by plain loops."""
    layer = workloads.custom(3, 128, 8, max(rank, 1), fmt, seed=43, n_outliers=2)
    X, W, b = workloads.to_f64(layer.X), workloads.to_f64(layer.W), workloads.to_f64(layer.bias)
    a = S.calibrate_absmax(X)
    p = S.prepare(W, b, a, fmt, 0.5, rank, smooth=smooth)
    assert p.L1.shape == (128, rank) and p.L2.shape == (rank, 8)
    y = S.forward(p, X).Y
    yb = _brute_force_layer(X, W, b, a, fmt, rank, p.L1, p.L2, smooth=smooth)
    assert np.allclose(y, yb, rtol=1e-12, atol=1e-12)


def test_rank0_residual_is_the_migrated_weight_and_the_branch_is_empty():
    layer = workloads.custom(16, 128, 64, 1, "nvfp4_g16", seed=44)
    X, W, b = workloads.to_f64(layer.X), workloads.to_f64(layer.W), workloads.to_f64(layer.bias)
    p = S.prepare(W, b, S.calibrate_absmax(X), "nvfp4_g16", 0.5, 0)
    assert np.array_equal(p.R.view(np.uint32), S.migrate_weight(W, p.s).view(np.uint32))
    r = S.forward(p, X)
    assert r.T.shape == (16, 0)
    assert np.array_equal(r.Y, r.main + p.bias[None, :])
    y = S.forward_unquantized(p, X)  # the equivalence holds without a branch too
    assert np.linalg.norm(y - (X @ W + b)) / np.linalg.norm(X @ W + b) < 2e-6


def test_no_smoothing_leaves_activations_and_weights_as_they_are():
    layer = workloads.custom(16, 128, 64, 4, "int4_g64", seed=45)
    X, W, b = workloads.to_f64(layer.X), workloads.to_f64(layer.W), workloads.to_f64(layer.bias)
    p = S.prepare(W, b, S.calibrate_absmax(X), "int4_g64", 0.5, 4, smooth=False)
    assert np.all(p.s == 1.0) and np.all(p.inv_s == 1.0)
    assert np.array_equal(S.smooth_activations(X, p.inv_s), X.astype(F32))
    y = S.forward_unquantized(p, X)
    assert np.linalg.norm(y - (X @ W + b)) / np.linalg.norm(X @ W + b) < 2e-6


def test_ablation_error_ordering_on_outlier_data():
    """Diagnostic (abstract; section 2.1): on outlier activations the full
    method beats smoothing alone, which beats no smoothing, in both formats."""
    for fmt in workloads.FORMATS:
        layer = workloads.custom(128, 512, 256, 32, fmt, seed=46, n_outliers=6)
        X, W, b = workloads.to_f64(layer.X), workloads.to_f64(layer.W), workloads.to_f64(layer.bias)
        ref = X @ W + b
        a = S.calibrate_absmax(X)
        err = lambda p: np.linalg.norm(S.forward(p, X).Y - ref) / np.linalg.norm(ref)
        full = err(S.prepare(W, b, a, fmt, 0.5, 32))
        smooth_only = err(S.prepare(W, b, a, fmt, 0.5, 0))
        naive = err(S.prepare(W, b, a, fmt, 0.5, 0, smooth=False))
        assert full < smooth_only < naive, (fmt, full, smooth_only, naive)


# ------------------------------------------- per-row adapter selection

def test_selected_adapters_follow_their_definition():
    """Per-row selection against the composition it must equal: all bits set
    is the layer with both adapters concatenated (attach_lora twice), no bit
    set is the layer alone, one bit is the layer with that adapter alone."""
    layer = workloads.custom(12, 128, 64, 4, "nvfp4_g16", seed=52, lora_rank=8)
    X, W, b = workloads.to_f64(layer.X), workloads.to_f64(layer.W), workloads.to_f64(layer.bias)
    A0, B0 = workloads.to_f64(layer.lora_A), workloads.to_f64(layer.lora_B)
    rng = np.random.Generator(np.random.PCG64(53))
    A1 = F.bf16_round(rng.normal(0, 0.01, (128, 16)))
    B1 = F.bf16_round(rng.normal(0, 0.01, (16, 64)))
    p = S.prepare(W, b, S.calibrate_absmax(X), "nvfp4_g16", 0.5, 4)
    ads = {0: S.lora_factors(p, A0, B0, 0.5), 1: S.lora_factors(p, A1, B1, 2.0)}
    mask = np.array([0b11, 0b00, 0b01, 0b10] * 3)
    y = S.forward_selected(p, ads, X, mask)
    both = S.forward(S.attach_lora(S.attach_lora(p, A0, B0, 0.5), A1, B1, 2.0), X).Y
    only0 = S.forward(S.attach_lora(p, A0, B0, 0.5), X).Y
    only1 = S.forward(S.attach_lora(p, A1, B1, 2.0), X).Y
    base = S.forward(p, X).Y
    for m in range(12):
        want = {0b11: both, 0b00: base, 0b01: only0, 0b10: only1}[mask[m]][m]
        assert np.allclose(y[m], want, rtol=1e-12, atol=1e-13), m
    assert np.array_equal(y[mask == 0], base[mask == 0])
    # a planted mistake: slot bits read the wrong way round
    y_bad = S.forward_selected(p, {0: ads[1], 1: ads[0]}, X, mask)
    assert not np.allclose(y_bad[mask == 0b01], only0[mask == 0b01], rtol=1e-6)


# ------------------------------------------------- the weight-only baseline

def test_weight_only_brute_force():
    layer = workloads.custom(3, 128, 8, 1, "int4_g64", seed=47)
    X, W, b = workloads.to_f64(layer.X), workloads.to_f64(layer.W), workloads.to_f64(layer.bias)
    p = S.prepare_weight_only(W, b)
    y = S.forward_weight_only(p, X)
    K, N = W.shape
    yb = np.zeros((3, N))
    for n in range(N):
        w = []
        for g0 in range(0, K, 64):
            col = [F32(W[k, n]) for k in range(g0, g0 + 64)]
            amax = F32(max(abs(float(v)) for v in col))
            if amax == 0:
                w += [0.0] * 64
                continue
            inv, sc = F32(F32(7.0) / amax), F32(amax / F32(7.0))
            for v in col:
                t = float(F32(v * inv))
                q = min(range(-8, 8), key=lambda c: (abs(t - c), c % 2))
                w.append(_bf(float(F32(F32(q) * sc))))
        for m in range(3):
            yb[m, n] = sum(X[m, k] * w[k] for k in range(K)) + b[n]
    assert np.allclose(y, yb, rtol=1e-12, atol=1e-12)


def test_weight_only_is_exact_on_representable_weights():
    """Weights that are already integer multiples (|q| <= 7, each group's
    largest |q| = 7) of a power-of-two group scale quantize without error:
    the baseline then computes X W + b exactly (every product and partial sum
    is exact in float64 for these small integers)."""
    rng = np.random.Generator(np.random.PCG64(48))
    K, N, M = 256, 16, 5
    q = rng.integers(-7, 8, size=(K, N))
    q[::64, :] = 7  # each group of 64 along k reaches amax = 7 * scale
    scale = 2.0 ** rng.integers(-6, -2, size=(K // 64, N))
    W = q * np.repeat(scale, 64, axis=0)
    X = rng.integers(-4, 5, size=(M, K)).astype(np.float64)
    b = rng.integers(-3, 4, size=N) * 0.125
    p = S.prepare_weight_only(W, b)
    assert np.array_equal(S.dequantize_weight_only(p), W.T)
    assert np.array_equal(S.forward_weight_only(p, X), X @ W + b)


# ------------------------------------------------------------- the MLP block

def test_gelu_closed_forms():
    x = np.array([0.0, 1.0, -1.0, 3.0, -3.0, 10.0, -10.0, 0.5])
    g = S.gelu_erf(x)
    assert g[0] == 0.0
    # GELU(x) - GELU(-x) = x exactly in the definition (Phi(x) + Phi(-x) = 1)
    assert np.allclose(g[1::2][:3] - g[2::2][:3], x[1::2][:3], rtol=0, atol=1e-15)
    assert abs(g[5] - 10.0) < 1e-20 and abs(g[6]) < 1e-20  # the tails
    assert abs(g[1] - 0.8413447460685429) < 1e-15  # Phi(1) = 0.8413447460685429...
    assert abs(g[7] - 0.5 * 0.6914624612740131) < 1e-15  # Phi(0.5)


def test_mlp_block_is_the_composition_of_two_brute_force_layers():
    """The block against two plain-loop layers with GELU between them (math.erf)."""
    up_l = workloads.custom(3, 128, 64, 2, "nvfp4_g16", seed=49, n_outliers=2)
    X, Wu, bu = workloads.to_f64(up_l.X), workloads.to_f64(up_l.W), workloads.to_f64(up_l.bias)
    rng = np.random.Generator(np.random.PCG64(50))
    Wd = F.bf16_round(rng.normal(0, 0.02, (64, 16)))
    bd = F.bf16_round(rng.normal(0, 0.01, 16))
    p_up = S.prepare(Wu, bu, S.calibrate_absmax(X), "nvfp4_g16", 0.5, 2)
    y_up = F.bf16_round(_brute_force_layer(X, Wu, bu, S.calibrate_absmax(X), "nvfp4_g16", 2, p_up.L1, p_up.L2))
    h = F.bf16_round(np.array([[0.5 * v * (1 + math.erf(v / math.sqrt(2))) for v in row] for row in y_up]))
    a_d = S.calibrate_absmax(h)
    p_down = S.prepare(Wd, bd, a_d, "nvfp4_g16", 0.5, 2)
    want = _brute_force_layer(h, Wd, bd, a_d, "nvfp4_g16", 2, p_down.L1, p_down.L2)
    r = S.mlp_forward(p_up, p_down, X)
    assert np.array_equal(r.y_up, y_up) and np.array_equal(r.h, h)
    assert np.allclose(r.down.Y, want, rtol=1e-12, atol=1e-12)
