"""Shared helpers of the GPU parity tests: run the oracle and the CUDA path on the
same seeded inputs and bring the CUDA path's outputs into the oracle's
canonical layouts (index permutations and byte decoding only)."""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

import oracle
from oracle import formats as F
from oracle import svdquant as S
import workloads

Y_TOL = 4e-3  # normwise ||Y_gpu - Y|| / ||Y|| (bf16 output)
T_TOL = 2e-3  # normwise on T = x_hat L1 (bf16 storage)


def rel(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def bf16_tensor(a: np.ndarray, device="cuda") -> torch.Tensor:
    """float64 array holding bf16 values -> bf16 tensor (exact)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(torch.bfloat16)
    assert np.array_equal(t.to(torch.float64).numpy(), a), "values are not bf16"
    return t.to(device)


@dataclass
class Case:
    layer: workloads.Layer
    X: np.ndarray
    W: np.ndarray
    b: np.ndarray
    a: np.ndarray
    p: oracle.Prepared
    r: object  # ForwardResult


def oracle_case(layer: workloads.Layer) -> Case:
    """The oracle on the layer's inputs; layer.meta["smooth"] = False selects
    the no-smoothing ablation (rank 0, the smoothing-only one, is layer.rank)."""
    X, W, b = workloads.to_f64(layer.X), workloads.to_f64(layer.W), workloads.to_f64(layer.bias)
    a = S.calibrate_absmax(X)
    p = S.prepare(W, b, a, layer.fmt, layer.alpha, layer.rank, smooth=layer.meta.get("smooth", True))
    return Case(layer, X, W, b, a, p, S.forward(p, X))


def gpu_prepare(case: Case, with_factors: bool = True):
    import rank_gemm_quantize_b200 as rq
    L = case.layer
    W = L.W.cuda()
    bias = L.bias.cuda()
    a = torch.from_numpy(case.a).cuda()
    factors = (bf16_tensor(case.p.L1), bf16_tensor(case.p.L2)) if with_factors else None
    return rq.Layer.prepare(W, bias, a, L.fmt, L.rank, alpha=L.alpha, factors=factors,
                            smooth=L.meta.get("smooth", True))


def canonical_weight_codes(p: oracle.Prepared) -> np.ndarray:
    """The oracle's weight codes in the export layout: packed nibbles [N, K/2]."""
    return F.pack_nibbles(p.w_codes)


def gpu_activations(layer_gpu, X: torch.Tensor, fmt: str, M: int, K: int):
    """K1 outputs in canonical layout: (codes [M, K], scales [M, K/G], T [M, rank_pad] unscaled)."""
    info = layer_gpu.info()
    codes, scales, T = layer_gpu.quantize_activations(X)
    torch.cuda.synchronize()
    codes = codes.cpu().numpy()
    T_all = f64(T) / np.float64(np.float32(info.t_scale))
    T = T_all[:M]
    t_pad_ok = bool(np.all(T_all[M:] == 0))
    if fmt == workloads.INT4_G64:
        vals = F.e4m3_decode(codes[:M])
        assert np.all(vals == np.rint(vals)), "INT4 codes must be integers"
        q = vals.astype(np.int8)
        sc = scales.cpu().numpy().T[:M].copy()  # [K/64][M_pad] -> [M, K/64]
        pad_ok = bool(np.all(codes[M:] == 0)) and t_pad_ok
    else:
        q = F.unpack_nibbles(codes[:M], signed=False)
        atoms = scales.cpu().numpy()
        m = np.arange(M)[:, None]
        i = np.arange(K // 16)[None, :]
        idx = ((m // 128) * (K // 64) + i // 4) * 512 + (m % 32) * 16 + ((m // 32) % 4) * 4 + i % 4
        sc = atoms[idx]
        pad_ok = bool(np.all(codes[M:] == 0)) and t_pad_ok
    return q, sc, T, pad_ok
