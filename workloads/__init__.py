"""Seeded synthetic inputs for the SVDQuant W4A4 + low-rank linear layer.

This module is shared by the CPU oracle, the tests and the benchmark. It only
draws random numbers and arranges them into the shapes of the FLUX-like layers;
it holds none of the method's arithmetic (no smoothing, no SVD, no quantizer).

Recipes (one numpy PCG64 stream per config, seed = 1000 + config id):

* cfg 0  single linear, INT4 g64: X [256,512] ~ N(0,1) with 4 random channels
  multiplied by 50; W [512,512] ~ N(0,0.02); bias ~ N(0,0.01); alpha 0.5, r 16.
* cfg 1  FLUX-like attention projection, INT4 g64: X [4608,3072] ~ N(0,1)
  (4096 image + 512 text tokens), round(1% of K) channels each multiplied by
  an independent U(20,100); W [3072,3072] ~ N(0,0.02); bias ~ N(0,0.01); r 32.
* cfg 2  FLUX-like MLP pair, INT4 g64: up X [4608,3072] -> W [3072,12288];
  down X [4608,12288] = erf-GELU of the up layer's unquantized output
  X_up @ W_up + b_up (float32), with the same outlier recipe re-applied to
  round(1% of 12288) channels; W_down [12288,3072]; r 32.
* cfg 3  the cfg 2 pair in NVFP4 (same seed, hence identical X/W/bias).
* cfg 4  sweep at K = N = 3072: M in {256,1024,4096,16384}, r in
  {16,32,64,128}, either format, optionally a rank-32 LoRA with
  A, B ~ N(0,0.01) and scale 1 (its own stream, seed 1104).

Every tensor is drawn in float64, rounded once to bfloat16 (round to nearest
even, by torch's CPU conversion) and returned as a CPU bfloat16 tensor.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

INT4_G64 = "int4_g64"
NVFP4_G16 = "nvfp4_g16"
FORMATS = (INT4_G64, NVFP4_G16)

SWEEP_M = (256, 1024, 4096, 16384)
SWEEP_R = (16, 32, 64, 128)


@dataclass
class Layer:
    """One linear layer's synthetic inputs (all CPU bfloat16 tensors)."""

    name: str
    fmt: str
    M: int
    K: int
    N: int
    rank: int
    alpha: float
    X: torch.Tensor  # [M, K]
    W: torch.Tensor  # [K, N]
    bias: torch.Tensor  # [N]
    lora_A: Optional[torch.Tensor] = None  # [K, r_l]
    lora_B: Optional[torch.Tensor] = None  # [r_l, N]
    lora_scale: float = 1.0
    seed: int = 0
    meta: dict = field(default_factory=dict)


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(torch.float32).to(torch.bfloat16)


def _outlier_x(rng: np.random.Generator, M: int, K: int, n_out: int, fixed_gain: Optional[float]) -> np.ndarray:
    x = rng.standard_normal((M, K))
    ch = rng.permutation(K)[:n_out]
    if fixed_gain is None:
        gain = rng.uniform(20.0, 100.0, size=n_out)
    else:
        gain = np.full(n_out, fixed_gain)
    x[:, ch] *= gain
    return x


def _linear_inputs(rng, M, K, N, n_out, fixed_gain=None):
    x = _outlier_x(rng, M, K, n_out, fixed_gain)
    w = rng.normal(0.0, 0.02, size=(K, N))
    b = rng.normal(0.0, 0.01, size=(N,))
    return _bf16(x), _bf16(w), _bf16(b)


def one_percent(K: int) -> int:
    return int(round(0.01 * K))


def custom(M: int, K: int, N: int, rank: int, fmt: str, seed: int, *, n_outliers: Optional[int] = None,
           alpha: float = 0.5, lora_rank: int = 0, name: str = "custom") -> Layer:
    """A small seeded layer with the cfg 1 recipe (used for ragged parity cases)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    n_out = one_percent(K) if n_outliers is None else n_outliers
    X, W, b = _linear_inputs(rng, M, K, N, n_out)
    layer = Layer(name, fmt, M, K, N, rank, alpha, X, W, b, seed=seed)
    if lora_rank:
        _attach_lora_inputs(layer, lora_rank, seed + 100)
    return layer


def _attach_lora_inputs(layer: Layer, r_l: int, seed: int) -> None:
    rng = np.random.Generator(np.random.PCG64(seed))
    layer.lora_A = _bf16(rng.normal(0.0, 0.01, size=(layer.K, r_l)))
    layer.lora_B = _bf16(rng.normal(0.0, 0.01, size=(r_l, layer.N)))
    layer.lora_scale = 1.0


def _gelu_erf(y: torch.Tensor) -> torch.Tensor:
    return torch.nn.functional.gelu(y, approximate="none")


def config(cfg_id: int, *, M: Optional[int] = None, rank: Optional[int] = None, fmt: Optional[str] = None,
           lora: bool = False) -> list[Layer]:
    """The layers of one configuration (two for the MLP pair configs)."""
    seed = 1000 + cfg_id
    rng = np.random.Generator(np.random.PCG64(seed))
    if cfg_id == 0:
        X, W, b = _linear_inputs(rng, 256, 512, 512, 4, fixed_gain=50.0)
        return [Layer("cfg0_single_linear", INT4_G64, 256, 512, 512, 16, 0.5, X, W, b, seed=seed)]
    if cfg_id == 1:
        Mv = 4608 if M is None else M
        X, W, b = _linear_inputs(rng, Mv, 3072, 3072, one_percent(3072))
        return [Layer("cfg1_attn_proj", fmt or INT4_G64, Mv, 3072, 3072, rank or 32, 0.5, X, W, b, seed=seed)]
    if cfg_id in (2, 3):
        seed = 1002  # cfg 3 is the cfg 2 pair in NVFP4: identical data
        rng = np.random.Generator(np.random.PCG64(seed))
        f = fmt or (INT4_G64 if cfg_id == 2 else NVFP4_G16)
        Mv = 4608 if M is None else M
        Xu, Wu, bu = _linear_inputs(rng, Mv, 3072, 12288, one_percent(3072))
        Wd = _bf16(rng.normal(0.0, 0.02, size=(12288, 3072)))
        bd = _bf16(rng.normal(0.0, 0.01, size=(3072,)))
        # the up layer's plain (unquantized) output, then exact GELU
        with torch.no_grad():
            yu = Xu.float() @ Wu.float() + bu.float()
            hd = _gelu_erf(yu).double().numpy()
        del yu
        n_out = one_percent(12288)
        ch = rng.permutation(12288)[:n_out]
        hd[:, ch] *= rng.uniform(20.0, 100.0, size=n_out)
        Xd = _bf16(hd)
        del hd
        tag = "int4" if f == INT4_G64 else "nvfp4"
        up = Layer(f"cfg{cfg_id}_mlp_up_{tag}", f, Mv, 3072, 12288, rank or 32, 0.5, Xu, Wu, bu, seed=seed)
        down = Layer(f"cfg{cfg_id}_mlp_down_{tag}", f, Mv, 12288, 3072, rank or 32, 0.5, Xd, Wd, bd, seed=seed)
        return [up, down]
    if cfg_id == 4:
        Mv = 4096 if M is None else M
        if Mv not in SWEEP_M:
            raise ValueError(f"sweep M must be one of {SWEEP_M}")
        r = 32 if rank is None else rank
        if r not in SWEEP_R:
            raise ValueError(f"sweep rank must be one of {SWEEP_R}")
        rng = np.random.Generator(np.random.PCG64(seed * 100 + Mv))
        X, W, b = _linear_inputs(rng, Mv, 3072, 3072, one_percent(3072))
        layer = Layer(f"cfg4_sweep_M{Mv}_r{r}", fmt or NVFP4_G16, Mv, 3072, 3072, r, 0.5, X, W, b, seed=seed)
        if lora:
            _attach_lora_inputs(layer, 32, 1104)
        return [layer]
    raise ValueError(f"unknown config {cfg_id}")


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a bfloat16/float32 CPU tensor."""
    return t.detach().to(torch.float64).cpu().numpy()
