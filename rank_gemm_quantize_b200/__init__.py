"""Python binding of the SVDQuant W4A4 + low-rank linear layer for B200 (sm_100a).

Argument marshalling only: every step of the layer runs in the CUDA kernels of
``libsvdq.so`` (built in-tree by ``rank_gemm_quantize_b200.build``), reached
through the C ABI declared in ``include/svdq.h``. PyTorch is used for device
memory and the current CUDA stream; there is no CPU or PyTorch fallback -
importing this module without the built library raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from enum import IntEnum
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsvdq.so")

INT4_G64 = "int4_g64"
NVFP4_G16 = "nvfp4_g16"
_FMT = {INT4_G64: 0, NVFP4_G16: 1}
_FMT_NAME = {0: INT4_G64, 1: NVFP4_G16}


class Status(IntEnum):
    OK = 0
    INVALID_ARG = 1
    UNSUPPORTED = 2
    OOM = 3
    CUDA = 4
    NUMERIC = 5
    DEVICE_TIMEOUT = 6


class SvdqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{Status(status).name}: {message}")
        self.status = Status(status)


NO_SMOOTHING = 1  # svdq_config.flags: s = 1 for every channel
MAX_ADAPTERS = 8


class _Config(ctypes.Structure):
    _fields_ = [("K", ctypes.c_int), ("N", ctypes.c_int), ("rank", ctypes.c_int), ("alpha", ctypes.c_float),
                ("s_min", ctypes.c_float), ("fmt", ctypes.c_int), ("flags", ctypes.c_uint)]


class _Info(ctypes.Structure):
    _fields_ = [("K", ctypes.c_int), ("N", ctypes.c_int), ("rank", ctypes.c_int), ("rank_pad", ctypes.c_int),
                ("fmt", ctypes.c_int), ("alpha", ctypes.c_float), ("g_x", ctypes.c_float), ("g_w", ctypes.c_float),
                ("t_scale", ctypes.c_float), ("base_rank", ctypes.c_int), ("flags", ctypes.c_uint),
                ("adapter_slots", ctypes.c_uint), ("adapter_col_start", ctypes.c_int * (MAX_ADAPTERS + 1))]


class _BlobHeader(ctypes.Structure):
    _fields_ = [("magic", ctypes.c_uint32), ("version", ctypes.c_uint32), ("fmt", ctypes.c_int32),
                ("K", ctypes.c_int32), ("N", ctypes.c_int32), ("rank", ctypes.c_int32), ("alpha", ctypes.c_float),
                ("g_x", ctypes.c_float), ("g_w", ctypes.c_float), ("reserved", ctypes.c_float),
                ("off_s", ctypes.c_uint64), ("off_inv_s", ctypes.c_uint64), ("off_L1", ctypes.c_uint64),
                ("off_L2", ctypes.c_uint64), ("off_codes", ctypes.c_uint64), ("off_scales", ctypes.c_uint64),
                ("off_bias", ctypes.c_uint64), ("total", ctypes.c_uint64)]


# Every symbol include/svdq.h declares, with its ctypes signature.
_VP, _I, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "svdq_calibrate_absmax": [_VP, _I, _I, _VP, _VP],
    "svdq_prepare_weights": [ctypes.POINTER(_Config), _VP, _VP, _VP, _VP, ctypes.POINTER(_VP)],
    "svdq_prepare_weights_with_factors": [ctypes.POINTER(_Config), _VP, _VP, _VP, _VP, _VP, _VP, ctypes.POINTER(_VP)],
    "svdq_workspace_size": [_VP, _I, ctypes.POINTER(_SZ)],
    "svdq_linear_forward": [_VP, _VP, _I, _VP, _VP, _SZ, _VP],
    "svdq_linear_forward_profiled": [_VP, _VP, _I, _VP, _VP, _SZ, _VP, ctypes.POINTER(_VP)],
    "svdq_linear_forward_noalloc": [_VP, _VP, _I, _VP, _VP],
    "svdq_linear_forward_masked": [_VP, _VP, _I, _VP, _VP, _SZ, _VP, _VP],
    "svdq_attach_lora": [_VP, _VP, _VP, _I, _F, _VP, ctypes.POINTER(_I)],
    "svdq_detach_lora": [_VP, _I, _VP],
    "svdq_quantize_activations": [_VP, _VP, _I, _VP, _VP, _VP, _VP],
    "svdq_export_weights": [_VP, _VP, ctypes.POINTER(_SZ), _VP],
    "svdq_layer_get_info": [_VP, ctypes.POINTER(_Info)],
    "svdq_device_status": [_VP, _VP],
    "svdq_destroy": [_VP],
    "svdq_last_error": [],
    "svdq_selftest_bounded_wait": [ctypes.c_ulonglong, _VP],
    "svdq_debug_fail_allocation": [ctypes.c_longlong],
    "svdq_mlp_workspace_size": [_VP, _VP, _I, ctypes.POINTER(_SZ)],
    "svdq_mlp_workspace_layout": [_VP, _VP, _I, ctypes.POINTER(_SZ)],
    "svdq_mlp_forward": [_VP, _VP, _VP, _I, _VP, _VP, _SZ, _VP],
    "svdq_mlp_forward_profiled": [_VP, _VP, _VP, _I, _VP, _VP, _SZ, _VP, ctypes.POINTER(_VP)],
    "svdq_w4a16_prepare": [_VP, _VP, _I, _I, _VP, ctypes.POINTER(_VP)],
    "svdq_w4a16_forward": [_VP, _VP, _I, _VP, _VP],
    "svdq_w4a16_export": [_VP, _VP, _VP, _VP],
    "svdq_w4a16_destroy": [_VP],
}


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libsvdq.so and declares its C ABI. Raises if it is missing."""
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m rank_gemm_quantize_b200.build`")
    lib = ctypes.CDLL(path)
    for name, args in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = {"svdq_last_error": ctypes.c_char_p, "svdq_debug_fail_allocation": None}.get(name, ctypes.c_int)
    return lib


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = load_library()
    return _lib


def _check(status: int) -> None:
    if status != 0:
        raise SvdqError(status, lib().svdq_last_error().decode())


def _stream(stream=None) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensors must be contiguous CUDA tensors")
    return t.data_ptr()


def calibrate_absmax(X: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """A_scale (per input channel absolute maximum) folded into `out` (float32 [K])."""
    M, K = X.shape
    if out is None:
        out = torch.zeros(K, dtype=torch.float32, device=X.device)
    _check(lib().svdq_calibrate_absmax(_ptr(X), M, K, _ptr(out), _stream(stream)))
    return out


def selftest_bounded_wait(limit_ns: int = 50_000_000, stream=None) -> Status:
    st = lib().svdq_selftest_bounded_wait(limit_ns, _stream(stream))
    return Status(st)


@dataclass
class LayerInfo:
    K: int
    N: int
    rank: int
    rank_pad: int
    fmt: str
    alpha: float
    g_x: float
    g_w: float
    t_scale: float
    base_rank: int = 0
    flags: int = 0
    adapter_slots: int = 0
    adapter_col_start: tuple = ()


class Layer:
    """A prepared SVDQuant linear layer (owns its device buffers)."""

    def __init__(self, handle: int, device: Optional[torch.device] = None):
        self._h = ctypes.c_void_p(handle)
        self._ws: Optional[torch.Tensor] = None
        self._info: Optional[LayerInfo] = None
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else device

    @classmethod
    def prepare(cls, W: torch.Tensor, bias: Optional[torch.Tensor], act_absmax: torch.Tensor, fmt: str, rank: int,
                alpha: float = 0.5, s_min: float = 1e-5, factors=None, smooth: bool = True, stream=None) -> "Layer":
        """Offline preparation; rank 0 gives the smoothing-only layer, smooth=False
        keeps s = 1 (both ablations of the method)."""
        K, N = W.shape
        cfg = _Config(K, N, rank, alpha, s_min, _FMT[fmt], 0 if smooth else NO_SMOOTHING)
        out = ctypes.c_void_p()
        if factors is None:
            st = lib().svdq_prepare_weights(ctypes.byref(cfg), _ptr(W), _ptr(bias), _ptr(act_absmax), _stream(stream),
                                            ctypes.byref(out))
        else:
            L1, L2 = factors
            st = lib().svdq_prepare_weights_with_factors(ctypes.byref(cfg), _ptr(W), _ptr(bias), _ptr(act_absmax),
                                                         _ptr(L1), _ptr(L2), _stream(stream), ctypes.byref(out))
        _check(st)
        return cls(out.value, W.device)

    def info(self) -> LayerInfo:
        if self._info is None:
            i = _Info()
            _check(lib().svdq_layer_get_info(self._h, ctypes.byref(i)))
            self._info = LayerInfo(i.K, i.N, i.rank, i.rank_pad, _FMT_NAME[i.fmt], i.alpha, i.g_x, i.g_w, i.t_scale,
                                   i.base_rank, i.flags, i.adapter_slots, tuple(i.adapter_col_start))
        return self._info

    def workspace_size(self, M: int) -> int:
        n = ctypes.c_size_t()
        _check(lib().svdq_workspace_size(self._h, M, ctypes.byref(n)))
        return n.value

    def _check_io(self, X: torch.Tensor, out: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None) -> int:
        """The shapes, dtypes and placement the C ABI assumes; the library reads
        X through a tensor map built from the layer's K, so a narrower or
        strided X would be read past its end."""
        info = self.info()
        if X.dim() != 2 or X.shape[1] != info.K:
            raise ValueError(f"X must be [M, {info.K}], got {tuple(X.shape)}")
        if X.dtype != torch.bfloat16 or not X.is_contiguous():
            raise ValueError("X must be a contiguous bfloat16 tensor")
        if X.device != self.device:
            raise ValueError(f"X is on {X.device}, the layer on {self.device}")
        if out is not None:
            if tuple(out.shape) != (X.shape[0], info.N) or out.dtype != torch.bfloat16 or not out.is_contiguous():
                raise ValueError(f"out must be a contiguous bfloat16 [{X.shape[0]}, {info.N}] tensor")
            if out.device != self.device:
                raise ValueError(f"out is on {out.device}, the layer on {self.device}")
        if workspace is not None:
            if workspace.dtype != torch.uint8 or not workspace.is_contiguous() or workspace.device != self.device:
                raise ValueError("workspace must be a contiguous uint8 tensor on the layer's device")
        return info.N

    def workspace(self, M: int, device=None) -> torch.Tensor:
        need = self.workspace_size(M)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=device or "cuda")
        return self._ws

    def forward(self, X: torch.Tensor, out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
        N = self._check_io(X, out, workspace)
        M = X.shape[0]
        if out is None:
            out = torch.empty(M, N, dtype=torch.bfloat16, device=X.device)
        ws = workspace if workspace is not None else self.workspace(M, X.device)
        _check(lib().svdq_linear_forward(self._h, _ptr(X), M, _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))
        return out

    __call__ = forward

    def forward_noalloc(self, X: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """forward() on the library's fixed scratch array (no workspace, no allocation by the library)."""
        N = self._check_io(X, out)
        M = X.shape[0]
        if out is None:
            out = torch.empty(M, N, dtype=torch.bfloat16, device=X.device)
        _check(lib().svdq_linear_forward_noalloc(self._h, _ptr(X), M, _ptr(out), _stream(stream)))
        return out

    def forward_profiled(self, X: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor, events, stream=None):
        """forward() recording three torch.cuda.Event objects around its two kernels."""
        self._check_io(X, out, workspace)
        arr = (ctypes.c_void_p * 3)(*[e.cuda_event for e in events])
        _check(lib().svdq_linear_forward_profiled(self._h, _ptr(X), X.shape[0], _ptr(out), _ptr(workspace),
                                                  workspace.numel(), _stream(stream), arr))
        return out

    def quantize_activations(self, X: torch.Tensor, stream=None):
        """(codes, scales, T) of the activation kernel in its documented layouts."""
        info = self.info()
        M, K = X.shape
        M_pad = (M + 127) // 128 * 128
        dev = X.device
        if info.fmt == INT4_G64:
            codes = torch.empty(M_pad, K, dtype=torch.uint8, device=dev)
            scales = torch.empty(K // 64, M_pad, dtype=torch.float32, device=dev)
        else:
            codes = torch.empty(M_pad, K // 2, dtype=torch.uint8, device=dev)
            scales = torch.empty(M_pad // 128 * (K // 64) * 512, dtype=torch.uint8, device=dev)
        T = torch.empty(M_pad, info.rank_pad, dtype=torch.bfloat16, device=dev)
        _check(lib().svdq_quantize_activations(self._h, _ptr(X), M, _ptr(codes), _ptr(scales),
                                               _ptr(T) if info.rank_pad else None, _stream(stream)))
        return codes, scales, T

    def attach_lora(self, A: torch.Tensor, B: torch.Tensor, scale: float = 1.0, stream=None) -> int:
        """Adds scale * X A B to the branch; returns the adapter's slot."""
        self._info = None
        slot = ctypes.c_int(-1)
        _check(lib().svdq_attach_lora(self._h, _ptr(A), _ptr(B), A.shape[1], scale, _stream(stream),
                                      ctypes.byref(slot)))
        return slot.value

    def detach_lora(self, slot: int, stream=None) -> None:
        """Removes the adapter in `slot` (the branch returns to what it was without it)."""
        self._info = None
        _check(lib().svdq_detach_lora(self._h, slot, _stream(stream)))

    def forward_masked(self, X: torch.Tensor, row_adapter_mask: torch.Tensor, out: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """forward() where row m uses the adapters whose slot bits are set in
        row_adapter_mask[m] (int32/uint32 [M] on the layer's device)."""
        N = self._check_io(X, out, workspace)
        M = X.shape[0]
        if (row_adapter_mask.dim() != 1 or row_adapter_mask.shape[0] != M or row_adapter_mask.element_size() != 4
                or row_adapter_mask.device != self.device or not row_adapter_mask.is_contiguous()):
            raise ValueError("row_adapter_mask must be a contiguous 32-bit [M] tensor on the layer's device")
        if out is None:
            out = torch.empty(M, N, dtype=torch.bfloat16, device=X.device)
        ws = workspace if workspace is not None else self.workspace(M, X.device)
        _check(lib().svdq_linear_forward_masked(self._h, _ptr(X), M, _ptr(out), _ptr(ws), ws.numel(),
                                                _ptr(row_adapter_mask), _stream(stream)))
        return out

    def export(self, stream=None) -> dict:
        """Canonical prepared weights (numpy arrays)."""
        n = ctypes.c_size_t()
        _check(lib().svdq_export_weights(self._h, None, ctypes.byref(n), _stream(stream)))
        buf = (ctypes.c_uint8 * n.value)()
        _check(lib().svdq_export_weights(self._h, ctypes.cast(buf, ctypes.c_void_p), ctypes.byref(n), _stream(stream)))
        raw = np.frombuffer(buf, dtype=np.uint8).copy()
        hd = _BlobHeader.from_buffer_copy(raw[:ctypes.sizeof(_BlobHeader)].tobytes())
        K, N, r = hd.K, hd.N, hd.rank

        def sec(off, dtype, shape):
            cnt = int(np.prod(shape))
            return raw[off:off + cnt * np.dtype(dtype).itemsize].view(dtype).reshape(shape).copy()

        bf = lambda a: (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        out = {
            "fmt": _FMT_NAME[hd.fmt], "K": K, "N": N, "rank": r, "alpha": hd.alpha,
            "g_x": np.float32(hd.g_x), "g_w": np.float32(hd.g_w),
            "s": sec(hd.off_s, np.float32, (K,)), "inv_s": sec(hd.off_inv_s, np.float32, (K,)),
            "L1": bf(sec(hd.off_L1, np.uint16, (K, r))), "L2": bf(sec(hd.off_L2, np.uint16, (r, N))),
            "codes_packed": sec(hd.off_codes, np.uint8, (N, K // 2)),
            "bias": bf(sec(hd.off_bias, np.uint16, (N,))),
        }
        if hd.fmt == 0:
            out["scales"] = sec(hd.off_scales, np.float32, (N, K // 64))
        else:
            out["scales"] = sec(hd.off_scales, np.uint8, (N, K // 16))
        return out

    def device_status(self, stream=None) -> Status:
        return Status(lib().svdq_device_status(self._h, _stream(stream)))

    def close(self) -> None:
        if self._h is not None and self._h.value:
            lib().svdq_destroy(self._h)
        self._h = None
        self._ws = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class WeightOnlyLayer:
    """The 4-bit weight-only (W4A16) baseline: INT4 group-64 weights, bf16
    activations, dequantized on chip (include/svdq.h, svdq_w4a16_*)."""

    def __init__(self, W: torch.Tensor, bias: Optional[torch.Tensor] = None, stream=None):
        if W.dim() != 2 or W.dtype != torch.bfloat16 or not W.is_cuda or not W.is_contiguous():
            raise ValueError("W must be a contiguous bfloat16 CUDA tensor [K, N]")
        self.K, self.N = W.shape
        self.device = W.device
        out = ctypes.c_void_p()
        _check(lib().svdq_w4a16_prepare(_ptr(W), _ptr(bias), self.K, self.N, _stream(stream), ctypes.byref(out)))
        self._h = out

    def forward(self, X: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        if X.dim() != 2 or X.shape[1] != self.K or X.dtype != torch.bfloat16 or not X.is_contiguous() \
                or X.device != self.device:
            raise ValueError(f"X must be a contiguous bfloat16 [M, {self.K}] tensor on {self.device}")
        M = X.shape[0]
        if out is None:
            out = torch.empty(M, self.N, dtype=torch.bfloat16, device=X.device)
        elif tuple(out.shape) != (M, self.N) or out.dtype != torch.bfloat16 or not out.is_contiguous():
            raise ValueError(f"out must be a contiguous bfloat16 [{M}, {self.N}] tensor")
        _check(lib().svdq_w4a16_forward(self._h, _ptr(X), M, _ptr(out), _stream(stream)))
        return out

    __call__ = forward

    def export(self, stream=None):
        """(codes uint8 [N, K/2] packed nibbles, scales float32 [K/64, N])."""
        codes = np.zeros((self.N, self.K // 2), dtype=np.uint8)
        scales = np.zeros((self.K // 64, self.N), dtype=np.float32)
        _check(lib().svdq_w4a16_export(self._h, codes.ctypes.data, scales.ctypes.data, _stream(stream)))
        return codes, scales

    def close(self) -> None:
        if self._h is not None and self._h.value:
            lib().svdq_w4a16_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class MlpBlock:
    """Y = down(GELU(up(X))) for two prepared NVFP4 layers, with GELU and the
    down layer's quantization fused into the up layer's GEMM epilogue."""

    def __init__(self, up: Layer, down: Layer):
        self.up, self.down = up, down
        self._ws: Optional[torch.Tensor] = None

    def workspace_size(self, M: int) -> int:
        n = ctypes.c_size_t()
        _check(lib().svdq_mlp_workspace_size(self.up._h, self.down._h, M, ctypes.byref(n)))
        return n.value

    def workspace_layout(self, M: int):
        """(codes, scales, T) byte offsets of the down layer's activations in the workspace."""
        off = (ctypes.c_size_t * 3)()
        _check(lib().svdq_mlp_workspace_layout(self.up._h, self.down._h, M, off))
        return tuple(off)

    def workspace(self, M: int) -> torch.Tensor:
        need = self.workspace_size(M)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.up.device)
        return self._ws

    def forward(self, X: torch.Tensor, out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                stream=None, events=None) -> torch.Tensor:
        self.up._check_io(X, None, workspace)
        M = X.shape[0]
        N = self.down.info().N
        if out is None:
            out = torch.empty(M, N, dtype=torch.bfloat16, device=X.device)
        elif tuple(out.shape) != (M, N) or out.dtype != torch.bfloat16 or not out.is_contiguous():
            raise ValueError(f"out must be a contiguous bfloat16 [{M}, {N}] tensor")
        ws = workspace if workspace is not None else self.workspace(M)
        if events is None:
            _check(lib().svdq_mlp_forward(self.up._h, self.down._h, _ptr(X), M, _ptr(out), _ptr(ws), ws.numel(),
                                          _stream(stream)))
        else:
            arr = (ctypes.c_void_p * 5)(*[e.cuda_event for e in events])
            _check(lib().svdq_mlp_forward_profiled(self.up._h, self.down._h, _ptr(X), M, _ptr(out), _ptr(ws),
                                                   ws.numel(), _stream(stream), arr))
        return out

    __call__ = forward
