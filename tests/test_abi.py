"""The C-ABI library: it loads, and exports every symbol include/svdq.h declares
(no compute calls: this runs without a GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "svdq.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SVDQ_API\s+[\w\s\*]+?\b(svdq_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def libpath():
    from rank_gemm_quantize_b200 import build
    return build.build()


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("svdq_prepare_weights", "svdq_linear_forward", "svdq_attach_lora", "svdq_workspace_size",
                     "svdq_quantize_activations", "svdq_export_weights", "svdq_destroy", "svdq_last_error"):
        assert required in names


def test_library_exports_every_declared_symbol(libpath):
    out = subprocess.run(["nm", "-D", "--defined-only", libpath], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (svdq_\w+)", out))
    assert set(_declared()) <= exported, set(_declared()) - exported
    # nothing else of ours leaks out of the library
    assert all(s.startswith("svdq_") for s in exported)


def test_binding_signatures_cover_the_header(libpath):
    import rank_gemm_quantize_b200 as rq
    assert set(rq.SIGNATURES) == set(_declared())
    lib = rq.load_library(libpath)
    for name in _declared():
        assert hasattr(lib, name)
    assert lib.svdq_last_error() == b""


def test_library_is_built_for_sm100a_only():
    from rank_gemm_quantize_b200 import build
    cmd = " ".join(build.command())
    assert "arch=compute_100a,code=sm_100a" in cmd
    assert cmd.count("-gencode") == 1


def test_calls_fail_cleanly_without_arguments(libpath):
    import rank_gemm_quantize_b200 as rq
    lib = rq.load_library(libpath)
    assert lib.svdq_workspace_size(None, 16, None) == 1  # INVALID_ARG, no crash
    assert b"NULL" in lib.svdq_last_error()
    assert lib.svdq_destroy(None) == 0
    n = ctypes.c_size_t()
    assert lib.svdq_export_weights(None, None, ctypes.byref(n), None) == 1


def test_missing_library_raises(tmp_path):
    import rank_gemm_quantize_b200 as rq
    with pytest.raises(ImportError):
        rq.load_library(str(tmp_path / "nope.so"))


# ---------------------------------------------------------------- argument errors
# msModelSlim SVDQuant entry, section 2.6 (usage restrictions: 2-D linear
# weights, the rank bound) and the shape limits the header states. Every bad
# call below is refused with SVDQ_ERR_INVALID_ARG before any device work, so
# these run without a GPU. The pointers are never dereferenced.

FAKE = 0x10000  # a 16-byte-aligned address that is never touched


def _cfg(rq, K=512, N=512, rank=16, alpha=0.5, s_min=1e-5, fmt=0):
    return rq._Config(K, N, rank, alpha, s_min, fmt)


@pytest.mark.parametrize("field,value,msg", [
    ("K", 100, b"K must be"), ("K", 0, b"K must be"), ("N", 100, b"N must be"), ("rank", 257, b"rank"),
    ("rank", -1, b"rank"), ("alpha", 1.5, b"alpha"), ("s_min", 0.0, b"s_min"), ("fmt", 7, b"format"),
    ("flags", 6, b"flags"),
])
def test_prepare_refuses_bad_configurations(libpath, field, value, msg):
    import rank_gemm_quantize_b200 as rq
    lib = rq.load_library(libpath)
    cfg = _cfg(rq)
    setattr(cfg, field, value)
    out = ctypes.c_void_p(123)
    st = lib.svdq_prepare_weights(ctypes.byref(cfg), FAKE, None, FAKE, None, ctypes.byref(out))
    assert st == rq.Status.INVALID_ARG
    assert msg in lib.svdq_last_error()
    assert out.value is None  # no handle on failure


def test_prepare_refuses_rank_above_the_weight_dimensions(libpath):
    import rank_gemm_quantize_b200 as rq
    lib = rq.load_library(libpath)
    cfg = _cfg(rq, K=128, N=64, rank=100)
    out = ctypes.c_void_p()
    assert lib.svdq_prepare_weights(ctypes.byref(cfg), FAKE, None, FAKE, None, ctypes.byref(out)) == rq.Status.INVALID_ARG
    assert b"min(K, N)" in lib.svdq_last_error()


@pytest.mark.parametrize("W,bias,a", [(FAKE + 8, None, FAKE), (FAKE, FAKE + 2, FAKE), (FAKE, None, FAKE + 4)])
def test_prepare_refuses_misaligned_pointers(libpath, W, bias, a):
    import rank_gemm_quantize_b200 as rq
    lib = rq.load_library(libpath)
    cfg = _cfg(rq)
    out = ctypes.c_void_p()
    assert lib.svdq_prepare_weights(ctypes.byref(cfg), W, bias, a, None, ctypes.byref(out)) == rq.Status.INVALID_ARG
    assert b"aligned" in lib.svdq_last_error()


def test_prepare_refuses_null_inputs(libpath):
    import rank_gemm_quantize_b200 as rq
    lib = rq.load_library(libpath)
    cfg = _cfg(rq)
    out = ctypes.c_void_p()
    assert lib.svdq_prepare_weights(ctypes.byref(cfg), None, None, FAKE, None, ctypes.byref(out)) == rq.Status.INVALID_ARG
    assert lib.svdq_prepare_weights(None, FAKE, None, FAKE, None, ctypes.byref(out)) == rq.Status.INVALID_ARG
    assert lib.svdq_prepare_weights(ctypes.byref(cfg), FAKE, None, FAKE, None, None) == rq.Status.INVALID_ARG
    assert lib.svdq_prepare_weights_with_factors(ctypes.byref(cfg), FAKE, None, FAKE, None, FAKE, None,
                                                 ctypes.byref(out)) == rq.Status.INVALID_ARG


def test_forward_and_attach_refuse_a_null_layer(libpath):
    import rank_gemm_quantize_b200 as rq
    lib = rq.load_library(libpath)
    assert lib.svdq_linear_forward(None, FAKE, 16, FAKE, FAKE, 1 << 20, None) == rq.Status.INVALID_ARG
    assert lib.svdq_linear_forward_noalloc(None, FAKE, 16, FAKE, None) == rq.Status.INVALID_ARG
    assert lib.svdq_quantize_activations(None, FAKE, 16, FAKE, FAKE, FAKE, None) == rq.Status.INVALID_ARG
    assert lib.svdq_attach_lora(None, FAKE, FAKE, 8, 1.0, None, None) == rq.Status.INVALID_ARG
    assert lib.svdq_detach_lora(None, 0, None) == rq.Status.INVALID_ARG
    assert lib.svdq_linear_forward_masked(None, FAKE, 16, FAKE, FAKE, 1 << 20, FAKE, None) == rq.Status.INVALID_ARG
    assert lib.svdq_device_status(None, None) == rq.Status.INVALID_ARG


@pytest.mark.parametrize("X,M,K,out", [(None, 4, 64, FAKE), (FAKE, 0, 64, FAKE), (FAKE, 4, 64, None),
                                       (FAKE + 2, 4, 64, FAKE)])
def test_calibration_refuses_bad_arguments(libpath, X, M, K, out):
    import rank_gemm_quantize_b200 as rq
    lib = rq.load_library(libpath)
    assert lib.svdq_calibrate_absmax(X, M, K, out, None) == rq.Status.INVALID_ARG


def test_valid_prepare_without_a_device_fails_cleanly(libpath):
    """With no sm_100 device visible the call reports it (no crash, no handle)."""
    import torch

    import rank_gemm_quantize_b200 as rq
    if torch.cuda.is_available():
        pytest.skip("a GPU is visible: this checks the no-device path")
    lib = rq.load_library(libpath)
    cfg = _cfg(rq)
    out = ctypes.c_void_p()
    st = lib.svdq_prepare_weights(ctypes.byref(cfg), FAKE, None, FAKE, None, ctypes.byref(out))
    assert st in (rq.Status.UNSUPPORTED, rq.Status.CUDA)
    assert out.value is None
