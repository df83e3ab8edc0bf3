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
