"""The forward entry point that allocates nothing (svdq_linear_forward_noalloc).

It serves callers that may not allocate device memory themselves, such as a
host whose device memory belongs to its own allocator. It must give the same
result as svdq_linear_forward with a caller workspace, call after call (its
scratch array keeps the previous call's contents), and refuse a layer whose
workspace would not fit the fixed scratch. Collected last so a run that stops
at the first failure has already run every other test; it also passes alone
in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads
from parity import Y_TOL, f64, gpu_prepare, oracle_case, rel

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20


def _noalloc(g, X, Y):
    import rank_gemm_quantize_b200 as rq
    return rq.lib().svdq_linear_forward_noalloc(g._h, X.data_ptr(), X.shape[0], Y.data_ptr(),
                                                torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("name", ["cfg0_int4", "ragged_nvfp4", "cfg1_int4"])
def test_noalloc_matches_workspace_forward_twice(name):
    layer = {
        "cfg0_int4": lambda: workloads.config(0)[0],
        "ragged_nvfp4": lambda: workloads.custom(129, 384, 144, 40, workloads.NVFP4_G16, seed=72),
        "cfg1_int4": lambda: workloads.config(1)[0],
    }[name]()
    case = oracle_case(layer)
    g = gpu_prepare(case)
    try:
        X = layer.X.cuda()
        ref = g.forward(X)  # the existing entry point, caller-provided workspace
        torch.cuda.synchronize()
        y_ref = f64(ref)
        for call in range(2):  # the scratch keeps the previous call's contents
            Y = torch.full((layer.M, layer.N), float("nan"), dtype=torch.bfloat16, device="cuda")
            assert _noalloc(g, X, Y) == 0
            torch.cuda.synchronize()
            y = f64(Y)
            assert np.all(np.isfinite(y)), f"call {call}"
            assert rel(y, y_ref) <= Y_TOL, f"call {call}"
        assert rel(y, case.r.Y) <= Y_TOL
        assert g.device_status() == 0
    finally:
        g.close()


def test_noalloc_refuses_a_workspace_beyond_the_scratch():
    import rank_gemm_quantize_b200 as rq
    layer = workloads.config(0)[0]  # K = N = 512
    case = oracle_case(layer)
    g = gpu_prepare(case)
    try:
        M = 80000  # workspace for M x 512 INT4 codes alone is ~41 MB
        assert g.workspace_size(M) > SCRATCH_BYTES
        X = torch.zeros(M, layer.K, dtype=torch.bfloat16, device="cuda")
        Y = torch.zeros(M, layer.N, dtype=torch.bfloat16, device="cuda")
        st = _noalloc(g, X, Y)
        assert st == rq.Status.INVALID_ARG
        assert b"scratch" in rq.lib().svdq_last_error()
        # the refusal launched nothing: Y is untouched and the layer still works
        torch.cuda.synchronize()
        assert int(torch.count_nonzero(Y)) == 0
        Y2 = g.forward_noalloc(layer.X.cuda())
        torch.cuda.synchronize()
        assert rel(f64(Y2), case.r.Y) <= Y_TOL
    finally:
        g.close()


@pytest.mark.parametrize("fmt", workloads.FORMATS)
def test_attention_projection_at_rank_128_fits_the_scratch(fmt):
    """The fixed scratch covers the 4608 x 3072 x 3072 attention projection up
    to rank 128 in both formats (the activation kernel's K split, which sets
    the size of its float partials, included)."""
    import rank_gemm_quantize_b200 as rq
    M, K, N, r = 4608, 3072, 3072, 128
    gen = torch.Generator(device="cpu").manual_seed(5)
    W = (torch.randn(K, N, generator=gen) * 0.02).to(torch.bfloat16).cuda()
    L1 = (torch.randn(K, r, generator=gen) * 0.02).to(torch.bfloat16).cuda()
    L2 = (torch.randn(r, N, generator=gen) * 0.02).to(torch.bfloat16).cuda()
    a = torch.ones(K, dtype=torch.float32, device="cuda")
    g = rq.Layer.prepare(W, None, a, fmt, r, factors=(L1, L2))
    try:
        need = g.workspace_size(M)
        assert need <= SCRATCH_BYTES, need
        Y = g.forward_noalloc(torch.zeros(M, K, dtype=torch.bfloat16, device="cuda"))
        torch.cuda.synchronize()
        assert int(torch.count_nonzero(Y)) == 0  # zero input, no bias: Y = 0
    finally:
        g.close()
