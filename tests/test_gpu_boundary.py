"""Boundary failures on a B200, injected on the host (msModelSlim SVDQuant entry,
section 2.6, usage restrictions; the limits include/svdq.h states).

Every refused call must return its status, launch nothing (Y untouched) and
leave the layer usable; every allocation failure inside an allocating call
must unwind without leaking device memory or handing out a handle. Nothing
here faults, traps or hangs a GPU: the failures are bad arguments and a
library allocation made to fail by the test hook svdq_debug_fail_allocation.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads
from parity import Y_TOL, bf16_tensor, f64, gpu_prepare, oracle_case, rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def small():
    case = oracle_case(workloads.custom(160, 256, 128, 16, workloads.NVFP4_G16, seed=91))
    g = gpu_prepare(case)
    yield case, g
    g.close()


def _fwd(g, X, M, Y, ws, nbytes):
    import rank_gemm_quantize_b200 as rq
    return rq.lib().svdq_linear_forward(g._h, X, M, Y, ws, nbytes, torch.cuda.current_stream().cuda_stream)


def _sentinel(M, N):
    return torch.full((M, N), 3.0, dtype=torch.bfloat16, device="cuda")


def _still_works(case, g):
    Y = g.forward(case.layer.X.cuda())
    torch.cuda.synchronize()
    assert rel(f64(Y), case.r.Y) <= Y_TOL


def test_refused_forwards_launch_nothing(small):
    import rank_gemm_quantize_b200 as rq
    case, g = small
    L = case.layer
    X = L.X.cuda()
    need = g.workspace_size(L.M)
    ws = torch.empty(need + 512, dtype=torch.uint8, device="cuda")
    Y = _sentinel(L.M, L.N)
    bad = [
        (X.data_ptr(), L.M, Y.data_ptr(), ws.data_ptr(), need - 1),          # workspace too small
        (X.data_ptr() + 2, L.M, Y.data_ptr(), ws.data_ptr(), need),           # X misaligned
        (X.data_ptr(), L.M, Y.data_ptr() + 8, ws.data_ptr(), need),           # Y misaligned
        (X.data_ptr(), L.M, Y.data_ptr(), ws.data_ptr() + 16, need),          # workspace not 256-aligned
        (X.data_ptr(), 0, Y.data_ptr(), ws.data_ptr(), need),                 # M < 1
        (None, L.M, Y.data_ptr(), ws.data_ptr(), need),                       # NULL X
    ]
    for args in bad:
        assert _fwd(g, *args) == rq.Status.INVALID_ARG, args
    torch.cuda.synchronize()
    assert bool(torch.all(Y == 3.0)), "a refused call wrote Y"
    assert g.device_status() == rq.Status.OK
    _still_works(case, g)


def test_binding_checks_shapes_dtypes_and_placement(small):
    case, g = small
    L = case.layer
    X = L.X.cuda()
    with pytest.raises(ValueError):
        g.forward(X[:, :128].contiguous())                       # wrong K
    with pytest.raises(ValueError):
        g.forward(X.float())                                     # wrong dtype
    with pytest.raises(ValueError):
        g.forward(torch.cat([X, X], 1)[:, ::2])                  # strided view
    with pytest.raises(ValueError):
        g.forward(X, out=torch.empty(L.M, L.N + 16, dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError):
        g.forward(X.cpu())                                       # not on the layer's device
    with pytest.raises(ValueError):
        g.forward_noalloc(X[:, :128].contiguous())


def test_attach_beyond_the_rank_limit_leaves_the_layer_unchanged(small):
    import rank_gemm_quantize_b200 as rq
    case, g = small
    L = case.layer
    before = g.export()
    A = torch.zeros(L.K, 256 - L.rank + 1, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(256 - L.rank + 1, L.N, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rq.SvdqError) as e:
        g.attach_lora(A, B)
    assert e.value.status == rq.Status.INVALID_ARG
    after = g.export()
    for k in ("L1", "L2", "codes_packed", "scales"):
        assert np.array_equal(before[k], after[k])
    _still_works(case, g)


@pytest.mark.skipif(torch.cuda.device_count() < 2, reason="needs a second device to make current")
def test_calls_on_another_device_are_refused(small):
    import rank_gemm_quantize_b200 as rq
    case, g = small
    with torch.cuda.device(1):
        X = case.layer.X.cuda(1)
        Y = torch.empty(case.layer.M, case.layer.N, dtype=torch.bfloat16, device="cuda:1")
        ws = torch.empty(g.workspace_size(case.layer.M), dtype=torch.uint8, device="cuda:1")
        assert _fwd(g, X.data_ptr(), case.layer.M, Y.data_ptr(), ws.data_ptr(), ws.numel()) == rq.Status.INVALID_ARG
        assert b"device" in rq.lib().svdq_last_error()


def _free_bytes():
    torch.cuda.synchronize()
    return torch.cuda.mem_get_info()[0]


def test_allocation_failures_unwind_without_leaks():
    """Fail the library's 1st, 2nd, ... device allocation inside prepare (with
    given factors), attach and the activation inspection call: each returns
    SVDQ_ERR_OOM, hands out no handle, leaves an existing layer unchanged, and
    the device's free memory comes back to where it started."""
    import rank_gemm_quantize_b200 as rq
    lib = rq.lib()
    case = oracle_case(workloads.custom(130, 384, 160, 24, workloads.INT4_G64, seed=92))
    L = case.layer
    W, bias, a = L.W.cuda(), L.bias.cuda(), torch.from_numpy(case.a).cuda()
    L1, L2 = bf16_tensor(case.p.L1), bf16_tensor(case.p.L2)
    cfg = rq._Config(L.K, L.N, L.rank, L.alpha, 1e-5, 0)
    stream = torch.cuda.current_stream().cuda_stream
    free0 = _free_bytes()
    failures = 0
    try:
        for idx in range(64):
            lib.svdq_debug_fail_allocation(idx)
            out = ctypes.c_void_p()
            st = lib.svdq_prepare_weights_with_factors(ctypes.byref(cfg), W.data_ptr(), bias.data_ptr(), a.data_ptr(),
                                                       L1.data_ptr(), L2.data_ptr(), stream, ctypes.byref(out))
            lib.svdq_debug_fail_allocation(-1)
            if st == rq.Status.OK:
                lib.svdq_destroy(out)
                break
            assert st == rq.Status.OOM, (idx, st, lib.svdq_last_error())
            assert out.value is None
            failures += 1
        else:
            pytest.fail("prepare never succeeded")
        assert failures >= 5  # every allocation of prepare was made to fail once
        assert abs(_free_bytes() - free0) < (8 << 20)

        g = gpu_prepare(case)
        try:
            before = g.export()
            lA = torch.zeros(L.K, 8, dtype=torch.bfloat16, device="cuda")
            lB = torch.zeros(8, L.N, dtype=torch.bfloat16, device="cuda")
            for idx in range(32):
                lib.svdq_debug_fail_allocation(idx)
                try:
                    slot = g.attach_lora(lA, lB)
                except rq.SvdqError as err:
                    assert err.status == rq.Status.OOM
                    continue
                finally:
                    lib.svdq_debug_fail_allocation(-1)
                assert idx >= 6  # the adapter's factors and the four branch buffers each failed once
                g.detach_lora(slot)
                break
            after = g.export()
            for k in ("L1", "L2", "codes_packed", "scales"):
                assert np.array_equal(before[k], after[k])
            assert after["rank"] == before["rank"]
            lib.svdq_debug_fail_allocation(0)
            try:
                g.quantize_activations(L.X.cuda())
                hook_hit = False  # the K split was 1: no scratch to allocate
            except rq.SvdqError as err:
                hook_hit = True
                assert err.status == rq.Status.OOM
            finally:
                lib.svdq_debug_fail_allocation(-1)
            _still_works(case, g)
        finally:
            g.close()
        assert abs(_free_bytes() - free0) < (8 << 20)
    finally:
        lib.svdq_debug_fail_allocation(-1)
