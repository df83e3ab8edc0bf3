"""Several LoRA adapters on one prepared layer, on a B200 ("SVDQuant",
abstract: off-the-shelf LoRAs without re-quantization).

* Adapters take slots; the branch is the base factors followed by the occupied
  slots in slot order, and the residual's codes and scales never change.
* Detaching an adapter gives back, byte for byte, the branch the layer had
  without it (the exported factors and the forward's output bits).
* Per-row selection: row m uses the adapters whose slot bits are set in its
  mask, checked element-wise against the oracle's definition (the base output
  plus each selected adapter's branch product).
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import formats as F
from oracle import svdquant as S
from parity import Y_TOL, bf16_tensor, f64, gpu_prepare, oracle_case, rel

pytestmark = pytest.mark.gpu


def _adapters(K, N, seed, ranks):
    rng = np.random.Generator(np.random.PCG64(seed))
    return [(F.bf16_round(rng.normal(0, 0.01, (K, r))), F.bf16_round(rng.normal(0, 0.01, (r, N)))) for r in ranks]


@pytest.mark.parametrize("fmt", workloads.FORMATS)
def test_slots_detach_and_per_row_selection(fmt):
    layer = workloads.custom(300, 512, 384, 32, fmt, seed=101)
    case = oracle_case(layer)
    p = case.p
    ads = _adapters(layer.K, layer.N, 102, [16, 8, 24])
    scales = [0.5, 1.0, 2.0]
    g = gpu_prepare(case)
    try:
        X = layer.X.cuda()
        ex0 = g.export()
        y0 = g.forward(X).clone()
        slots = [g.attach_lora(bf16_tensor(A), bf16_tensor(B), sc) for (A, B), sc in zip(ads, scales)]
        assert slots == [0, 1, 2]
        info = g.info()
        assert info.rank == 32 + 16 + 8 + 24 and info.adapter_slots == 0b111
        assert info.adapter_col_start[:4] == (32, 48, 56, 80)
        ex = g.export()
        assert np.array_equal(ex["codes_packed"], ex0["codes_packed"]) and np.array_equal(ex["scales"], ex0["scales"])
        q = p
        for (A, B), sc in zip(ads, scales):
            q = S.attach_lora(q, A, B, sc)
        assert np.array_equal(ex["L1"], q.L1) and np.array_equal(ex["L2"], q.L2)

        # every row with every adapter: the concatenated layer
        Y = g.forward(X)
        torch.cuda.synchronize()
        assert rel(f64(Y), S.forward(q, case.X).Y) <= Y_TOL

        # per-row selection
        rng = np.random.Generator(np.random.PCG64(103))
        mask = rng.integers(0, 8, size=layer.M).astype(np.int32)
        mask[:4] = [0, 1, 2, 7]
        factors = {s: S.lora_factors(p, A, B, sc) for s, ((A, B), sc) in zip(slots, zip(ads, scales))}
        want = S.forward_selected(p, factors, case.X, mask)
        Ym = g.forward_masked(X, torch.from_numpy(mask).cuda())
        torch.cuda.synchronize()
        ym = f64(Ym)
        assert rel(ym, want) <= Y_TOL
        for m in range(layer.M):  # row by row too: each row's own error stays in bounds
            assert rel(ym[m], want[m]) <= 2 * Y_TOL, m
        # a row that selects nothing gives the layer without adapters (the
        # adapters' T columns are zero; only the wider branch contraction's
        # rounding may differ, within one bf16 unit)
        assert torch.allclose(Ym[0].float(), y0[0].float(), rtol=2 ** -7, atol=1e-6)

        # detach the middle adapter: slots 0 and 2 stay, the layout closes up
        g.detach_lora(1)
        info = g.info()
        assert info.adapter_slots == 0b101 and info.rank == 32 + 16 + 24
        ex1 = g.export()
        q02 = S.attach_lora(S.attach_lora(p, *ads[0], scales[0]), *ads[2], scales[2])
        assert np.array_equal(ex1["L1"], q02.L1) and np.array_equal(ex1["L2"], q02.L2)
        # the freed slot is reused first
        assert g.attach_lora(bf16_tensor(ads[1][0]), bf16_tensor(ads[1][1]), scales[1]) == 1
        g.detach_lora(1)
        g.detach_lora(2)
        g.detach_lora(0)
        # back to the layer as prepared: byte for byte
        ex2 = g.export()
        for k in ("L1", "L2", "codes_packed", "scales", "s", "inv_s", "bias"):
            assert np.array_equal(ex2[k], ex0[k]), k
        y2 = g.forward(X)
        torch.cuda.synchronize()
        assert torch.equal(y2, y0)
        assert g.info().adapter_slots == 0
        with pytest.raises(Exception):
            g.detach_lora(0)  # empty slot
    finally:
        g.close()


def test_slot_limit_and_rank_zero_base():
    """A rank-0 layer (no SVD branch) takes adapters too; a ninth adapter is
    refused and leaves the layer as it was."""
    import rank_gemm_quantize_b200 as rq
    layer = workloads.custom(130, 256, 128, 0, workloads.INT4_G64, seed=104)
    case = oracle_case(layer)
    g = gpu_prepare(case)
    try:
        ads = _adapters(layer.K, layer.N, 105, [4] * 9)
        for i in range(8):
            assert g.attach_lora(bf16_tensor(ads[i][0]), bf16_tensor(ads[i][1]), 1.0) == i
        before = g.export()
        with pytest.raises(rq.SvdqError) as e:
            g.attach_lora(bf16_tensor(ads[8][0]), bf16_tensor(ads[8][1]), 1.0)
        assert e.value.status == rq.Status.INVALID_ARG
        after = g.export()
        assert np.array_equal(before["L1"], after["L1"]) and after["rank"] == 32
        q = case.p
        for A, B in ads[:8]:
            q = S.attach_lora(q, A, B, 1.0)
        Y = g.forward(layer.X.cuda())
        torch.cuda.synchronize()
        assert rel(f64(Y), S.forward(q, case.X).Y) <= Y_TOL
        mask = np.full(layer.M, 0b100, dtype=np.int32)  # adapter 2 alone
        Ym = g.forward_masked(layer.X.cuda(), torch.from_numpy(mask).cuda())
        torch.cuda.synchronize()
        want = S.forward_selected(case.p, {2: S.lora_factors(case.p, *ads[2], 1.0)}, case.X, mask)
        assert rel(f64(Ym), want) <= Y_TOL
    finally:
        g.close()
