"""The multi-GPU path on CPU: two gloo ranks in child processes.

The layer is token-parallel: each rank quantizes and multiplies its own rows
against its own copy of the prepared weights, and nothing crosses ranks on the
data path. That is sound because every step of the forward is row-local:
activation groups run along K inside one row, T = x_hat L1 is per row, and
the NVFP4 activation tensor scale g_x is fixed at preparation time from the
calibration statistic (a scale taken from the live batch would couple the
rows of a batch and the ranks of a job). These tests check that property on
the oracle across ranks, and the timing arithmetic bench.py runs across ranks
(the slowest rank's time; the whole job's work).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, fmt, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import workloads
        from oracle import svdquant as S

        # timing arithmetic: every rank sees the slowest rank's time
        ms = 10.0 + 5.0 * rank
        got = bench.max_over_ranks(ms, world, torch.device("cpu"))
        # token-parallel forward: rank r takes rows r::world of the batch
        layer = workloads.config(0)[0]
        layer.fmt = fmt
        X, W, b = workloads.to_f64(layer.X), workloads.to_f64(layer.W), workloads.to_f64(layer.bias)
        a = S.calibrate_absmax(X)  # calibration: offline, identical on every rank
        p = S.prepare(W, b, a, fmt, layer.alpha, layer.rank)
        rows = np.arange(rank, layer.M, world)
        r = S.forward(p, X[rows])
        parts = [None] * world
        dist.all_gather_object(parts, (rows, r.x_codes, r.x_scales, r.T, r.Y))
        q.put((rank, got, parts if rank == 0 else None, None))
    except Exception as e:  # reported to the parent, which fails the test
        q.put((rank, None, None, repr(e)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("fmt", ["int4_g64", "nvfp4_g16"])
def test_token_parallel_shards_match_the_whole_batch(fmt):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, WORLD, port, fmt, q)) for r in range(WORLD)]
    for pr in procs:
        pr.start()
    results = {}
    try:
        for _ in range(WORLD):
            rank, got, parts, err = q.get(timeout=240)
            assert err is None, f"rank {rank}: {err}"
            results[rank] = (got, parts)
    finally:
        for pr in procs:
            pr.join(timeout=60)
            if pr.is_alive():
                pr.kill()
    # the slowest rank's time everywhere
    assert [results[r][0] for r in range(WORLD)] == [10.0 + 5.0 * (WORLD - 1)] * WORLD

    import workloads
    from oracle import svdquant as S
    layer = workloads.config(0)[0]
    layer.fmt = fmt
    X, W, b = workloads.to_f64(layer.X), workloads.to_f64(layer.W), workloads.to_f64(layer.bias)
    p = S.prepare(W, b, S.calibrate_absmax(X), fmt, layer.alpha, layer.rank)
    full = S.forward(p, X)
    seen = np.zeros(layer.M, bool)
    for rows, codes, scales, T, Y in results[0][1]:
        assert not seen[rows].any()
        seen[rows] = True
        # codes and scales are decided per row: bit-identical to the whole batch
        assert np.array_equal(codes, full.x_codes[rows])
        assert np.array_equal(np.asarray(scales).view(np.uint8), np.asarray(full.x_scales[rows]).view(np.uint8))
        # float64 sums may be blocked differently for a different row count
        assert np.max(np.abs(T - full.T[rows])) <= 1e-12 * np.max(np.abs(full.T))
        assert np.max(np.abs(Y - full.Y[rows])) <= 1e-12 * np.max(np.abs(full.Y))
    assert seen.all()


def test_whole_job_value_counts_every_rank():
    import bench
    # 2 ranks, 10 steps of 1e12 ops each per rank in 20 ms (the slowest rank)
    assert bench.whole_job_tops(1e12, 10, 2, 20.0) == pytest.approx(1000.0)
    assert bench.max_over_ranks(7.5, 1, None) == 7.5
