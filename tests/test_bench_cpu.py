"""bench.py's bookkeeping on CPU: the work a layer counts, the algorithmic
bytes of the activation kernel, the DRAM-traffic records and their staleness
rule, and the whole-job aggregation (the multi-rank timing itself is covered
in test_multirank_cpu.py)."""
import os

import pytest

import bench


def test_layer_ops_counts_the_4bit_product_and_both_branch_products():
    # Y = Q(x_hat) Q(R) + (x_hat L1) L2: 2MKN for the 4-bit product, 2MrK for
    # the down-projection, 2MrN for the up-projection
    M, K, N, r = 4608, 3072, 3072, 32
    assert bench.layer_ops(M, K, N, r) == 2 * M * K * N + 2 * M * r * K + 2 * M * r * N
    assert bench.gemm_ops(M, K, N, r) == 2 * M * K * N + 2 * M * r * N


@pytest.mark.parametrize("fmt,G,sbytes", [("int4_g64", 64, 4), ("nvfp4_g16", 16, 1)])
def test_activation_kernel_bytes(fmt, G, sbytes):
    M, K, r = 4608, 3072, 32
    expect = 2 * M * K + M * K / 2 + M * K / G * sbytes + 2 * M * r + 2 * K * r
    assert bench.k1_bytes(M, K, r, fmt) == expect
    # the attention projection: about 36.8 MB for either format
    assert abs(bench.k1_bytes(M, K, r, fmt) / 1e6 - 36.8) < 0.6


def test_whole_job_value_is_weak_scaling():
    one = bench.whole_job_tops(1e12, 100, 1, 50.0)
    four = bench.whole_job_tops(1e12, 100, 4, 50.0)
    assert four == pytest.approx(4 * one)
    # the slowest rank sets the time
    assert bench.whole_job_tops(1e12, 100, 2, 100.0) == pytest.approx(one)


def test_traffic_records_are_dropped_once_the_kernel_source_changes(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    digest = bench.source_digest(["k.cu"])
    rec = tmp_path / "records.txt"
    rec.write_text("# comment\n" + f"my_kernel cfg1_key 12345 {digest} k.cu\n")
    monkeypatch.setattr(bench, "TRAFFIC_RECORDS_FILE", str(rec))
    assert bench.traffic_for("my_kernel", "cfg1_key") == 12345.0
    assert bench.traffic_for("my_kernel", "other_key") is None
    assert bench.traffic_for("other_kernel", "cfg1_key") is None
    src.write_text("kernel v2\n")  # the kernel changed since the capture
    assert bench.traffic_for("my_kernel", "cfg1_key") is None


def test_committed_traffic_records_name_existing_sources():
    path = bench.TRAFFIC_RECORDS_FILE
    assert os.path.exists(path)
    n = 0
    with open(path) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, key, nbytes, digest, srcs = line.split()
            assert float(nbytes) > 0 and len(digest) == 16
            for s in srcs.split(","):
                assert os.path.exists(os.path.join(bench.ROOT, s)), s
            n += 1
    assert n >= 1


def test_workload_names_carry_the_shapes():
    import workloads
    d = bench.workload_desc(1, workloads.config(0))  # any layer list; the name follows the config id
    assert "attention projection" in d


def test_peak_follows_the_length_of_the_timed_region():
    peaks = {"bf16_tflops": 1640.7, "bf16_tflops_sustained": 1376.5}
    burst, d1 = bench.tensor_peak_for(peaks, "nvfp4_g16", 0.0065)
    assert burst == pytest.approx(4 * 1640.7) and "burst" in d1
    sus, d2 = bench.tensor_peak_for(peaks, "nvfp4_g16", 6.5)
    assert sus == pytest.approx(4 * 1376.5) and "sustained" in d2
    assert bench.tensor_peak_for(peaks, "int4_g64", 0.003)[0] == pytest.approx(2 * 1640.7)


def test_both_arms_emit_the_same_config():
    import argparse

    import workloads
    args = argparse.Namespace(config=0, M=0, rank=0, fmt=None)
    layers = bench.load_layers(args)
    a, b = bench.config_dict(args, layers), bench.config_dict(args, workloads.config(0))
    assert a == b and "l2" in a and a["config_id"] == 0
    n_sets, set_bytes = bench.rotation_sets(layers)
    assert n_sets * set_bytes > 2 * bench.L2_BYTES


def test_default_workload_is_the_nvfp4_mlp_pair():
    args = bench.parse_args([])
    assert args.config == 3 and args.gpus == 1 and args.impl == "ours"
    assert bench.parse_args(["--config", "1"]).config == 1
