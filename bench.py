#!/usr/bin/env python
"""Benchmark of the SVDQuant W4A4 + low-rank linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config 3]

One step = one pass of the whole hot path (svdq_linear_forward: the activation
kernel + the 4-bit GEMM with the fused low-rank/bias epilogue) over one batch
of the configuration's synthetic inputs (for the MLP-pair configurations, both
layers). Default workload: the FLUX-like MLP pair in NVFP4 (up 4608 x 3072 ->
12288, then down 4608 x 12288 -> 3072, rank 32, E2M1 group 16), the largest
configuration. Prints one JSON line on rank 0.

Multi-GPU (torchrun, one process per GPU): the layer is token-parallel - every
rank runs its own batch against its own copy of the weights, with no
collective on the data path (weak scaling); only the timing uses a barrier and
a max-reduce over ranks.

--impl reference times the CPU oracle (oracle/, float64 numpy) on the host
cores on a row sample of the same workload, sized so the run ends in minutes.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A4+low-rank linear TOPS & µs/layer (FLUX shapes), % of FP4/INT8 tensor peak"
L2_BYTES = 126 * 2 ** 20
# dense datasheet peaks (context): FP4 9.0 PFLOP/s, INT8/FP8 4.5 POPS
DATASHEET_TOPS = {"nvfp4_g16": 9000.0, "int4_g64": 4500.0}
# tensor-rate ratio of the MMA kind each format runs on, relative to bf16
RATE_VS_BF16 = {"nvfp4_g16": 4.0, "int4_g64": 2.0}  # mxf4nvf4 = 4x bf16; f8f6f4 = 2x bf16

# DRAM bytes per launch from an ncu capture (dram__bytes_read.sum + dram__bytes_write.sum),
# valid only while the kernel source it was taken from is unchanged.
TRAFFIC_RECORDS_FILE = os.path.join(ROOT, "profiles", "traffic_records.txt")


def is_fused(args, layers) -> bool:
    """An NVFP4 MLP pair runs as one fused MLP block unless --unfused."""
    return (args.config in (2, 3) and layers[0].fmt == "nvfp4_g16" and not getattr(args, "unfused", False)
            and len(layers) == 2)


def workload_desc(cfg: int, layers, fused: bool = False) -> str:
    L = layers[0]
    if fused:
        return (f"FLUX-like MLP block, fused: up [{L.M},{L.K}]x[{L.K},{L.N}] -> GELU of the up output -> down "
                f"[{L.M},{layers[1].K}]x[{layers[1].K},{layers[1].N}], rank {L.rank}, {L.fmt}")
    if cfg == 1:
        return f"FLUX-like attention projection: X bf16 [{L.M},{L.K}] x W [{L.K},{L.N}], rank {L.rank}, {L.fmt}"
    if cfg in (2, 3):
        return (f"FLUX-like MLP pair: up [{L.M},{L.K}]x[{L.K},{L.N}] then down [{L.M},{layers[1].K}]x"
                f"[{layers[1].K},{layers[1].N}], rank {L.rank}, {L.fmt}")
    if cfg == 4:
        lora = "" if L.lora_A is None else f" + a rank-{L.lora_A.shape[1]} LoRA in the branch"
        return f"sweep point K=N=3072, M={L.M}, rank {L.rank}{lora}, {L.fmt}"
    return f"single linear [{L.M},{L.K}]x[{L.K},{L.N}], rank {L.rank}, {L.fmt}"


def layer_ops(M, K, N, r) -> float:
    return 2.0 * M * K * N + 2.0 * M * r * (K + N)


def gemm_ops(M, K, N, r) -> float:
    return 2.0 * M * K * N + 2.0 * M * r * N


def k1_bytes(M, K, r, fmt) -> float:
    """Algorithmic HBM bytes of the activation kernel: X read, 4-bit codes and
    group scales written, T written, L1 read once."""
    G = 64 if fmt == "int4_g64" else 16
    sbytes = 4 if fmt == "int4_g64" else 1
    return 2.0 * M * K + M * K / 2 + M * K / G * sbytes + 2.0 * M * r + 2.0 * K * r


def load_layers(args):
    import workloads
    kw = {}
    if args.M:
        kw["M"] = args.M
    if args.rank:
        kw["rank"] = args.rank
    if args.fmt:
        kw["fmt"] = args.fmt
    if getattr(args, "lora", False):
        if args.config != 4:
            raise SystemExit("--lora belongs to the sweep (--config 4)")
        kw["lora"] = True
    layers = workloads.config(args.config, **kw)
    return layers


def branch_rank(L) -> int:
    """Columns of the layer's low-rank branch: its rank plus an attached adapter's."""
    return L.rank + (0 if L.lora_A is None else int(L.lora_A.shape[1]))


# A timed region shorter than this is a burst: the clocks have not settled
# under the power cap, so the burst peak is the fair denominator.
BURST_REGION_S = 1.0


def tensor_peak_for(peaks: dict, fmt: str, timed_region_s: float):
    """(peak TFLOP/s, description): the measured bf16 GEMM peak for the length
    of the timed region (burst when it is shorter than BURST_REGION_S, else
    sustained) times the nominal rate ratio of the MMA kind the format uses."""
    burst = timed_region_s < BURST_REGION_S
    key = "bf16_tflops" if burst else "bf16_tflops_sustained"
    kind = "mxf4nvf4" if fmt == "nvfp4_g16" else "f8f6f4"
    desc = (f"bf16 {'burst' if burst else 'sustained'} {peaks[key]} TFLOP/s x {RATE_VS_BF16[fmt]:g} "
            f"(nominal {kind}/bf16 rate; timed region {timed_region_s:.3f} s)")
    return peaks[key] * RATE_VS_BF16[fmt], desc


def ws_bytes_lower_bound(L) -> int:
    """Activation codes + scales + T of one forward (the K-share partials left out)."""
    M_pad = (L.M + 127) // 128 * 128
    codes = M_pad * L.K if L.fmt == "int4_g64" else M_pad * L.K // 2
    scales = M_pad * (L.K // 64) * 4 if L.fmt == "int4_g64" else M_pad * (L.K // 16)
    return codes + scales + M_pad * ((L.rank + 31) // 32 * 32) * 2


def rotation_sets(layers, fused: bool = False) -> tuple[int, int]:
    """(sets, bytes per set): enough rotating copies of inputs, outputs,
    workspace and prepared weights that one step's data is out of L2 again
    when its set comes back. The fused MLP block reads only the first layer's
    X and writes only the last layer's Y."""
    set_bytes = 0
    for i, L in enumerate(layers):
        if not fused or i == 0:
            set_bytes += L.M * L.K * 2
        if not fused or i == len(layers) - 1:
            set_bytes += L.M * L.N * 2
        set_bytes += ws_bytes_lower_bound(L)
        set_bytes += L.N * L.K // 2 * (2 if L.fmt == "int4_g64" else 1) + L.N * L.K // 16
    return max(2, math.ceil(2 * L2_BYTES / max(set_bytes, 1))), set_bytes


def config_dict(args, layers) -> dict:
    """The `config` object of the JSON line, identical in both arms."""
    fused = is_fused(args, layers)
    n_sets, set_bytes = rotation_sets(layers, fused)
    L = layers[0]
    return {"workload": workload_desc(args.config, layers, fused), "config_id": args.config,
            "M": L.M, "K": L.K, "N": L.N, "rank": L.rank, "lora_rank": branch_rank(L) - L.rank, "format": L.fmt,
            "layers_per_step": len(layers),
            "pipeline": ("fused MLP block (activation kernel, up GEMM with GELU and the down layer's quantization "
                         "in its epilogue, T sum, down GEMM)" if fused else "one forward per layer"),
            "l2": f"inputs larger than L2: {n_sets} rotating sets of prepared layer + X/Y/workspace "
                  f"(>= {n_sets * set_bytes / 2**20:.0f} MiB > 2 x 126 MiB L2)"}


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def source_digest(files) -> str:
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload_key: str):
    """Per-launch DRAM bytes recorded from ncu, or None when absent or stale."""
    if not os.path.exists(TRAFFIC_RECORDS_FILE):
        return None
    with open(TRAFFIC_RECORDS_FILE) as f:
        for line in f:
            parts = line.split()
            if len(parts) < 5 or line.startswith("#"):
                continue
            name, wk, nbytes, digest, src = parts[0], parts[1], parts[2], parts[3], parts[4].split(",")
            if name == kernel and wk == workload_key:
                try:
                    if source_digest(src) == digest:
                        return float(nbytes)
                except OSError:
                    return None
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.25)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self, t0, t1):
        if self.proc is None:
            return {"samples": 0, "note": "nvidia-smi unavailable"}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        inside = [l for (t, l) in self.lines if t0 <= t <= t1 + 0.1]
        use = inside or [l for (_, l) in self.lines]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in use:
            p = [x.strip() for x in l.split(",")]
            if len(p) < 8:
                continue
            try:
                sm.append(float(p[0]))
                mx.append(float(p[1]))
            except ValueError:
                continue
            for name, v in zip(names, p[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "samples_inside_timed_region": len(inside)}


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's duration: the whole job is done when the last rank is."""
    if world == 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tops(ops_per_rank_step: float, steps: int, world: int, max_ms: float) -> float:
    """Weak scaling: every rank runs its own batch of tokens through the layers
    each step, so the job's work is world x the per-rank work, done in the
    slowest rank's time."""
    return ops_per_rank_step * steps * world / (max_ms * 1e-3) / 1e12


def init_dist(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    return world, rank, local


def run_ours(args):
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist

    import rank_gemm_quantize_b200 as rq

    world, rank, local = init_dist(args)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    layers = load_layers(args)
    peaks, peak_kind = read_peaks()

    # ---- prepare: one layer instance per rotating set (the first with the GPU
    # SVD, the others from its factors), plus X / Y / workspace per set. The
    # fused MLP block's down layer is calibrated on the GELU of the up layer's
    # output, which is what it receives.
    fused = is_fused(args, layers)
    preps = []
    for li, L in enumerate(layers):
        if fused and li == 1:
            with torch.no_grad():
                g_up0 = preps[0][3]
                h = torch.nn.functional.gelu(g_up0.forward(preps[0][1]).float()).to(torch.bfloat16)
            X0 = None
            a = rq.calibrate_absmax(h)
            del h
        else:
            X0 = L.X.to(dev)
            a = rq.calibrate_absmax(X0)
        g0 = rq.Layer.prepare(L.W.to(dev), L.bias.to(dev), a, L.fmt, L.rank, alpha=L.alpha)
        ex = g0.export()  # the prepared layer's own factors, before any adapter
        if L.lora_A is not None:
            g0.attach_lora(L.lora_A.to(dev), L.lora_B.to(dev), L.lora_scale)
        preps.append((L, X0, a, g0, ex))
    n_sets, _ = rotation_sets(layers, fused)
    sets = []
    for s in range(n_sets):
        items = []
        for (L, X0, a, g0, ex) in preps:
            if s == 0:
                g = g0
            else:
                L1 = torch.from_numpy(ex["L1"]).to(torch.bfloat16).to(dev)
                L2 = torch.from_numpy(ex["L2"]).to(torch.bfloat16).to(dev)
                g = rq.Layer.prepare(L.W.to(dev), L.bias.to(dev), a, L.fmt, L.rank, alpha=L.alpha, factors=(L1, L2))
                if L.lora_A is not None:
                    g.attach_lora(L.lora_A.to(dev), L.lora_B.to(dev), L.lora_scale)
            X = None if X0 is None else (X0 if s == 0 else X0.clone())
            Y = torch.empty(L.M, L.N, dtype=torch.bfloat16, device=dev) if not fused or L is layers[-1] else None
            ws = None if fused else torch.empty(g.workspace_size(L.M), dtype=torch.uint8, device=dev)
            items.append([g, X, Y, ws])
        if fused:
            blk = rq.MlpBlock(items[0][0], items[1][0])
            items[0][3] = torch.empty(blk.workspace_size(layers[0].M), dtype=torch.uint8, device=dev)
            items.append(blk)
        sets.append(items)
    torch.cuda.synchronize()

    n_layers = len(layers)
    K_steps, W_steps = args.steps, args.warmup
    # events: per step and layer, before K1 / between / after the GEMM; the
    # fused block records five: before K1, after K1, after the fused up GEMM,
    # after the T sum, after the down GEMM
    n_ev = [5] if fused else [3] * n_layers
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(n)] for n in n_ev] for _ in range(K_steps)]
    for per_step in evs:  # torch creates the CUDA event at its first record
        for per_layer in per_step:
            for e in per_layer:
                e.record()

    def step(i, events=None):
        items = sets[i % n_sets]
        if fused:
            blk = items[2]
            blk.forward(items[0][1], out=items[1][2], workspace=items[0][3], events=None if events is None else events[0])
            return
        for li, (g, X, Y, ws) in enumerate(items):
            if events is None:
                g.forward(X, out=Y, workspace=ws)
            else:
                g.forward_profiled(X, Y, ws, events[li])

    for i in range(W_steps):
        step(i)
    torch.cuda.synchronize()

    uuid = str(torch.cuda.get_device_properties(local).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0_wall = time.time()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(K_steps):
        step(i, evs[i])
    end.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t1_wall = time.time()
    clocks = sampler.stop(t0_wall, t1_wall)
    elapsed_ms = start.elapsed_time(end)
    mean_ms = lambda li, a, b: statistics.fmean(evs[i][li][a].elapsed_time(evs[i][li][b]) for i in range(K_steps))
    if fused:
        k1_ms = [mean_ms(0, 0, 1)]
        gemm_ms = [mean_ms(0, 1, 2), mean_ms(0, 3, 4)]
        reduce_ms = mean_ms(0, 2, 3)
    else:
        k1_ms = [mean_ms(li, 0, 1) for li in range(n_layers)]
        gemm_ms = [mean_ms(li, 1, 2) for li in range(n_layers)]
        reduce_ms = None
    max_ms = max_over_ranks(elapsed_ms, world, dev)

    step_ops = sum(layer_ops(L.M, L.K, L.N, branch_rank(L)) for L in layers)
    value = whole_job_tops(step_ops, K_steps, world, max_ms)
    ms_per_step = max_ms / K_steps

    # ---- e2e through the public API with host buffers. Every step copies its
    # inputs in from pinned host memory and its outputs back out. The batches
    # are independent, so step i+1's inputs travel host->device on one copy
    # stream and step i-1's outputs device->host on another (PCIe is full
    # duplex) while step i computes; events keep each rotating set's buffers
    # from being overwritten before the step that last used them is done.
    e2e_steps = max(3, min(args.e2e_steps, K_steps))
    io = [0] if fused else list(range(n_layers))  # layers whose X comes from the host
    oo = [n_layers - 1] if fused else list(range(n_layers))  # layers whose Y goes back
    hostX = {li: layers[li].X.pin_memory() for li in io}
    hostY = {li: torch.empty(layers[li].M, layers[li].N, dtype=torch.bfloat16).pin_memory() for li in oo}
    h2d = sum(layers[li].M * layers[li].K * 2 for li in io)
    d2h = sum(layers[li].M * layers[li].N * 2 for li in oo)
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(n):
        fwd_done = [None] * n_sets  # forward of the last step that used the set (its X is free after it)
        out_done = [None] * n_sets  # D2H of the last step that used the set (its Y is free after it)
        for i in range(n):
            k = i % n_sets
            with torch.cuda.stream(s_in):
                if fwd_done[k] is not None:
                    s_in.wait_event(fwd_done[k])
                for li in io:
                    sets[k][li][1].copy_(hostX[li], non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
            comp.wait_event(ev_in)
            if out_done[k] is not None:
                comp.wait_event(out_done[k])
            if fused:
                sets[k][2].forward(sets[k][0][1], out=sets[k][1][2], workspace=sets[k][0][3], stream=comp)
            else:
                for li, (g, X, Y, ws) in enumerate(sets[k][:n_layers]):
                    g.forward(X, out=Y, workspace=ws, stream=comp)
            fwd_done[k] = torch.cuda.Event()
            fwd_done[k].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(fwd_done[k])
                for li in oo:
                    hostY[li].copy_(sets[k][li][2], non_blocking=True)
                out_done[k] = torch.cuda.Event()
                out_done[k].record(s_out)
        for ev in out_done:  # the region ends when the last output is on the host
            if ev is not None:
                comp.wait_event(ev)

    e2e_run(2)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    e2e_run(e2e_steps)
    e1.record(comp)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = whole_job_tops(step_ops, e2e_steps, world, e2e_ms)
    # the last step's outputs reached the host: compare them with the device copies
    for li in oo:
        if not torch.equal(hostY[li], sets[(e2e_steps - 1) % n_sets][li][2].cpu()):
            raise SystemExit("e2e: the host copy of the output differs from the device result")

    # ---- the 4-bit weight-only (W4A16) baseline of the abstract's speedup
    # claim, on the same workload: its own quantized weights per rotating
    # set, the same X, timed the same way (outside the timed region above)
    w4a16 = None
    if not args.no_w4a16:
        w4_sets = [[rq.WeightOnlyLayer(L.W.to(dev), L.bias.to(dev)) for L in layers] for _ in range(n_sets)]
        # the same shapes: each layer's own input and output buffers (the
        # fused block's missing ones are made here)
        w4_io = [[(it[1] if it[1] is not None else layers[li].X.to(dev),
                   it[2] if it[2] is not None else torch.empty(layers[li].M, layers[li].N, dtype=torch.bfloat16,
                                                               device=dev))
                  for li, it in enumerate(st[:n_layers])] for st in sets]

        def w4_step(i):
            for li, (X, Y) in enumerate(w4_io[i % n_sets]):
                w4_sets[i % n_sets][li].forward(X, out=Y)

        for i in range(max(3, W_steps)):
            w4_step(i)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        w0.record()
        for i in range(K_steps):
            w4_step(i)
        w1.record()
        torch.cuda.synchronize()
        w4_ms = max_over_ranks(w0.elapsed_time(w1), world, dev) / K_steps
        w4_ops = sum(2.0 * L.M * L.K * L.N for L in layers)
        w4a16 = {"ms_per_step": w4_ms, "tops": w4_ops / (w4_ms * 1e-3) / 1e12,
                 "w4a4_speedup": w4_ms / ms_per_step,
                 "what": "INT4 g64 weights alone (no smoothing, no branch), bf16 activations, tcgen05 kind::f16 "
                         "after on-chip dequantization; one kernel per layer"}
        for row in w4_sets:
            for wl in row:
                wl.close()

    # device status: no kernel gave up a wait
    for items in sets:
        for (g, X, Y, ws) in items[:n_layers]:
            if g.device_status() != rq.Status.OK:
                raise SystemExit("a kernel reported a timed-out pipeline wait")

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    # ---- roofline of the dominant kernel (the GEMM) and of the activation kernel
    fmt = layers[0].fmt
    wl_key = f"cfg{args.config}_M{layers[0].M}_r{layers[0].rank}_{fmt}" + ("_fused" if fused else "")
    g_ops = sum(gemm_ops(L.M, L.K, L.N, branch_rank(L)) for L in layers)
    g_s = sum(gemm_ms) * 1e-3
    tensor_peak, peak_desc = tensor_peak_for(peaks, fmt, elapsed_ms * 1e-3)
    gemm_name = "gemm_int4_kernel" if fmt == "int4_g64" else "gemm_nvfp4_kernel"
    traffic = traffic_for(gemm_name, wl_key)
    roofline = {"bound": "tensor", "kernel": gemm_name, "achieved": g_ops / g_s / 1e12,
                "peak": tensor_peak, "unit": "TFLOP/s", "frac": g_ops / g_s / 1e12 / tensor_peak,
                "traffic": traffic,
                "peak_source": f"{peak_kind} {peak_desc}",
                "algorithmic": "2MKN + 2MrN per launch", "frac_of_datasheet_dense": g_ops / g_s / 1e12 / DATASHEET_TOPS[fmt]}
    k_bytes = sum(k1_bytes(L.M, L.K, branch_rank(L), fmt) for L in (layers[:1] if fused else layers))
    k_s = sum(k1_ms) * 1e-3
    k1_roof = {"bound": "hbm", "kernel": "act_quant_kernel", "achieved": k_bytes / k_s / 1e9, "peak": peaks["hbm_gbs"],
               "unit": "GB/s", "frac": k_bytes / k_s / 1e9 / peaks["hbm_gbs"],
               "traffic": traffic_for("act_quant_kernel", wl_key),
               "algorithmic": "2MK + MK/2 + MK/G*scale + 2Mr + 2Kr bytes per launch"}

    cpu = None
    if not args.no_cpu_baseline:
        cpu = cpu_baseline(layers, budget_s=args.cpu_seconds)

    out = {
        "metric": METRIC,
        "value": value,
        "unit": "TOPS",
        "n_gpus": world,
        "steps": K_steps,
        "warmup": W_steps,
        "ms_per_step": ms_per_step,
        "us_per_layer": ms_per_step * 1e3 / n_layers,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int4" if fmt == "int4_g64" else "nvfp4",
        "data": "synthetic",
        "config": config_dict(args, layers),
        "pct_of_datasheet_dense_peak": 100.0 * value / DATASHEET_TOPS[fmt],
        "roofline": roofline,
        "kernels": {"act_quant": {"ms": k1_ms, **k1_roof}, "gemm": {"ms": gemm_ms},
                    **({"t_sum": {"ms": reduce_ms}} if fused else {})},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "TOPS", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps},
        "gpu_launches": (4 if fused else 2 * n_layers) * K_steps,
        "w4a16_baseline": w4a16,
        "clocks": clocks,
        "impl": "ours",
    }
    print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()


# The method's ablations (msModelSlim SVDQuant entry, related terms: SmoothQuant
# is the rank-0 special case; section 2.3 eq. 2: alpha sets the migration
# strength): (name, rank, alpha, smooth).
ABLATIONS = [
    ("W4A4, no smoothing, no branch", 0, 0.5, False),
    ("smoothing only (SmoothQuant, rank 0)", 0, 0.5, True),
    ("low-rank branch without smoothing", None, 0.5, False),
    ("SVDQuant alpha 0.3", None, 0.3, True),
    ("SVDQuant alpha 0.5", None, 0.5, True),
    ("SVDQuant alpha 0.7", None, 0.7, True),
]


def run_ablation(args):
    """One JSON line: for each ablation of the method, the layer's normwise
    error against the unquantized X W + b (float64) and its time per layer,
    on the configuration's first layer, both formats."""
    import torch

    import rank_gemm_quantize_b200 as rq
    import workloads
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    L = load_layers(args)[0]
    X, W, b = L.X.to(dev), L.W.to(dev), L.bias.to(dev)
    ref = X.double() @ W.double() + b.double()  # the layer without quantization
    a = rq.calibrate_absmax(X)
    rows = []
    for fmt in workloads.FORMATS:
        for name, rank, alpha, smooth in ABLATIONS:
            r = L.rank if rank is None else rank
            g = rq.Layer.prepare(W, b, a, fmt, r, alpha=alpha, smooth=smooth)
            try:
                Y = g.forward(X)
                err = float(torch.linalg.norm(Y.double() - ref) / torch.linalg.norm(ref))
                ws = g.workspace(L.M)
                for _ in range(3):
                    g.forward(X, out=Y, workspace=ws)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                n = 20
                e0.record()
                for _ in range(n):
                    g.forward(X, out=Y, workspace=ws)
                e1.record()
                torch.cuda.synchronize()
                us = e0.elapsed_time(e1) * 1e3 / n
                rows.append({"format": fmt, "variant": name, "rank": r, "alpha": alpha, "smooth": smooth,
                             "rel_err_vs_xw_plus_b": err, "us_per_layer": us,
                             "tops": layer_ops(L.M, L.K, L.N, r) / (us * 1e-6) / 1e12})
            finally:
                g.close()
    print(json.dumps({"ablation": rows, "config": config_dict(args, [L]) | {"layers_per_step": 1},
                      "note": "L2-hot back-to-back timing of one layer; errors are normwise against float64 X W + b"}),
          flush=True)


def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


def _oracle_prepare(layers):
    import workloads
    from oracle import svdquant as S
    out = []
    for L in layers:
        X = workloads.to_f64(L.X)
        a = S.calibrate_absmax(X)
        p = S.prepare(workloads.to_f64(L.W), workloads.to_f64(L.bias), a, L.fmt, L.alpha, L.rank)
        if L.lora_A is not None:
            p = S.attach_lora(p, workloads.to_f64(L.lora_A), workloads.to_f64(L.lora_B), L.lora_scale)
        S.dequantized_weight(p)
        out.append((L, X, p))
    return out


def _rows_for(preps, seconds: float, M: int) -> int:
    """Rows of the oracle's forward (row-local, so any row sample is a fair
    sample of the batch) that take about `seconds` on this host."""
    from oracle import svdquant as S
    t = time.perf_counter()
    for (L, X, p) in preps:
        S.forward(p, X[:128])
    per_row = max((time.perf_counter() - t) / 128, 1e-6)
    return int(max(1, min(M, seconds / per_row)))


def cpu_baseline(layers, budget_s: float = 10.0, rows=None):
    """The oracle's forward timed on the host cores on a row sample of the workload."""
    from oracle import svdquant as S
    preps = _oracle_prepare(layers)
    M = layers[0].M
    r = rows or _rows_for(preps, budget_s / 3, M)
    t_total, n, ops = 0.0, 0, 0.0
    while True:
        t = time.perf_counter()
        for (L, X, p) in preps:
            S.forward(p, X[:r])
        t_total += time.perf_counter() - t
        n += 1
        ops += sum(layer_ops(r, L.K, L.N, branch_rank(L)) for L in layers)
        if t_total >= budget_s or n >= 50:
            break
    return {"value": ops / t_total / 1e12, "unit": "TOPS", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{n} oracle forward(s) of {r} of {M} rows per layer ({len(layers)} layer(s)), "
                      f"{t_total:.1f} s; prepare (numpy SVD) excluded"}


def run_reference(args):
    world, rank, _ = init_dist(args)
    if rank != 0:
        return  # rank 0 alone runs the CPU reference; the others exit without work
    layers = load_layers(args)
    from oracle import svdquant as S
    preps = _oracle_prepare(layers)
    # size the row sample so that warmup + steps fit in about 80 s
    rows = _rows_for(preps, 80.0 / max(1, args.steps + args.warmup), layers[0].M)
    for _ in range(args.warmup):
        for (L, X, p) in preps:
            S.forward(p, X[:rows])
    t = time.perf_counter()
    for _ in range(args.steps):
        for (L, X, p) in preps:
            S.forward(p, X[:rows])
    dt = time.perf_counter() - t
    ops = sum(layer_ops(rows, L.K, L.N, branch_rank(L)) for L in layers) * args.steps
    value = ops / dt / 1e12
    fmt = layers[0].fmt
    cores = _blas_threads()
    sample = f"{rows} of {layers[0].M} rows per step per layer"
    out = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(args, layers),
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=3)
    ap.add_argument("--M", type=int, default=0)
    ap.add_argument("--rank", type=int, default=0)
    ap.add_argument("--fmt", choices=["int4_g64", "nvfp4_g16"], default=None)
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-w4a16", action="store_true", help="skip timing the weight-only baseline")
    ap.add_argument("--unfused", action="store_true",
                    help="run an NVFP4 MLP pair as two layer forwards instead of the fused MLP block")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--lora", action="store_true", help="sweep (--config 4) with a rank-32 LoRA in the branch")
    ap.add_argument("--ablation", action="store_true",
                    help="print the error / time table of the method's ablations instead of the benchmark line")
    return ap.parse_args(argv)


def main():
    args = parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.ablation:
        run_ablation(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
