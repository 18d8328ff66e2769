"""Benchmark of the AWQ scale search on B200: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 5] [--impl ours|reference]

A step is one pass of the whole path over one layer: the activation statistic, the search (scale table,
weight-error producer, tensor-core loss GEMM, argmin) and the packed INT4 artefact at the best scales.
Inputs are resident in HBM when a step starts; L2 is flushed between steps (a 512 MiB write). The
metric is candidates/s (n_grid candidates per step); the loss GEMM is also timed alone (events recorded
around its launch inside the library) for the roofline. ``e2e`` repeats the measurement through the
public Python API with pinned host buffers: H2D of X and W, the path, D2H of codes/steps/zeros/scales/
losses/best_j, all inside the timed region.

The default workload is 5, the largest single-GPU configuration (X 16384 x 28672, W 8192 x 28672).

With N > 1 (torchrun) every rank quantizes its own layer (independent replicas, no data exchange); the
time is the max over ranks and ``value`` counts every rank's candidates. ``--impl reference`` times the
CPU oracle on a bounded sample of the same workload (rank 0 only), the same sample as ``cpu_baseline``.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "AWQ search candidates/sec per layer and effective TFLOP/s vs BF16 peak"
UNIT = "candidates/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
GEMM_SOURCES = ["kernel_loss_gemm.cuh", "ptx.cuh", "kernels_simple.cuh", "numerics.cuh"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def gemm_source_hash() -> str:
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(os.path.join(ROOT, "weight_only_quantization_act_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "loss_gemm_traffic.json")


def profiled_traffic(workload: int):
    """Per-launch DRAM bytes (read + write) of the loss GEMM from the committed ncu summary
    (profiles/loss_gemm_traffic.json), if it was taken on the current kernel source (same hash) for this
    workload; otherwise (None, why)."""
    if not os.path.exists(TRAFFIC_FILE):
        return None, "no ncu traffic record"
    with open(TRAFFIC_FILE) as f:
        rec = json.load(f)
    if rec.get("kernel_source_sha256_16") != gemm_source_hash():
        return None, "the loss kernel changed since its DRAM counters were taken"
    w = rec.get("workloads", {}).get(str(workload))
    if w is None:
        return None, f"no ncu DRAM capture for workload {workload}"
    return float(w["dram_bytes_per_launch"]), w.get("how", "")


class ClockSampler:
    """nvidia-smi samples (200 ms) of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------------------ oracle arm
SAMPLE_TOKENS = 512   # the loss GEMM is timed on the first 512 tokens and scaled by N / 512
SAMPLE_BLOCKS = 8     # the quantizer and the loss are timed in 8 blocks of output rows


def _blocks(O):
    step = -(-O // SAMPLE_BLOCKS)
    return [(r0, min(O, r0 + step)) for r0 in range(0, O, step)]


class OracleSample:
    """The one bounded sample of the oracle that both ``cpu_baseline`` and ``--impl reference`` time.

    For one candidate (ratio j = n_grid // 2): its scale-table row (correctly rounded powers over K), then,
    block by block over 8 blocks of output rows, the quantizer (scale, group-quantize, dequantize,
    unscale) on the block's rows of the full W and the fp64 loss GEMM of the first 512 tokens against the
    block. The quantizer is thus timed in full; the loss time is scaled by N / 512 (the loss GEMM is
    linear in N). The statistic over all N tokens is timed once. One layer of n_grid candidates is then
    t_statistic + n_grid * (t_scale_row + sum over blocks of (t_quant + t_loss * N / 512))."""

    def __init__(self, wl, X, W):
        from oracle import awq_oracle as orc

        self.orc, self.wl, self.X, self.W = orc, wl, X, W
        self.tokens = min(SAMPLE_TOKENS, wl.N)
        self.scale = wl.N / self.tokens
        self.j = wl.n_grid // 2
        self.blocks = _blocks(W.shape[0])
        t0 = time.perf_counter()
        self.act = orc.act_mean(X)
        self.t_act = time.perf_counter() - t0
        t0 = time.perf_counter()
        self.s = orc.scale_candidates(self.act, orc.ratio(self.j, wl.n_grid))
        self.t_scale = time.perf_counter() - t0
        self.wall = self.t_act + self.t_scale

    def block(self, b):
        """Quantizer and loss for block b; returns its extrapolated seconds (loss scaled by N / tokens)."""
        r0, r1 = self.blocks[b]
        Wb = self.W[r0:r1]
        t0 = time.perf_counter()
        w_hat, _, _, _ = self.orc.pseudo_quantize(Wb, self.s)
        t1 = time.perf_counter()
        self.orc.loss_of(self.X[:self.tokens], Wb, w_hat)
        t2 = time.perf_counter()
        self.wall += t2 - t0
        return (t1 - t0) + (t2 - t1) * self.scale

    def per_layer_s(self, block_times):
        """Extrapolated seconds of one layer from the mean extrapolated block time."""
        per_cand = self.t_scale + len(self.blocks) * float(np.mean(block_times))
        return self.t_act + self.wl.n_grid * per_cand

    def describe(self, n_block_runs):
        wl = self.wl
        return (f"workload {wl.number}: statistic over all {wl.N} tokens; candidate j={self.j} of {wl.n_grid}: "
                f"scale row, then in {len(self.blocks)} blocks of output rows the quantizer over the full W "
                f"and the fp64 loss GEMM on the first {self.tokens} tokens ({n_block_runs} block runs); loss "
                f"time scaled by N/{self.tokens} = {self.scale:g}; extrapolated to one layer of {wl.n_grid} "
                f"candidates")


def oracle_sample(wl, X, W):
    """cpu_baseline: the sample once (every block of one candidate), extrapolated to candidates/s."""
    smp = OracleSample(wl, X, W)
    smp.block(0)  # one untimed block first (page faults of numpy's first large temporaries)
    times = [smp.block(b) for b in range(len(smp.blocks))]
    per_layer = smp.per_layer_s(times)
    return {
        "value": wl.n_grid / per_layer,
        "unit": UNIT,
        "cores": int(os.cpu_count() or 1),
        "kind": "oracle",
        "sample": smp.describe(len(times)) + " (after one untimed warm-up block)",
        "extrapolated": True,
        "sample_wall_s": smp.wall,
        "loss_scale_factor": smp.scale,
        "threads": _blas_threads(),
    }


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info

        return sum(int(i.get("num_threads", 0)) for i in threadpool_info() if i.get("user_api") == "blas") or None
    except Exception:
        return None


def run_reference(args, rank, world):
    """The oracle as the reference arm: the same sample as cpu_baseline, one block of output rows per step
    (blocks in turn), so a step is a bounded piece of one candidate's work."""
    from weight_only_quantization_act_b200 import inputs

    if rank != 0:
        return
    wl = inputs.workload(args.workload)
    X, W, _ = inputs.make_inputs(wl)
    smp = OracleSample(wl, X, W)
    nb = len(smp.blocks)
    for k in range(args.warmup):
        smp.block(k % nb)
    wall0 = smp.wall
    times = [smp.block((args.warmup + k) % nb) for k in range(args.steps)]
    per_layer = smp.per_layer_s(times)
    value = wl.n_grid / per_layer
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * (smp.wall - wall0) / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(wl, args.gpus),
        "extrapolated": True,
        "ms_per_step_is": "measured wall time of one sample step (one block of output rows of one candidate)",
        "layer_ms_extrapolated": 1e3 * per_layer,
        "sample_wall_s": smp.wall - wall0,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": int(os.cpu_count() or 1), "kind": "oracle",
                         "sample": smp.describe(len(times)), "extrapolated": True,
                         "sample_wall_s": smp.wall, "loss_scale_factor": smp.scale},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(wl, gpus):
    return {"workload": f"AWQ search, workload {wl.number}: {wl.name}", "N": wl.N, "K": wl.K, "O": wl.O,
            "out_rows": list(wl.out_rows), "group": wl.group, "n_grid": wl.n_grid,
            "parallelism": f"replicas x{gpus}" if gpus > 1 else "single GPU",
            "l2": "flushed between steps (512 MiB write)"}


# ------------------------------------------------------------------------------------------ our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from weight_only_quantization_act_b200 import awq, inputs, replicas  # noqa: F401

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    awq.load_library()
    wl = inputs.workload(args.workload)
    # each rank quantizes its own layer: same shapes, its own draw
    X, W, _ = inputs.make_inputs(replicas.replica_workload(wl, rank))
    Xh = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16)
    Wh = torch.from_numpy(W.view(np.int16)).view(torch.bfloat16)
    Xd, Wd = Xh.to(dev), Wh.to(dev)
    N, K, O, J = wl.N, wl.K, wl.O, wl.n_grid
    stream = torch.cuda.current_stream()

    act = torch.empty(K, dtype=torch.float32, device=dev)
    act_ws = torch.empty(awq.act_stats_workspace_size(N, K), dtype=torch.uint8, device=dev)
    res = awq.search(Xd, Wd, awq.act_stats(Xd, out=act, workspace=act_ws), n_grid=J)
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def step():
        awq.act_stats(Xd, out=act, workspace=act_ws)
        awq.search(Xd, Wd, act, n_grid=J, workspace=res.workspace, out=res)
        return awq.quantize_pack(Wd, res.scales)

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    for e in ev:
        for x in e:
            x.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for k in range(args.steps):
        flush.zero_()
        e = ev[k]
        e[0].record(stream)
        awq.act_stats(Xd, out=act, workspace=act_ws)
        e[1].record(stream)
        awq.set_profile_events(e[2], e[3])
        awq.search(Xd, Wd, act, n_grid=J, workspace=res.workspace, out=res)
        awq.set_profile_events(None, None)
        e[4].record(stream)
        awq.quantize_pack(Wd, res.scales)
        e[5].record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None

    step_ms = [e[0].elapsed_time(e[5]) for e in ev]
    act_ms = [e[0].elapsed_time(e[1]) for e in ev]
    search_ms = [e[1].elapsed_time(e[4]) for e in ev]
    gemm_ms = [e[2].elapsed_time(e[3]) for e in ev]
    pack_ms = [e[4].elapsed_time(e[5]) for e in ev]
    total_ms = replicas.max_over_ranks(float(np.sum(step_ms)), dev)

    # correctness guard on the timed result (cheap): a valid ratio and finite losses
    best = int(res.best_j.item())
    assert 0 <= best < J and torch.isfinite(res.losses).all()

    fold_ms = measure_fold(Wd, res.scales)
    rules_ms = measure_rules(Xd, Wd, act, J)
    int8_pack_ms = measure_int8_pack(Wd, res.scales)
    # The deployment GEMMs are another workload than the search: they are timed after a 2 s pause, so that
    # the SM clock has left the power-capped level the seconds-long search loop holds it at (both they and
    # their cuBLAS comparator see the same clock).
    torch.cuda.synchronize()
    time.sleep(2.0)
    w4 = measure_w4a16(Xd, Wd, res.scales)
    e2e = None if args.no_e2e else measure_e2e(args, Xh, Wh, dev, J)
    e2e_ms = replicas.max_over_ranks(e2e["ms"] if e2e else 0.0, dev)
    if e2e:
        e2e["ms"] = e2e_ms

    if rank != 0:
        return
    peaks, peaks_src = load_peaks()
    ms_per_step = total_ms / args.steps
    value = replicas.job_throughput(J * args.steps, world, total_ms / 1e3)
    flops = J * 2.0 * N * O * K
    gemm_avg_s = float(np.mean(gemm_ms)) / 1e3
    achieved_tflops = flops / gemm_avg_s / 1e12
    traffic, traffic_how = profiled_traffic(wl.number)
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        cpu = oracle_sample(wl, X, W)
        cpu.pop("threads", None)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(wl, world),
        "effective_tflops": flops / (ms_per_step / 1e3) / 1e12,
        "breakdown_ms": {"act_stats": float(np.mean(act_ms)), "search": float(np.mean(search_ms)),
                         "loss_gemm": float(np.mean(gemm_ms)), "quantize_pack": float(np.mean(pack_ms))},
        "roofline": {"bound": "tensor", "kernel": "loss_gemm_kernel", "achieved": achieved_tflops,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved_tflops / peaks["bf16_tflops"],
                     "frac_of_sustained": achieved_tflops / peaks["bf16_tflops_sustained"],
                     "peak_source": f"{peaks_src} bf16 burst (MEASURED_PEAKS.json)" if peaks_src == "measured"
                     else "fallback 1.59 PFLOP/s",
                     "traffic": traffic, "traffic_source": traffic_how, "algorithmic_flops_per_launch": flops},
        "hbm": {"act_stats_gbs": (2.0 * N * K + 4.0 * K) / (np.mean(act_ms) / 1e3) / 1e9,
                "quantize_pack_gbs": (2.0 * O * K + 4.0 * K + O * K / 2.0 + 8.0 * O * K / 128)
                / (np.mean(pack_ms) / 1e3) / 1e9,
                "fold_gbs": (4.0 * O * K + 4.0 * K) / (fold_ms / 1e3) / 1e9,
                "int8_pack_gbs": (2.0 * O * K + 4.0 * K + 1.0 * O * K + 4.0 * O) / (int8_pack_ms / 1e3) / 1e9,
                "peak_gbs": peaks.get("hbm_gbs")},
        "search_ms_by_rule": rules_ms,
        "w4a16": w4a16_summary(w4, peaks),
        "gpu_launches": launches_per_step(J) * args.steps,
        "clocks": clocks,
        "best_j": best,
        "wall_s": wall,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if e2e is not None:
        line["e2e"] = {"value": replicas.job_throughput(J, world, e2e["ms"] / 1e3), "unit": UNIT,
                       "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                       "ms_per_step": e2e["ms"], "pipelining": e2e["overlap"]}
    print(json.dumps(line), flush=True)


def measure_fold(Wd, scales):
    """Applying the chosen scales to W (W diag(s), bf16 out): an HBM-bound step after the search."""
    import torch

    from weight_only_quantization_act_b200 import awq

    out = torch.empty_like(Wd)
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=Wd.device)
    times = []
    for i in range(6):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        awq.scale_columns(Wd, scales, out=out)
        e1.record()
        torch.cuda.synchronize()
        if i >= 2:
            times.append(e0.elapsed_time(e1))
    return float(np.mean(times))


def measure_rules(Xd, Wd, act, J):
    """awq_search time with each candidate-scale rule (the default, page 2's weight-aware rule, page 1's
    RMS-normalised 11-point grid), and with the INT8 per-channel quantizer in place of INT4."""
    import torch

    from weight_only_quantization_act_b200 import awq

    out = {}
    N, K = Xd.shape
    ws = awq._workspace(awq.search_workspace_size(N, K, Wd.shape[0], J), Xd.device, None)  # shared by all rules
    for rule, n, quant in (("p4", J, "int4"), ("weight_aware", J, "int4"), ("rms", 11, "int4"), ("p4", J, "int8")):
        res = awq.search(Xd, Wd, act, n_grid=n, rule=rule, quant=quant, workspace=ws)
        times = []
        for i in range(4):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            awq.search(Xd, Wd, act, n_grid=n, rule=rule, quant=quant, workspace=res.workspace, out=res)
            e1.record()
            torch.cuda.synchronize()
            if i >= 1:
                times.append(e0.elapsed_time(e1))
        out[f"{rule}_n{n}" if quant == "int4" else f"{quant}_{rule}_n{n}"] = float(np.mean(times))
    return out


def measure_int8_pack(Wd, scales):
    """awq_quantize_pack_int8 alone (L2 flushed before every launch), in ms."""
    import torch

    from weight_only_quantization_act_b200 import awq

    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=Wd.device)
    times = []
    for i in range(6):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        awq.quantize_pack_int8(Wd, scales)
        e1.record()
        torch.cuda.synchronize()
        if i >= 2:
            times.append(e0.elapsed_time(e1))
    return float(np.mean(times))


def measure_w4a16(Xd, Wd, scales):
    """The deployment GEMM on the quantized layer, and a dense bf16 GEMM (torch.matmul) of the same shapes
    on the same harness as a comparator (measurement only): a prefill of all N calibration tokens and a
    16-token decode on the whole layer, and a 4096-token prefill and a 16-token decode on its first 4096
    rows and in-features.
    Each is timed cold: a batch of launches, each after a 512 MiB L2 flush, between two events, minus a
    batch of flushes alone timed just before (single launches of a few microseconds would be read off an
    event clock that ticks in ~2 us steps); the median over seven such pairs. Batches hold 40 launches,
    fewer for launches longer than 0.1 ms."""
    import torch

    from weight_only_quantization_act_b200 import awq

    lib = awq.load_library()
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=Xd.device)

    def batch(fn, n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            flush.zero_()
            if fn is not None:
                fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    def cold_ms(fn):
        n = 4
        est = batch(fn, n) - batch(None, n)
        n = int(max(3, min(40, 4.0 / max(est, 1e-3))))  # ~4 ms of kernel time per batch
        # flush-only and flush+kernel batches alternate, so a drift of the flush time cancels in each
        # pair; the median of the pairs' differences is the kernel time
        diffs = []
        for _ in range(7):
            base = batch(None, n)
            diffs.append(batch(fn, n) - base)
        return float(np.median(diffs))

    out = {}
    layers = [("", Xd, Wd, scales)]
    if Xd.shape[1] > 4096 or Wd.shape[0] > 4096:
        Ks, Os = min(4096, Xd.shape[1]), min(4096, Wd.shape[0])
        layers.append(("small_", Xd[:, :Ks].contiguous(), Wd[:Os, :Ks].contiguous(), scales[:Ks].contiguous()))
    for prefix, X, W, s in layers:
        codes, steps, zeros = awq.quantize_pack(W, s)
        Xs = awq.scale_columns(X, s, divide=True)
        ws = torch.zeros(lib.awq_w4a16_workspace_size(X.shape[1], codes.shape[0]), dtype=torch.uint8,
                         device=X.device)
        cases = (("prefill", Xs[:4096].contiguous()), ("decode", Xs[:16].contiguous())) if prefix else \
            (("prefill", Xs), ("decode", Xs[:16].contiguous()))
        for name, A in cases:
            Y = torch.empty((A.shape[0], codes.shape[0]), dtype=torch.bfloat16, device=X.device)
            fn = lambda A=A, Y=Y: awq.w4a16_gemm(A, codes, steps, zeros, out=Y, workspace=ws)
            ref = lambda A=A, Y=Y, W=W: torch.matmul(A, W.t(), out=Y)
            out[f"{prefix}{name}_ms"] = cold_ms(fn)
            out[f"{prefix}{name}_bf16_ms"] = cold_ms(ref)
            out[f"{prefix}{name}_shape"] = [int(A.shape[0]), int(X.shape[1]), int(codes.shape[0])]
    return out


def w4a16_summary(w4, peaks):
    """Rates of the W4A16 launches: prefill in TFLOP/s, decodes in HBM GB/s of their algorithmic bytes
    (codes O*K/2, steps and zeros 8*O*K/128, X' 2*M*K, Y 2*M*O), each beside the bf16 comparator."""
    out = {"comparator": "torch.matmul bf16 on the same shapes and harness (measurement only)"}
    for prefix in ("", "small_"):
        if f"{prefix}prefill_ms" not in w4:
            continue
        M, K, O = w4[f"{prefix}prefill_shape"]
        ms = w4[f"{prefix}prefill_ms"]
        tf = 2.0 * M * O * K / (ms / 1e3) / 1e12
        out.update({f"{prefix}prefill_shape_MKO": [M, K, O], f"{prefix}prefill_ms": ms,
                    f"{prefix}prefill_bf16_ms": w4[f"{prefix}prefill_bf16_ms"], f"{prefix}prefill_tflops": tf,
                    f"{prefix}prefill_frac_of_peak": tf / peaks["bf16_tflops"]})
    for prefix in ("", "small_"):
        if f"{prefix}decode_ms" not in w4:
            continue
        M, K, O = w4[f"{prefix}decode_shape"]
        nbytes = 0.5 * O * K + 8.0 * O * K / 128 + 2.0 * M * K + 2.0 * M * O
        ms = w4[f"{prefix}decode_ms"]
        out.update({f"{prefix}decode_shape_MKO": [M, K, O], f"{prefix}decode_ms": ms,
                    f"{prefix}decode_bf16_ms": w4[f"{prefix}decode_bf16_ms"],
                    f"{prefix}decode_gbs": nbytes / (ms / 1e3) / 1e9,
                    f"{prefix}decode_frac_of_hbm": nbytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]})
    return out


def launches_per_step(n_grid: int) -> int:
    """Kernels of one step: statistic (2), scale table (2), fused producer + loss GEMM (1), finalize (1),
    pack (1)."""
    return 2 + 2 + 1 + 1 + 1


def measure_e2e(args, Xh, Wh, dev, J):
    """Same path through the public API with pinned host buffers; every step's H2D copy of X and W and
    D2H read of its results are inside the timed region. As a user quantizing layer after layer would,
    the next step's inputs are uploaded on a copy stream (into the other of two device buffers) while
    the current step runs; the pinned host buffers are allocated once, before timing."""
    import torch

    from weight_only_quantization_act_b200 import awq

    Xp, Wp = Xh.pin_memory(), Wh.pin_memory()
    comp = torch.cuda.current_stream()
    copy = torch.cuda.Stream()
    down = torch.cuda.Stream()
    Xd = [torch.empty(Xp.shape, dtype=Xp.dtype, device=dev) for _ in range(2)]
    Wd = [torch.empty(Wp.shape, dtype=Wp.dtype, device=dev) for _ in range(2)]
    copied = [torch.cuda.Event() for _ in range(2)]
    freed = [torch.cuda.Event() for _ in range(2)]
    keys = ("codes", "steps", "zeros", "scales", "losses", "best_j")
    host = {}

    def upload(i):  # inputs of step i into buffer i % 2
        b = i % 2
        with torch.cuda.stream(copy):
            if i >= 2:
                copy.wait_event(freed[b])
            Xd[b].copy_(Xp, non_blocking=True)
            Wd[b].copy_(Wp, non_blocking=True)
            copied[b].record(copy)

    def compute(i):
        b = i % 2
        comp.wait_event(copied[b])
        out = awq.quantize_layer(Xd[b], Wd[b], n_grid=J, stream=comp)
        freed[b].record(comp)
        # the results go down on their own stream while the next step runs
        with torch.cuda.stream(down):
            down.wait_event(freed[b])
            for k in keys:
                if k not in host:
                    host[k] = torch.empty(out[k].shape, dtype=out[k].dtype, pin_memory=True)
                host[k].copy_(out[k], non_blocking=True)
                out[k].record_stream(down)

    def run(steps, start=None):
        if start is not None:
            copy.wait_event(start)
        upload(0)
        for i in range(steps):
            if i + 1 < steps:
                upload(i + 1)
            compute(i)

    run(3)
    torch.cuda.synchronize()
    comp.wait_stream(down)
    steps = max(3, min(args.steps, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    run(steps, start=e0)
    comp.wait_stream(down)  # the last step's results are on the host before the clock stops
    e1.record(comp)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    h2d = Xh.numel() * 2 + Wh.numel() * 2
    d2h = sum(h.numel() * h.element_size() for h in host.values())
    return {"ms": ms, "h2d": int(h2d), "d2h": int(d2h),
            "overlap": "next step's H2D and previous step's D2H on their own streams"}


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    import datetime

    import torch
    import torch.distributed as dist

    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group(backend="nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
