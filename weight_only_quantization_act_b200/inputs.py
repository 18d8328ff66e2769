"""Seeded synthetic inputs for the AWQ scale search (calibration activations X and weights W).

This module holds no part of the method's arithmetic: it only draws the random matrices that both the
CPU oracle and the CUDA path consume. Calibration sets and trained weights are not available here, so
the workloads are synthetic stand-ins with the statistics the AWQ pages describe: a few activation
channels carry large magnitudes at fixed positions ("Outlier Activations" on the gsyq.cn AWQ page; the
"activation statistics" section on the hncyxsy.com outlier page says their positions barely change).

Recipe (every step deterministic given the seed, same bits on every x86-64 host with this numpy):
  * generators: ``numpy.random.SeedSequence(seed).spawn(2)`` gives one PCG64 stream for X and one
    for W, seed = 1000 + workload number (so X can be truncated to its first rows without
    changing W);
  * outlier channels: ``permutation(K)[:n_out]`` from the X stream, drawn before X itself;
  * X for the attention-input workloads: standard normals (float32 ziggurat), outlier columns times
    ``factor``; X for the down_proj workloads: ``silu(a) * b`` with a, b standard normals, evaluated in
    float64, outlier columns times ``factor``;
  * W: standard normals times sigma; the fused QKV workload draws q, k, v in that order and stacks rows;
  * every value is rounded to float32 and then to bfloat16, both round-to-nearest-even.

Matrices are returned as ``numpy.uint16`` arrays holding bfloat16 bit patterns (row-major, [rows, K]).
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import hashlib
import os

import numpy as np

__all__ = ["Workload", "WORKLOADS", "workload", "make_inputs", "f32_to_bf16_bits", "bf16_bits_to_f32",
           "random_bf16", "sha256_of"]


@dataclasses.dataclass(frozen=True)
class Workload:
    number: int            # 1-based workload number (also selects the seed)
    name: str
    N: int                 # calibration tokens (rows of X)
    K: int                 # input features
    out_rows: tuple        # output rows of each linear sharing X (concatenated in this order)
    sigma: float           # weight standard deviation
    n_out: int             # number of outlier channels
    factor: float          # outlier magnitude multiplier
    gated: bool            # X = silu(a) * b instead of plain normals
    group: int = 128
    n_grid: int = 20

    @property
    def O(self) -> int:
        return int(sum(self.out_rows))

    @property
    def seed(self) -> int:
        return 1000 + self.number

    @property
    def flops_per_candidate(self) -> int:
        return 2 * self.N * self.O * self.K


WORKLOADS = {
    1: Workload(1, "tiny 512x256 / 256x256", 512, 256, (256,), 0.02, 3, 50.0, False),
    2: Workload(2, "LLaMA-7B q_proj 4096x4096 / 4096x4096", 4096, 4096, (4096,), 0.02, 41, 30.0, False),
    3: Workload(3, "fused QKV (GQA) 8192x4096 / (4096+1024+1024)x4096", 8192, 4096, (4096, 1024, 1024), 0.02,
                20, 100.0, False),
    4: Workload(4, "down_proj 8192x14336 / 4096x14336", 8192, 14336, (4096,), 0.015, 29, 40.0, True),
    5: Workload(5, "70B down_proj 16384x28672 / 8192x28672", 16384, 28672, (8192,), 0.01, 29, 150.0, True),
}


_GEN_THREADS = max(1, min(8, os.cpu_count() or 1))


def workload(number: int) -> Workload:
    return WORKLOADS[int(number)]


def f32_to_bf16_bits(x) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return the 16-bit patterns.

    In 32-bit integer arithmetic: for every finite or infinite value the bit pattern plus 0x7FFF plus the
    kept lowest bit stays below 2^32 (the largest, -inf, is 0xFF800000); NaNs are replaced afterwards."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    r = ((u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(b) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def _silu_times(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    a64 = a.astype(np.float64)
    return (a64 / (1.0 + np.exp(-a64))) * b.astype(np.float64)


def make_inputs(wl: Workload, rows: int | None = None, chunk_rows: int = 2048):
    """Draw (X_bits [N,K] uint16, W_bits [O,K] uint16, outlier_channels) for a workload.

    ``rows`` truncates X to its first rows; they are the same rows as in the full matrix."""
    sx, sw = np.random.SeedSequence(wl.seed).spawn(2)
    rng = np.random.Generator(np.random.PCG64(sx))
    rngw = np.random.Generator(np.random.PCG64(sw))
    N, K = wl.N, wl.K
    outliers = np.sort(rng.permutation(K)[: wl.n_out])
    mult = np.ones(K, np.float64)
    mult[outliers] = wl.factor
    keep = N if rows is None else min(int(rows), N)
    X = np.empty((keep, K), np.uint16)

    def transform(r0, a, b):  # element-wise, so row pieces can run on worker threads
        v = _silu_times(a, b) * mult if wl.gated else a.astype(np.float64) * mult
        X[r0:r0 + a.shape[0]] = f32_to_bf16_bits(v.astype(np.float32))

    # The draws stay in one sequential stream (chunk by chunk, a then b); their element-wise transforms
    # run on a few threads (numpy releases the GIL), at most two chunks in flight.
    pending = []
    with concurrent.futures.ThreadPoolExecutor(max_workers=_GEN_THREADS) as pool:
        for r0 in range(0, keep, chunk_rows):
            r1 = min(keep, r0 + chunk_rows)
            a = rng.standard_normal((r1 - r0, K), dtype=np.float32)
            b = rng.standard_normal((r1 - r0, K), dtype=np.float32) if wl.gated else None
            if len(pending) >= 2:
                for f in pending.pop(0):
                    f.result()
            step = max(1, -(-(r1 - r0) // _GEN_THREADS))
            pending.append([pool.submit(transform, r0 + i, a[i:i + step], None if b is None else b[i:i + step])
                            for i in range(0, r1 - r0, step)])
        for fs in pending:
            for f in fs:
                f.result()
    Ws = []
    for o in wl.out_rows:
        Ws.append(f32_to_bf16_bits(
            (rngw.standard_normal((o, K), dtype=np.float32).astype(np.float64) * wl.sigma).astype(np.float32)))
    W = np.concatenate(Ws, axis=0) if len(Ws) > 1 else Ws[0]
    return X, W, outliers


def random_bf16(shape, seed: int, scale: float = 1.0, outliers: int = 0, factor: float = 1.0):
    """Small ad-hoc bf16 matrix (rows, K) for ragged parity cases; optional outlier columns."""
    rng = np.random.Generator(np.random.PCG64(seed))
    rows, K = shape
    cols = np.sort(rng.permutation(K)[:outliers]) if outliers else np.empty(0, np.int64)
    v = rng.standard_normal((rows, K), dtype=np.float32).astype(np.float64) * scale
    if outliers:
        v[:, cols] *= factor
    return f32_to_bf16_bits(v.astype(np.float32))


def sha256_of(*arrays) -> str:
    h = hashlib.sha256()
    for a in arrays:
        h.update(np.ascontiguousarray(a).tobytes())
    return h.hexdigest()
