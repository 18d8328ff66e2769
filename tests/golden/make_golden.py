"""Write the oracle's full-size expected values for the five synthetic workloads.

    python tests/golden/make_golden.py [--workloads 1 2 3 4 5] [--quant int4|int8]

Calls only the CPU oracle (oracle/awq_oracle.py) on the seeded inputs of
weight_only_quantization_act_b200/inputs.py, and stores per workload (search_w<n>.json):
  - sha256 of the input bits (X, W), so a test can tell whether its inputs are the same;
  - the fp64 losses of all n_grid ratios and the first argmin;
  - sha256 of act_mean, of the scale table, and of the codes / steps / zeros at the best ratio.
With --quant int8 the search scores the symmetric per-channel INT8 quantizer instead and the file is
search_int8_w<n>.json (codes int8 [O, K], steps [O], no zeros).
The full-size loss GEMMs take hours of fp64 time on the GPU machine's host, so the GPU tests read these values
instead of recomputing them (workload 5: 1.5e14 fp64 flops).
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from oracle import awq_oracle as orc  # noqa: E402
from weight_only_quantization_act_b200 import inputs  # noqa: E402


def golden_int8(number: int) -> dict:
    wl = inputs.workload(number)
    t0 = time.time()
    X, W, _ = inputs.make_inputs(wl)
    act = orc.act_mean(X)
    table = orc.scale_table(act, wl.n_grid)
    x64 = inputs.bf16_bits_to_f32(X).astype(np.float64)
    losses = []
    for j in range(wl.n_grid):
        w_hat, _, _ = orc.pseudo_quantize_int8(W, table[j])
        losses.append(orc.loss_of(x64, W, w_hat))
        print(f"workload {number} int8 ratio {j}: {losses[-1]:.6e} ({time.time() - t0:.0f} s)", flush=True)
    best = orc.argmin_first(losses)
    codes, steps = orc.quantize_pack_int8(W, table[best])
    return {
        "workload": number, "quant": "int8", "name": wl.name, "N": wl.N, "K": wl.K, "O": wl.O,
        "n_grid": wl.n_grid, "sha256_X": inputs.sha256_of(X), "sha256_W": inputs.sha256_of(W),
        "sha256_table": inputs.sha256_of(table), "losses": [float(v) for v in losses], "best_j": int(best),
        "sha256_scales": inputs.sha256_of(table[best]), "sha256_codes": inputs.sha256_of(codes),
        "sha256_steps": inputs.sha256_of(steps), "oracle_seconds": time.time() - t0,
    }


def golden(number: int) -> dict:
    wl = inputs.workload(number)
    t0 = time.time()
    X, W, outliers = inputs.make_inputs(wl)
    act = orc.act_mean(X)
    table = orc.scale_table(act, wl.n_grid)
    x64 = inputs.bf16_bits_to_f32(X).astype(np.float64)
    losses = []
    for j in range(wl.n_grid):
        w_hat, _, _, _ = orc.pseudo_quantize(W, table[j], wl.group)
        losses.append(orc.loss_of(x64, W, w_hat))
        print(f"workload {number} ratio {j}: {losses[-1]:.6e} ({time.time() - t0:.0f} s)", flush=True)
    best = orc.argmin_first(losses)
    codes, steps, zeros = orc.quantize_pack(W, table[best], wl.group)
    return {
        "workload": number, "name": wl.name, "N": wl.N, "K": wl.K, "O": wl.O, "n_grid": wl.n_grid,
        "group": wl.group, "outlier_channels": [int(c) for c in outliers],
        "sha256_X": inputs.sha256_of(X), "sha256_W": inputs.sha256_of(W),
        "sha256_act_mean": inputs.sha256_of(act), "sha256_table": inputs.sha256_of(table),
        "losses": [float(v) for v in losses], "best_j": int(best),
        "sha256_scales": inputs.sha256_of(table[best]), "sha256_codes": inputs.sha256_of(codes),
        "sha256_steps": inputs.sha256_of(steps), "sha256_zeros": inputs.sha256_of(zeros),
        "oracle_seconds": time.time() - t0,
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workloads", type=int, nargs="*", default=[1, 2, 3, 4, 5])
    ap.add_argument("--quant", choices=["int4", "int8"], default="int4")
    args = ap.parse_args()
    for n in args.workloads:
        g = golden(n) if args.quant == "int4" else golden_int8(n)
        name = f"search_w{n}.json" if args.quant == "int4" else f"search_int8_w{n}.json"
        with open(os.path.join(HERE, name), "w") as f:
            json.dump(g, f, indent=1)
        print(f"wrote {name} in {g['oracle_seconds']:.0f} s", flush=True)


if __name__ == "__main__":
    main()
