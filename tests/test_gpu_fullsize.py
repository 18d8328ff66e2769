"""Full-size parity on the five synthetic workloads, in the launch configuration bench.py times.

The oracle's full fp64 losses take minutes to hours at these sizes, so they come from
tests/golden/search_w<n>.json (written by tests/golden/make_golden.py, which calls only the oracle). The
test checks that its inputs are the ones the golden values were computed on (sha256), then compares:
  - act_mean and the whole scale table bit for bit against the live oracle;
  - every per-ratio loss within 2e-2 of the golden oracle loss, and the argmin rule;
  - the scales, codes, steps and zeros at the chosen ratio against the golden hashes (and, sampled, row
    by row against the live oracle);
  - sampled per-tile partial sums against the live oracle's fp64 sum over the same 32 x 256 block.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import awq_oracle as orc
from tests._helpers import LOSS_RTOL, assert_bits_equal, bf16_to_device, check_argmin_rule, loss_rel_err
from weight_only_quantization_act_b200 import awq, inputs

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_golden(n):
    path = os.path.join(GOLDEN, f"search_w{n}.json")
    if not os.path.exists(path):
        pytest.fail(f"missing golden file {path}: run tests/golden/make_golden.py --workloads {n}")
    with open(path) as f:
        return json.load(f)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    awq.load_library()


@pytest.mark.parametrize("number", [1, 2, 3, 4, 5])
def test_workload_full_size(number):
    wl = inputs.workload(number)
    g = load_golden(number)
    X, W, _ = inputs.make_inputs(wl)
    assert inputs.sha256_of(X) == g["sha256_X"] and inputs.sha256_of(W) == g["sha256_W"], \
        "synthetic inputs differ from the ones the golden values were computed on"
    Xd, Wd = bf16_to_device(X), bf16_to_device(W)

    act = awq.act_stats(Xd)
    act_h = act.cpu().numpy()
    assert inputs.sha256_of(act_h) == g["sha256_act_mean"], "act_mean differs from the oracle"

    res = awq.search(Xd, Wd, act, n_grid=wl.n_grid)
    assert awq.search_status(res) == 0
    losses = res.losses.cpu().numpy()
    err = loss_rel_err(losses, g["losses"])
    print(f"workload {number}: max loss rel err {err.max():.2e}, best {int(res.best_j.item())} "
          f"(oracle {g['best_j']})")
    assert np.all(err <= LOSS_RTOL), (err.max(), losses, g["losses"])
    best = int(res.best_j.item())
    assert best == int(np.argmin(losses))
    check_argmin_rule(best, g["losses"])

    table = orc.scale_table(act_h, wl.n_grid)
    assert inputs.sha256_of(table) == g["sha256_table"], "oracle scale table differs from the golden one"
    assert_bits_equal(res.scales, table[best], "scales")

    codes, steps, zeros = awq.quantize_pack(Wd, res.scales)
    codes_h = codes.cpu().numpy().view(np.uint32)
    steps_h, zeros_h = steps.cpu().numpy(), zeros.cpu().numpy()
    if best == g["best_j"]:
        assert inputs.sha256_of(table[best]) == g["sha256_scales"]
        assert inputs.sha256_of(codes_h) == g["sha256_codes"]
        assert inputs.sha256_of(steps_h) == g["sha256_steps"]
        assert inputs.sha256_of(zeros_h) == g["sha256_zeros"]
    rng = np.random.default_rng(number)
    rows = np.unique(np.concatenate([[0, wl.O - 1], rng.integers(0, wl.O, 6)]))
    wc, ws, wz = orc.quantize_pack(W[rows], table[best])
    assert np.array_equal(codes_h[rows], wc)
    assert_bits_equal(steps_h[rows], ws, "steps rows")
    assert_bits_equal(zeros_h[rows], wz, "zeros rows")

    # sampled tile partial sums, recomputed by the oracle on the same 32-token x 256-row blocks
    lay = awq.search_layout(wl.N, wl.K, wl.O, wl.n_grid)
    parts = awq.tile_partials(res, wl.N, wl.K, wl.O, wl.n_grid).cpu().numpy()
    sub = lay.tile_n // lay.partials_per_tile
    picks = [(0, 0, 0, 0), (wl.n_grid - 1, lay.tiles_o - 1, lay.tiles_n - 1, lay.partials_per_tile - 1)]
    for _ in range(3):
        picks.append((int(rng.integers(wl.n_grid)), int(rng.integers(lay.tiles_o)), int(rng.integers(lay.tiles_n)),
                      int(rng.integers(lay.partials_per_tile))))
    for j, a, b, e in picks:
        r0 = b * lay.tile_n + e * sub
        xb = X[r0:r0 + sub]
        w_rows = W[a * lay.tile_o:min(wl.O, (a + 1) * lay.tile_o)]
        w_hat, _, _, _ = orc.pseudo_quantize(w_rows, table[j])
        E = inputs.bf16_bits_to_f32(xb).astype(np.float64) @ (
            inputs.bf16_bits_to_f32(w_rows).astype(np.float64) - w_hat.astype(np.float64)).T
        want = float((E * E).sum())
        assert abs(parts[j, a, b, e] - want) <= LOSS_RTOL * want, (number, j, a, b, e, parts[j, a, b, e], want)
