"""GPU parity of the INT8 symmetric per-channel quantizer (search and pack) against the CPU oracle.

Bit-exact: codes, steps and the chosen scales. Within 2e-2 relative: the per-ratio losses. The full-size
case reads tests/golden/search_int8_w2.json (written by tests/golden/make_golden.py --quant int8, which
calls only the oracle)."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import awq_oracle as orc
from tests._helpers import LOSS_RTOL, assert_bits_equal, bf16_to_device, check_argmin_rule, loss_rel_err
from weight_only_quantization_act_b200 import awq, inputs

pytestmark = pytest.mark.gpu
F32 = np.float32
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    awq.load_library()


def adversarial_rows(K=512):
    rng = np.random.default_rng(808)
    w = (rng.standard_normal((19, K)) * 0.02).astype(F32)
    w[0, :] = 0.0                                    # zero row: step at the floor, all codes 0
    w[1, :] = -0.125                                 # constant row: every code -127
    w[2, 7] = 23.0                                   # one outlier flattens the rest of the row to 0
    w[3, :] = rng.standard_normal(K) * 1e-7          # tiny row: step at the floor
    w[4, :] = rng.standard_normal(K) * 50            # large values
    lv = (np.arange(K) % 255) - 127
    w[5, :] = lv * 2.0 ** -9                         # on the grid: codes are the levels
    w[6, :] = ((np.arange(K) % 252) - 125.5) * 2.0 ** -9  # step 2^-9 exactly: half-integer quotients, ties to even
    w[6, 0] = 127 * 2.0 ** -9
    w[7, :] = np.abs(w[7, :])                        # one-signed rows
    w[8, :] = -np.abs(w[8, :])
    return inputs.f32_to_bf16_bits(w)


def pack_and_compare(W, s, flags=0, Wd=None):
    Wd = bf16_to_device(W) if Wd is None else Wd
    codes, steps = awq.quantize_pack_int8(Wd, torch.from_numpy(np.ascontiguousarray(s, F32)).cuda(), flags=flags)
    wc, ws = orc.quantize_pack_int8(W, s)
    got = codes.cpu().numpy()
    bad = np.argwhere(got != wc)
    assert bad.size == 0, (f"{len(bad)} codes differ, first {tuple(bad[0])}: got {got[tuple(bad[0])]}, "
                           f"want {wc[tuple(bad[0])]}")
    assert_bits_equal(steps, ws, "steps")
    return got, steps


@pytest.mark.parametrize("flags", [0, awq.FLAG_EXACT_DIVISION])
@pytest.mark.parametrize("scale_kind", ["ones", "table"])
def test_int8_pack_bit_exact_edges(flags, scale_kind):
    W = adversarial_rows()
    K = W.shape[1]
    if scale_kind == "ones":
        s = np.ones(K, F32)
    else:
        s = orc.scale_table(orc.act_mean(inputs.random_bf16((200, K), seed=3, outliers=4, factor=80)), 20)[11]
    codes, _ = pack_and_compare(W, s, flags)
    if scale_kind == "ones":
        assert np.all(codes[0] == 0) and np.all(codes[1] == -127)
        assert np.array_equal(codes[5], ((np.arange(K) % 255) - 127).astype(np.int8))


def test_int8_pack_worked_example_row():
    """The outlier page's case on the GPU: with 23.0 in the row, 0.03 codes to 0; without it, to 38."""
    w = np.zeros((2, 8), F32)
    w[0, :3] = [23.0, 0.03, -5.0]
    w[1, :3] = [0.1, 0.03, -0.05]
    W = inputs.f32_to_bf16_bits(w)
    codes, _ = pack_and_compare(W, np.ones(8, F32))
    wq = inputs.bf16_bits_to_f32(W)
    assert codes[0, 1] == 0 and codes[0, 0] == 127
    assert codes[1, 1] == np.rint(wq[1, 1] / F32(wq[1, 0] / F32(127))) and codes[1, 0] == 127


@pytest.mark.parametrize("shape", [(1, 8), (77, 136), (300, 1024), (1000, 4104)])
def test_int8_pack_ragged_shapes(shape):
    O, K = shape
    W = inputs.random_bf16((O, K), seed=O + K, scale=0.02)
    s = np.exp(np.random.default_rng(K).uniform(-2, 2, K)).astype(F32)
    pack_and_compare(W, s)


def test_int8_pack_strided_rows():
    W = inputs.random_bf16((65, 640), seed=12, scale=0.02)
    big = np.zeros((65, 768), np.uint16)
    big[:, :640] = W
    s = orc.scale_table(orc.act_mean(inputs.random_bf16((64, 640), 13, outliers=3, factor=40)), 20)[17]
    pack_and_compare(W, s, Wd=bf16_to_device(big)[:, :640])


def test_int8_pack_rejects_bad_arguments():
    Wd = bf16_to_device(inputs.random_bf16((4, 12), seed=1))
    with pytest.raises(RuntimeError, match="multiple of 8"):
        awq.quantize_pack_int8(Wd, torch.ones(12, device="cuda"))


# ------------------------------------------------------------------------------------------------ search
def search_and_compare(X, W, n_grid=20, flags=0):
    Xd, Wd = bf16_to_device(X), bf16_to_device(W)
    act = awq.act_stats(Xd)
    res = awq.search(Xd, Wd, act, n_grid=n_grid, flags=flags, quant="int8")
    assert awq.search_status(res) == 0
    ref = orc.search(X, W, n_grid=n_grid, quant="int8")
    err = loss_rel_err(res.losses.cpu().numpy(), ref["losses"])
    assert np.all(err <= LOSS_RTOL), (err.max(), res.losses.cpu().numpy(), ref["losses"])
    best = int(res.best_j.item())
    check_argmin_rule(best, ref["losses"])
    assert_bits_equal(res.scales, ref["table"][best], "scales")
    pack_and_compare(W, ref["table"][best], Wd=Wd)
    return res, ref, err


def test_int8_search_tiny_workload():
    X, W, _ = inputs.make_inputs(inputs.workload(1))
    res, ref, err = search_and_compare(X, W)
    assert int(res.best_j.item()) == ref["best_j"]
    print("int8 max loss rel err", err.max())


def test_int8_search_ragged_tails_and_outlier_rows():
    X = inputs.random_bf16((300, 384), seed=21, outliers=4, factor=50)
    w = inputs.bf16_bits_to_f32(inputs.random_bf16((600, 384), seed=22, scale=0.02)).copy()
    w[5, 17] = 3.0      # a row whose step is set by one weight
    w[9, :] = 0.0       # a zero row
    search_and_compare(X, inputs.f32_to_bf16_bits(w))


def test_int8_search_single_row_and_flags_agree():
    X = inputs.random_bf16((1, 128), seed=23, outliers=1, factor=20)
    W = inputs.random_bf16((1, 128), seed=24, scale=0.05)
    search_and_compare(X, W, n_grid=8)
    X = inputs.random_bf16((384, 512), seed=51, outliers=3, factor=40)
    W = inputs.random_bf16((512, 512), seed=52, scale=0.02)
    Xd, Wd = bf16_to_device(X), bf16_to_device(W)
    act = awq.act_stats(Xd)
    a = awq.search(Xd, Wd, act, quant="int8")
    b = awq.search(Xd, Wd, act, quant="int8", flags=awq.FLAG_EXACT_DIVISION | awq.FLAG_EXACT_POW)
    # the exact paths change only the unscale w_hat = deq / s (an IEEE division instead of deq * RN32(1/s)),
    # which moves a weight error by at most one fp32 ulp before its bf16 rounding
    assert torch.equal(a.scales, b.scales) and int(a.best_j.item()) == int(b.best_j.item())
    rel = (a.losses - b.losses).abs() / b.losses.abs()
    assert float(rel.max()) <= 1e-3, rel
    search_and_compare(X, W, flags=awq.FLAG_EXACT_DIVISION | awq.FLAG_EXACT_POW)  # the exact run against the oracle


def test_int8_search_rejects_group_with_int8():
    Xd = bf16_to_device(inputs.random_bf16((16, 128), seed=1))
    Wd = bf16_to_device(inputs.random_bf16((16, 128), seed=2))
    act = awq.act_stats(Xd)
    lib = awq.load_library()
    ws = torch.empty(awq.search_workspace_size(16, 128, 16, 20), dtype=torch.uint8, device="cuda")
    out = torch.empty(20, dtype=torch.float64, device="cuda")
    bj = torch.empty(1, dtype=torch.int32, device="cuda")
    sc = torch.empty(128, dtype=torch.float32, device="cuda")
    rc = lib.awq_search_ex(Xd.data_ptr(), 16, 128, 128, Wd.data_ptr(), 16, 128, act.data_ptr(), 128, 20,
                           awq.FLAG_QUANT_INT8, ws.data_ptr(), ws.numel(), out.data_ptr(), bj.data_ptr(),
                           sc.data_ptr(), None)
    assert rc == 2 and b"per channel" in lib.awq_last_error()


def test_int8_search_full_size_workload2():
    path = os.path.join(GOLDEN, "search_int8_w2.json")
    with open(path) as f:
        g = json.load(f)
    wl = inputs.workload(2)
    X, W, _ = inputs.make_inputs(wl)
    assert inputs.sha256_of(X) == g["sha256_X"] and inputs.sha256_of(W) == g["sha256_W"]
    Xd, Wd = bf16_to_device(X), bf16_to_device(W)
    act = awq.act_stats(Xd)
    res = awq.search(Xd, Wd, act, n_grid=wl.n_grid, quant="int8")
    assert awq.search_status(res) == 0
    losses = res.losses.cpu().numpy()
    err = loss_rel_err(losses, g["losses"])
    print(f"int8 workload 2: max loss rel err {err.max():.2e}, best {int(res.best_j.item())} (oracle {g['best_j']})")
    assert np.all(err <= LOSS_RTOL), (err.max(), losses, g["losses"])
    best = int(res.best_j.item())
    check_argmin_rule(best, g["losses"])
    table = orc.scale_table(act.cpu().numpy(), wl.n_grid)
    assert inputs.sha256_of(table) == g["sha256_table"]
    assert_bits_equal(res.scales, table[best], "scales")
    codes, steps = awq.quantize_pack_int8(Wd, res.scales)
    codes_h, steps_h = codes.cpu().numpy(), steps.cpu().numpy()
    if best == g["best_j"]:
        assert inputs.sha256_of(codes_h) == g["sha256_codes"]
        assert inputs.sha256_of(steps_h) == g["sha256_steps"]
    rows = np.unique(np.concatenate([[0, wl.O - 1], np.random.default_rng(2).integers(0, wl.O, 6)]))
    wc, ws = orc.quantize_pack_int8(W[rows], table[best])
    assert np.array_equal(codes_h[rows], wc)
    assert_bits_equal(steps_h[rows], ws, "steps rows")
