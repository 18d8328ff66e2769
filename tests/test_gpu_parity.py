"""GPU parity of every step of the path against the CPU oracle, through the C ABI (via the ctypes
binding), on sizes the oracle finishes in seconds: several tiles, ragged tails, edge cases.

Bit-exact: act_mean, the scale table, best_j (up to the tolerance rule), scales, codes, steps, zeros.
Within 2e-2 relative: the per-ratio losses and the per-tile partial sums."""
import numpy as np
import pytest
import torch

from oracle import awq_oracle as orc
from tests._helpers import (LOSS_RTOL, assert_bits_equal, bf16_to_device, check_argmin_rule, loss_rel_err)
from tests.test_oracle_pins import near_midpoint_cases, on_grid_weight
from weight_only_quantization_act_b200 import awq, inputs

pytestmark = pytest.mark.gpu
F32 = np.float32


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    awq.load_library()


# ------------------------------------------------------------------------------------------------ a1
@pytest.mark.parametrize("shape", [(512, 256), (300, 640), (1, 256), (257, 128), (1000, 8), (4096, 1024)])
def test_act_stats_bit_exact(shape):
    X = inputs.random_bf16(shape, seed=shape[0] * 7 + shape[1], outliers=min(3, shape[1]), factor=60)
    got = awq.act_stats(bf16_to_device(X))
    assert_bits_equal(got, orc.act_mean(X), f"act_mean {shape}")


def test_act_stats_strided_input():
    wide = inputs.random_bf16((333, 512), seed=5, outliers=2, factor=30)
    Xd = bf16_to_device(wide)[:, 128:384]          # row stride 512, 256 columns
    assert Xd.stride(0) == 512
    assert_bits_equal(awq.act_stats(Xd), orc.act_mean(wide[:, 128:384]), "strided")


@pytest.mark.parametrize("shape", [(600, 1030), (37, 2), (513, 2056), (256, 1024), (51277, 1030)])
def test_act_stats_special_magnitudes(shape):
    """Zeros, subnormals and magnitudes across the whole finite bf16 exponent range, both signs, with a
    ragged last column block (K % 8 != 0) and row counts off the load blocks. The small shapes take the
    narrow chunk-sum kernel; 51277 x 1030 (201 chunks, the last ragged, x 3 column blocks) takes the wide
    one, whose last column block holds 6 columns."""
    rng = np.random.default_rng(shape[0] + 31 * shape[1])
    u16 = np.uint16
    e = rng.integers(0, 255, shape, dtype=u16)
    small = rng.integers(0, 2, shape, dtype=np.uint8).astype(bool)
    e[small] = e[small] & u16(3)                   # half the entries: exponent fields 0-3 (subnormal, tiny)
    X = (rng.integers(0, 2, shape, dtype=u16) << u16(15)) | (e << u16(7)) | rng.integers(0, 128, shape, dtype=u16)
    X[rng.integers(0, 10, shape, dtype=np.uint8) == 0] = 0
    ld = -(-shape[1] // 8) * 8                     # row stride: the next multiple of 8
    wide = np.zeros((shape[0], ld), np.uint16)
    wide[:, :shape[1]] = X
    Xd = bf16_to_device(wide)[:, :shape[1]]
    assert_bits_equal(awq.act_stats(Xd), orc.act_mean(X), f"special magnitudes {shape}")


def test_act_stats_tiny_workload():
    X, _, _ = inputs.make_inputs(inputs.workload(1))
    assert_bits_equal(awq.act_stats(bf16_to_device(X)), orc.act_mean(X), "workload 1")


# ------------------------------------------------------------------------------------------------ a2
def edge_act_vector():
    rng = np.random.default_rng(77)
    v = np.concatenate([rng.random(300) * 2, 10.0 ** rng.uniform(-9, 3, 300),
                        [0.0, 1e-30, 1.4e-45, 1e-4, 1.0, 2.0, 256.0, 3.0e4]]).astype(F32)
    return v


@pytest.mark.parametrize("exact_pow", [False, True])
def test_scale_table_bit_exact_edges(exact_pow):
    act = edge_act_vector()
    got = awq.scale_table(torch.from_numpy(act).cuda(), 20, exact_pow=exact_pow)
    assert_bits_equal(got, orc.scale_table(act, 20), f"scale table exact_pow={exact_pow}")


@pytest.mark.parametrize("exact_pow", [False, True])
def test_scale_table_near_fp32_midpoints(exact_pow):
    cases = near_midpoint_cases(count=24, seed=9)
    act = np.array([a for a, _ in cases] + [0.5, 4.0], F32)
    got = awq.scale_table(torch.from_numpy(act).cuda(), 20, exact_pow=exact_pow)
    assert_bits_equal(got, orc.scale_table(act, 20), "near-midpoint scale table")


def test_scale_table_other_grids():
    act = edge_act_vector()[:257]
    for n in (1, 7, 64):
        got = awq.scale_table(torch.from_numpy(act).cuda(), n)
        assert_bits_equal(got, orc.scale_table(act, n), f"n_grid={n}")


# ------------------------------------------------------------------------------------------------ a6
def adversarial_weight():
    rng = np.random.default_rng(88)
    w = (rng.standard_normal((40, 512)) * 0.02).astype(F32)
    w[0, :128] = 0.3                              # constant group: step at the floor
    w[1, :] = -0.125
    w[2, :256] += 3.0                             # all-positive groups: negative zero point
    w[3, :256] -= 3.0                             # all-negative groups
    q = np.arange(128) % 16
    w[4, :128] = ((q - 3) * 2.0 ** -7)            # on the grid
    w[5, :128] = ((q + 0.5) * 2.0 ** -7)          # every quotient a half-integer (ties to even)
    w[5, 0], w[5, 1] = 0.0, 15 * 2.0 ** -7
    w[6, 128:256] = 0.0                           # zero group
    w[7, :] = (rng.standard_normal(512) * 1e-7)   # tiny values, step at the floor
    w[8, :] = (rng.standard_normal(512) * 50)     # large values
    return inputs.f32_to_bf16_bits(w)


@pytest.mark.parametrize("flags", [0, awq.FLAG_EXACT_DIVISION])
@pytest.mark.parametrize("scale_kind", ["ones", "table"])
def test_quantize_pack_bit_exact(flags, scale_kind):
    W = adversarial_weight()
    K = W.shape[1]
    if scale_kind == "ones":
        s = np.ones(K, F32)
    else:
        X = inputs.random_bf16((200, K), seed=3, outliers=4, factor=80)
        s = orc.scale_table(orc.act_mean(X), 20)[13]
    codes, steps, zeros = awq.quantize_pack(bf16_to_device(W), torch.from_numpy(s).cuda(), flags=flags)
    wcodes, wsteps, wzeros = orc.quantize_pack(W, s)
    assert np.array_equal(codes.cpu().numpy().view(np.uint32), wcodes)
    assert_bits_equal(steps, wsteps, "steps")
    assert_bits_equal(zeros, wzeros, "zeros")


def test_quantize_pack_very_wide_rows():
    """More 1024-in-feature segments than CTAs fit on the device (576 > 3 per SM x 148), so a CTA walks
    several segments and restages the segment's scales between them: K = 589824 (576 whole segments) and
    K = 589440 (the last segment 640 in-features, its upper lanes idle)."""
    for K in (589824, 589824 - 384):
        W = inputs.random_bf16((9, K), seed=21, scale=0.02)
        s = (1.0 + np.random.default_rng(22).random(K)).astype(F32)
        codes, steps, zeros = awq.quantize_pack(bf16_to_device(W), torch.from_numpy(s).cuda())
        wc, ws, wz = orc.quantize_pack(W, s)
        assert np.array_equal(codes.cpu().numpy().view(np.uint32), wc), K
        assert_bits_equal(steps, ws, f"steps K={K}")
        assert_bits_equal(zeros, wz, f"zeros K={K}")


def test_quantize_pack_ragged_rows_and_stride():
    W = inputs.random_bf16((77, 640), seed=12, scale=0.02)
    s = orc.scale_table(orc.act_mean(inputs.random_bf16((64, 640), 13, outliers=3, factor=40)), 20)[17]
    big = np.zeros((77, 768), np.uint16)
    big[:, :640] = W
    Wd = bf16_to_device(big)[:, :640]
    codes, steps, zeros = awq.quantize_pack(Wd, torch.from_numpy(s).cuda())
    wc, ws, wz = orc.quantize_pack(W, s)
    assert np.array_equal(codes.cpu().numpy().view(np.uint32), wc)
    assert_bits_equal(steps, ws, "steps")
    assert_bits_equal(zeros, wz, "zeros")


# ------------------------------------------------------------------------------------------------ search
def run_and_compare(X, W, n_grid=20, flags=0, Ws=None):
    N, K = X.shape
    Xd = bf16_to_device(X)
    Wd = [bf16_to_device(w) for w in Ws] if Ws is not None else bf16_to_device(W)
    act = awq.act_stats(Xd)
    ref = orc.search(X, W, n_grid=n_grid)
    assert_bits_equal(act, ref["act_mean"], "act_mean")
    res = awq.search(Xd, Wd, act, n_grid=n_grid, flags=flags)
    assert awq.search_status(res) == 0
    losses = res.losses.cpu().numpy()
    err = loss_rel_err(losses, ref["losses"])
    assert np.all(err <= LOSS_RTOL), (err.max(), losses, ref["losses"])
    best = int(res.best_j.item())
    assert best == int(np.argmin(losses))
    check_argmin_rule(best, ref["losses"])
    assert_bits_equal(res.scales, ref["table"][best], "scales")
    codes, steps, zeros = awq.quantize_pack(Wd, res.scales)
    wc, ws, wz = orc.quantize_pack(W, ref["table"][best])
    assert np.array_equal(codes.cpu().numpy().view(np.uint32), wc)
    assert_bits_equal(steps, ws, "steps")
    assert_bits_equal(zeros, wz, "zeros")
    return res, ref, err


def test_search_tiny_workload():
    X, W, _ = inputs.make_inputs(inputs.workload(1))
    res, ref, err = run_and_compare(X, W)
    assert int(res.best_j.item()) == ref["best_j"]
    print("max loss rel err", err.max())


def test_search_ragged_tails():
    X = inputs.random_bf16((300, 384), seed=21, outliers=4, factor=50)
    W = inputs.random_bf16((600, 384), seed=22, scale=0.02)
    run_and_compare(X, W)


def test_search_single_row_single_output():
    X = inputs.random_bf16((1, 128), seed=23, outliers=1, factor=20)
    W = inputs.random_bf16((1, 128), seed=24, scale=0.05)
    run_and_compare(X, W, n_grid=8)


def test_search_shared_input_qkv():
    X = inputs.random_bf16((520, 256), seed=31, outliers=3, factor=100)
    Wq = inputs.random_bf16((256, 256), seed=32, scale=0.02)
    Wk = inputs.random_bf16((64, 256), seed=33, scale=0.02)
    Wv = inputs.random_bf16((64, 256), seed=34, scale=0.02)
    run_and_compare(X, np.concatenate([Wq, Wk, Wv]), Ws=[Wq, Wk, Wv])


def test_search_on_grid_weight_zero_loss_at_ratio_zero():
    W = on_grid_weight(256, 256, 41)
    X = inputs.random_bf16((256, 256), seed=42, outliers=2, factor=30)
    res, ref, _ = run_and_compare(X, W)
    assert res.losses[0].item() == 0.0
    assert int(res.best_j.item()) == 0


def test_search_flags_do_not_change_results():
    """The exact paths (IEEE division for every quotient and for the unscale w_hat = deq / s, the
    double-double power for every scale) give the same scales, argmin, codes, steps and zeros; the losses
    move by at most the bf16 rounding of a weight error that changed by one fp32 ulp, and stay within the
    tolerance of the oracle, whose unscale is the IEEE division."""
    X = inputs.random_bf16((384, 512), seed=51, outliers=3, factor=40)
    W = inputs.random_bf16((512, 512), seed=52, scale=0.02)
    Xd, Wd = bf16_to_device(X), bf16_to_device(W)
    act = awq.act_stats(Xd)
    ref = orc.search(X, W, n_grid=20)
    a = awq.search(Xd, Wd, act)
    b = awq.search(Xd, Wd, act, flags=awq.FLAG_EXACT_DIVISION | awq.FLAG_EXACT_POW)
    c = awq.search(Xd, Wd, act)
    d = awq.search(Xd, Wd, act, flags=awq.FLAG_EXACT_DIVISION | awq.FLAG_EXACT_POW)
    assert torch.equal(a.losses, c.losses) and torch.equal(b.losses, d.losses), "search must be deterministic"
    assert torch.equal(a.scales, b.scales) and int(a.best_j.item()) == int(b.best_j.item())
    for res in (a, b):
        err = loss_rel_err(res.losses.cpu().numpy(), ref["losses"])
        assert np.all(err <= LOSS_RTOL), err.max()
        check_argmin_rule(int(res.best_j.item()), ref["losses"])
    assert np.all(loss_rel_err(b.losses.cpu().numpy(), a.losses.cpu().numpy()) <= 1e-3)
    pa = awq.quantize_pack(Wd, a.scales)
    pb = awq.quantize_pack(Wd, b.scales, flags=awq.FLAG_EXACT_DIVISION)
    for x, y in zip(pa, pb):
        assert torch.equal(x, y)


def test_tile_partials_match_oracle():
    X, W, _ = inputs.make_inputs(inputs.workload(1))
    N, K = X.shape
    O = W.shape[0]
    Xd, Wd = bf16_to_device(X), bf16_to_device(W)
    act = awq.act_stats(Xd)
    res = awq.search(Xd, Wd, act)
    parts = awq.tile_partials(res, N, K, O).cpu().numpy()
    lay = awq.search_layout(N, K, O)
    rows = lay.tile_n // lay.partials_per_tile
    table = orc.scale_table(orc.act_mean(X), 20)
    x = inputs.bf16_bits_to_f32(X).astype(np.float64)
    w = inputs.bf16_bits_to_f32(W).astype(np.float64)
    for j in (0, 5, 19):
        w_hat, _, _, _ = orc.pseudo_quantize(W, table[j])
        E = x @ (w - w_hat.astype(np.float64)).T
        for a in range(parts.shape[1]):
            for b in range(parts.shape[2]):
                for q in range(lay.partials_per_tile):
                    r0 = b * lay.tile_n + rows * q
                    blk = E[r0:r0 + rows, a * lay.tile_o:(a + 1) * lay.tile_o]
                    want = float((blk * blk).sum())
                    assert abs(parts[j, a, b, q] - want) <= LOSS_RTOL * want + 1e-300, (j, a, b, q)


# ------------------------------------------------------------------------------------------------ scale rules
@pytest.mark.parametrize("exact_pow", [False, True])
def test_scale_table_rules_bit_exact(exact_pow):
    act = edge_act_vector()
    rng = np.random.default_rng(131)
    wm = np.concatenate([rng.random(act.shape[0] - 2) * 0.05, [0.0, 1e-30]]).astype(F32)
    got = awq.scale_table(torch.from_numpy(act).cuda(), 20, exact_pow=exact_pow, rule="weight_aware",
                          weight_mean=torch.from_numpy(wm).cuda())
    assert_bits_equal(got, orc.scale_table_weight_aware(act, wm, 20), "weight-aware table")
    got = awq.scale_table(torch.from_numpy(act).cuda(), 11, exact_pow=exact_pow, rule="rms")
    assert_bits_equal(got, orc.scale_table_rms(act, 11), "rms table")


@pytest.mark.parametrize("rule,n_grid", [("weight_aware", 20), ("rms", 11)])
def test_search_with_alternative_rules(rule, n_grid):
    X = inputs.random_bf16((300, 384), seed=61, outliers=4, factor=50)
    W = inputs.random_bf16((600, 384), seed=62, scale=0.02)
    Xd, Wd = bf16_to_device(X), bf16_to_device(W)
    act = awq.act_stats(Xd)
    res = awq.search(Xd, Wd, act, n_grid=n_grid, rule=rule)
    assert awq.search_status(res) == 0
    ref = orc.search(X, W, n_grid=n_grid, mode=rule)
    losses = res.losses.cpu().numpy()
    assert np.all(loss_rel_err(losses, ref["losses"]) <= LOSS_RTOL)
    best = int(res.best_j.item())
    check_argmin_rule(best, ref["losses"])
    assert_bits_equal(res.scales, ref["table"][best], "scales")
