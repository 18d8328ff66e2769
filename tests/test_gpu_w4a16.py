"""The W4A16 deployment GEMM (a 'next' row) against the oracle, and the whole deploy path end to end."""
import numpy as np
import pytest
import torch

from oracle import awq_oracle as orc
from tests._helpers import bf16_to_device
from weight_only_quantization_act_b200 import awq, inputs

pytestmark = pytest.mark.gpu
F32 = np.float32


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    awq.load_library()


DECODE_MAX_TOKENS = 64   # up to this many tokens the library runs the few-token kernel


def check_against_oracle(Xp, words, steps, zeros, Y):
    """Many tokens (bf16 weight operand): |Y - ref| <= 2^-8 |ref| + (K/16 + 16) 2^-23 sum_k |x w|, the bf16
    output rounding plus fp32 accumulation.

    Few tokens (the weights enter at their fp32 dequantized value; per group g the tensor cores sum
    x (128 + q) exactly-rounded in fp32, and y += step (S_g - (128 + z) Sx_g) in fp32): |Y - ref| <= 2^-8 |ref|
    + 2^-24 sum_g step_g A_g (128 * 143 + 130 (128 + |z_g|) + (G + 18) (15 + |z_g|)) + 2^-23 sum_k |x w|, where
    A_g = sum over the group of |x|: the first term of the bracket bounds the accumulation of S_g (128
    additions of terms up to 143 |x|), the second that of Sx_g and the zero-point product, the third the
    running sums over groups and slices (at most 16); the last term covers the weight's own fp32 rounding."""
    M, K = Xp.shape
    x64 = inputs.bf16_bits_to_f32(Xp).astype(np.float64)
    got = Y.float().cpu().numpy().astype(np.float64)
    if M > DECODE_MAX_TOKENS:
        ref = orc.w4a16_matmul(Xp, words, steps, zeros)
        deq16 = inputs.bf16_bits_to_f32(orc.round_f32_to_bf16(orc.dequant_w4(words, steps, zeros))).astype(np.float64)
        tol = 2.0 ** -8 * np.abs(ref) + (K / 16 + 16) * 2.0 ** -23 * (np.abs(x64) @ np.abs(deq16).T)
    else:
        ref = orc.w4a16_matmul(Xp, words, steps, zeros, weights="fp32")
        deq = orc.dequant_w4(words, steps, zeros).astype(np.float64)
        G = K // 128
        A = np.abs(x64).reshape(M, G, 128).sum(axis=2)                     # [M, G]
        z = np.abs(np.asarray(zeros, np.float64))
        coef = np.asarray(steps, np.float64) * (128 * 143 + 130 * (128 + z) + (G + 18) * (15 + z))  # [O, G]
        tol = 2.0 ** -8 * np.abs(ref) + 2.0 ** -24 * (A @ coef.T) + 2.0 ** -23 * (np.abs(x64) @ np.abs(deq).T)
    bad = np.abs(got - ref) > tol
    assert not bad.any(), (np.argwhere(bad)[:5], got[bad][:5], ref[bad][:5])


def quantized(O, K, seed):
    W = inputs.random_bf16((O, K), seed, scale=0.02)
    s = orc.scale_candidates(orc.act_mean(inputs.random_bf16((64, K), seed + 1, outliers=3, factor=40)),
                             orc.ratio(8, 20))
    return W, s, orc.quantize_pack(W, s)


@pytest.mark.parametrize("M,K,O", [(300, 384, 600), (1, 128, 8), (256, 256, 256), (513, 4096, 1032)])
def test_w4a16_matches_oracle(M, K, O):
    _, _, (words, steps, zeros) = quantized(O, K, M + K + O)
    Xp = inputs.random_bf16((M, K), 7 * M + 1, scale=1.0)
    Y = awq.w4a16_gemm(bf16_to_device(Xp), torch.from_numpy(words.view(np.int32)).cuda(),
                       torch.from_numpy(steps).cuda(), torch.from_numpy(zeros).cuda())
    torch.cuda.synchronize()
    check_against_oracle(Xp, words, steps, zeros, Y)


# Few tokens on layers with more 128-row blocks than CTAs fit on the device at once (B200: 296 at 16
# tokens, 148 above), so the GEMM runs in several waves with one slice per block, next to a layer that
# fits one wave; run twice on one workspace (the per-block counters are handed back at zero).
@pytest.mark.parametrize("M,K,O", [(16, 256, 38400), (40, 384, 19200), (16, 256, 512)])
def test_w4a16_decode_more_blocks_than_one_wave(M, K, O):
    _, _, (words, steps, zeros) = quantized(O, K, M + K + O + 5)
    Xp = inputs.random_bf16((M, K), 3 * M + 2, scale=1.0)
    lib = awq.load_library()
    ws = torch.zeros(lib.awq_w4a16_workspace_size(K, O), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        Y = awq.w4a16_gemm(bf16_to_device(Xp), torch.from_numpy(words.view(np.int32)).cuda(),
                           torch.from_numpy(steps).cuda(), torch.from_numpy(zeros).cuda(), workspace=ws)
        torch.cuda.synchronize()
        check_against_oracle(Xp, words, steps, zeros, Y)


# Many tokens at the tile counts the prefill kernel really runs: tiles of 512 tokens x 256 weight rows
# handed out dynamically over the device's CTA pairs (74 on B200), so most pairs run a second and a
# third tile. This is where the one-tile-ahead index publishing, the code ring across tiles and the
# accumulator handover after the epilogue are exercised: 4096^3 is 128 tiles, 4096 x 1024 x 4096 the same
# tile count with a short K loop, and 2600 x 512 x 4104 (ragged in tokens and rows) 102 tiles.
@pytest.mark.parametrize("M,K,O", [(4096, 4096, 4096), (4096, 1024, 4096), (2600, 512, 4104)])
def test_w4a16_prefill_many_tiles_per_pair(M, K, O):
    _, _, (words, steps, zeros) = quantized(O, K, M + 2 * K + O)
    Xp = inputs.random_bf16((M, K), 5 * M + 9, scale=1.0)
    Y = awq.w4a16_gemm(bf16_to_device(Xp), torch.from_numpy(words.view(np.int32)).cuda(),
                       torch.from_numpy(steps).cuda(), torch.from_numpy(zeros).cuda())
    torch.cuda.synchronize()
    check_against_oracle(Xp, words, steps, zeros, Y)


def test_deploy_path_end_to_end():
    """search -> pack -> fold the scales out of X -> W4A16 GEMM reproduces X W^T up to the quantization
    error the search measured (mean squared output error within 25% of the search's best loss)."""
    X = inputs.random_bf16((1024, 1024), 31, outliers=10, factor=40)
    W = inputs.random_bf16((512, 1024), 32, scale=0.02)
    Xd, Wd = bf16_to_device(X), bf16_to_device(W)
    out = awq.quantize_layer(Xd, Wd)
    Xs = awq.scale_columns(Xd, out["scales"], divide=True)
    Y = awq.w4a16_gemm(Xs, out["codes"], out["steps"], out["zeros"]).double()
    ref = Xd.double() @ Wd.double().T
    mse = float(((Y - ref) ** 2).mean())
    best = float(out["losses"][int(out["best_j"].item())])
    assert 0.5 * best < mse < 1.25 * best, (mse, best)


# ------------------------------------------------------------------------------------------------ few tokens
# M <= 64 runs the decode kernel (weight rows on the MMA's M side, k-blocks split into slices over
# independent CTAs whose fp32 partial sums go to the workspace, where the last CTA of a row block adds
# them in slice order); the shapes cover several slice counts, slices left without k-blocks (K = 384,
# 640), ragged weight-row blocks and every token rounding.
@pytest.mark.parametrize("M,K,O", [(1, 4096, 4096), (5, 384, 600), (16, 256, 136), (17, 1024, 520),
                                   (33, 640, 264), (64, 2048, 1024), (64, 128, 8), (65, 512, 256)])
def test_w4a16_few_tokens_match_oracle(M, K, O):
    _, _, (words, steps, zeros) = quantized(O, K, 3 * M + K + O)
    Xp = inputs.random_bf16((M, K), 11 * M + 5, scale=1.0)
    Y = awq.w4a16_gemm(bf16_to_device(Xp), torch.from_numpy(words.view(np.int32)).cuda(),
                       torch.from_numpy(steps).cuda(), torch.from_numpy(zeros).cuda())
    torch.cuda.synchronize()
    check_against_oracle(Xp, words, steps, zeros, Y)


@pytest.mark.parametrize("M,K,O", [(64, 256, 136), (16, 384, 256), (48, 1024, 520), (33, 4096, 128)])
def test_w4a16_few_tokens_one_hot_columns_exact(M, K, O):
    """Token m of X' is one-hot at in-feature k_m with a power-of-two value: its row of Y is then exactly
    bf16(x * RN32((q - z) * step)) of column k_m (the group sums reduce to one exact product, the zero-point
    term cancels exactly, and the other groups add zeros), so every nibble, the operand permutation, the
    swizzles, the group's step and zero and the split-K reduction are checked bit for bit."""
    rng = np.random.default_rng(M + K + O)
    _, _, (words, steps, zeros) = quantized(O, K, 7 * M + K + O)
    ks = rng.choice(K, size=M, replace=M > K)
    ks[:min(M, 8)] = np.arange(min(M, 8))  # the eight nibbles of the first word
    vals = np.array([0x3F80, 0x4000, 0x3E80, 0xBF00, 0x4100], np.uint16)  # 1, 2, 0.25, -0.5, 8
    Xp = np.zeros((M, K), np.uint16)
    Xp[np.arange(M), ks] = vals[np.arange(M) % vals.size]
    Y = awq.w4a16_gemm(bf16_to_device(Xp), torch.from_numpy(words.view(np.int32)).cuda(),
                       torch.from_numpy(steps).cuda(), torch.from_numpy(zeros).cuda())
    torch.cuda.synchronize()
    want = orc.round_f32_to_bf16(orc.w4a16_matmul(Xp, words, steps, zeros, weights="fp32").astype(np.float32))
    got = Y.cpu().view(torch.int16).numpy().view(np.uint16)
    bad = np.argwhere(got != want)
    assert bad.size == 0, (bad[:5], got[tuple(bad[0])], want[tuple(bad[0])])


def test_w4a16_few_tokens_deterministic_and_strided():
    _, _, (words, steps, zeros) = quantized(1024, 2048, 77)
    wide = inputs.random_bf16((8, 2304), 78, scale=1.0)
    Xd = bf16_to_device(wide)[:, 128:2176]  # row stride 2304
    args = (torch.from_numpy(words.view(np.int32)).cuda(), torch.from_numpy(steps).cuda(),
            torch.from_numpy(zeros).cuda())
    a = awq.w4a16_gemm(Xd, *args)
    b = awq.w4a16_gemm(Xd, *args)
    torch.cuda.synchronize()
    assert torch.equal(a, b), "the split-K reduction adds the slices' partial sums in a fixed order"
    check_against_oracle(np.ascontiguousarray(wide[:, 128:2176]), words, steps, zeros, a)


@pytest.mark.parametrize("M", [4, 300])
def test_w4a16_huge_zero_points(M):
    """Zero points beyond 2^19 (constant groups of large weights at the step floor) take the exact slow
    dequantization path in both kernels."""
    O, K = 256, 512
    _, _, (words, steps, zeros) = quantized(O, K, 91)
    steps, zeros = steps.copy(), zeros.copy()
    steps[3, :] = F32(1e-5)
    zeros[3, :] = F32(-3_000_000.0)
    steps[40, 1] = F32(2.0 ** -17)
    zeros[40, 1] = F32(9_999_999.0)
    zeros[41, 2] = F32(-524_288.0)
    zeros[42, 0] = F32(524_287.0)
    Xp = inputs.random_bf16((M, K), 92 + M, scale=1.0)
    Y = awq.w4a16_gemm(bf16_to_device(Xp), torch.from_numpy(words.view(np.int32)).cuda(),
                       torch.from_numpy(steps).cuda(), torch.from_numpy(zeros).cuda())
    torch.cuda.synchronize()
    check_against_oracle(Xp, words, steps, zeros, Y)


@pytest.mark.parametrize("M,K,O", [(513, 4096, 1032), (1024, 2048, 768), (16, 4096, 1024), (4096, 4096, 4096)])
def test_w4a16_repeated_runs_are_bit_identical(M, K, O):
    """Both kernels add in a fixed order, so any run-to-run difference is a race (a buffer handed back
    or reused too early); many k-blocks per tile and repeated launches give one room to show. 4096^3 runs
    128 tiles on the CTA pairs, so pairs hand tiles over to their next tile many times."""
    _, _, (words, steps, zeros) = quantized(O, K, 5 * M + K + O)
    Xp = inputs.random_bf16((M, K), 13 * M + 3, scale=1.0)
    Xd = bf16_to_device(Xp)
    args = (torch.from_numpy(words.view(np.int32)).cuda(), torch.from_numpy(steps).cuda(),
            torch.from_numpy(zeros).cuda())
    first = awq.w4a16_gemm(Xd, *args)
    torch.cuda.synchronize()
    check_against_oracle(Xp, words, steps, zeros, first)
    for _ in range(24):
        assert torch.equal(awq.w4a16_gemm(Xd, *args), first)


def test_w4a16_shared_workspace_across_calls_and_shapes():
    """One workspace, zero-filled once, serves every later call: the few-token kernel's per-block
    counters are handed back at zero by each call, whatever the shape (different slice counts), and
    many-token calls with more tiles than CTA pairs (2048 x 5120 outputs: 80 tiles) share it."""
    lib = awq.load_library()
    shapes = [(16, 4096, 1024), (5, 384, 600), (2048, 512, 5120), (64, 2048, 1024), (16, 4096, 1024),
              (2048, 512, 5120), (300, 512, 256), (1, 256, 136)]
    ws = torch.zeros(max(lib.awq_w4a16_workspace_size(K, O) for _, K, O in shapes), dtype=torch.uint8,
                     device="cuda")
    for n, (M, K, O) in enumerate(shapes):
        _, _, (words, steps, zeros) = quantized(O, K, 17 * n + 1)
        Xp = inputs.random_bf16((M, K), 19 * n + 2, scale=1.0)
        for _ in range(3):
            Y = awq.w4a16_gemm(bf16_to_device(Xp), torch.from_numpy(words.view(np.int32)).cuda(),
                               torch.from_numpy(steps).cuda(), torch.from_numpy(zeros).cuda(), workspace=ws)
            torch.cuda.synchronize()
            check_against_oracle(Xp, words, steps, zeros, Y)
