"""Scale folding on the GPU against the oracle, bit for bit (a 'next' row: applying the chosen scales)."""
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


def bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def scales(n, seed):
    act = orc.act_mean(inputs.random_bf16((100, n), seed, outliers=3, factor=60))
    return orc.scale_candidates(act, orc.ratio(13, 20))


@pytest.mark.parametrize("divide", [False, True])
@pytest.mark.parametrize("shape", [(1, 128), (37, 384), (300, 1024)])
def test_scale_columns_bit_exact(shape, divide):
    A = inputs.random_bf16(shape, shape[0] + 5, scale=0.03)
    s = scales(shape[1], 7)
    got = awq.scale_columns(bf16_to_device(A), torch.from_numpy(s).cuda(), divide=divide)
    assert np.array_equal(bits(got), orc.fold_columns(A, s, divide))


@pytest.mark.parametrize("divide", [False, True])
def test_scale_rows_bit_exact_in_place_and_strided(divide):
    A = inputs.random_bf16((256, 256), 11, scale=0.5)
    s = scales(256, 12)
    dev = bf16_to_device(A)
    awq.scale_rows(dev, torch.from_numpy(s).cuda(), divide=divide, out=dev)
    assert np.array_equal(bits(dev), orc.fold_rows(A, s, divide))
    wide = inputs.random_bf16((64, 512), 13, scale=0.5)
    view = bf16_to_device(wide)[:, 128:384]
    out = awq.scale_rows(view, torch.from_numpy(scales(64, 14)).cuda(), divide=divide)
    assert np.array_equal(bits(out), orc.fold_rows(wide[:, 128:384], scales(64, 14), divide))


def test_fold_helpers_match_the_oracle():
    K, H = 256, 384
    gamma = inputs.random_bf16((1, K), 21, scale=1.0)[0]
    Wq = inputs.random_bf16((128, K), 22, scale=0.02)
    s = scales(K, 23)
    g_d, w_d = bf16_to_device(gamma[None, :])[0], bf16_to_device(Wq)
    awq.fold_norm_linear(g_d, [w_d], torch.from_numpy(s).cuda())
    assert np.array_equal(bits(g_d), orc.fold_columns(gamma[None, :], s, True)[0])
    assert np.array_equal(bits(w_d), orc.fold_columns(Wq, s, False))
    W1 = inputs.random_bf16((H, K), 24, scale=0.05)
    b1 = inputs.random_bf16((1, H), 25, scale=0.1)[0]
    W2 = inputs.random_bf16((K, H), 26, scale=0.05)
    s2 = scales(H, 27)
    d1, db, d2 = bf16_to_device(W1), bf16_to_device(b1[None, :])[0], bf16_to_device(W2)
    awq.fold_linear_linear(d1, db, d2, torch.from_numpy(s2).cuda())
    assert np.array_equal(bits(d1), orc.fold_rows(W1, s2, True))
    assert np.array_equal(bits(db), orc.fold_columns(b1[None, :], s2, True)[0])
    assert np.array_equal(bits(d2), orc.fold_columns(W2, s2, False))
