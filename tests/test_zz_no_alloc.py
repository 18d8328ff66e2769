"""The statistic entry point that allocates nothing (awq_act_stats_noalloc), called through the C ABI.

It exists for callers that cannot call cudaMalloc when they run the statistic, such as a plugin inside an
inference engine that owns all device memory, or a process that reserved its HBM up front. Its scratch
is a fixed array inside the library, so this file checks it against the workspace entry point
(awq_act_stats, bit-identical results) on calls in a row with different inputs, since every call reuses
the previous call's scratch contents. This file is named to be collected last."""
import ctypes

import numpy as np
import pytest
import torch

from tests._helpers import bf16_to_device
from weight_only_quantization_act_b200 import awq, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return awq.load_library()


def call_noalloc(lib, X: torch.Tensor) -> torch.Tensor:
    N, K = X.shape
    out = torch.full((K,), float("nan"), dtype=torch.float32, device=X.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.awq_act_stats_noalloc(ctypes.c_void_p(X.data_ptr()), N, K, X.stride(0),
                                   ctypes.c_void_p(out.data_ptr()), stream)
    assert rc == 0, lib.awq_last_error().decode()
    return out


def test_noalloc_matches_workspace_entry_point_on_calls_in_a_row(lib):
    cases = [((4096, 4096), 1), ((700, 1024), 2), ((16384, 128), 3)]
    Xs = [bf16_to_device(inputs.random_bf16(shape, seed, outliers=3, factor=40)) for shape, seed in cases]
    refs = [awq.act_stats(X) for X in Xs]
    # two calls in a row on the same input, then other shapes (the larger first call leaves stale
    # partial sums in the shared scratch that the smaller ones must not pick up), then the first again
    order = [0, 0, 1, 2, 0]
    for i in order:
        got = call_noalloc(lib, Xs[i])
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int32), refs[i].view(torch.int32)), f"case {cases[i]}"


def test_noalloc_rejects_sizes_beyond_the_scratch(lib):
    fake = ctypes.c_void_p(1 << 24)  # rejected during validation, never dereferenced
    N, K = 16384 + 256, 32768        # ceil(N/256) * K = 65 * 32768 > 2**21
    rc = lib.awq_act_stats_noalloc(fake, N, K, K, fake, None)
    assert rc == 1
    assert "exceed the fixed scratch" in lib.awq_last_error().decode()
