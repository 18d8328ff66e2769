"""The statistic entry point that allocates nothing (awq_act_stats_noalloc), called through the C ABI.

It exists for callers that cannot call cudaMalloc when they run the statistic, such as a plugin inside an
inference engine that owns all device memory, or a process that reserved its HBM up front. Its scratch
is a fixed array inside the library, so this file checks it against the workspace entry point
(awq_act_stats, bit-identical results) and against the oracle on calls in a row with different inputs,
since every call reuses the previous call's scratch contents. This file is named to be collected last."""
import ctypes

import numpy as np
import pytest
import torch

from oracle import awq_oracle as orc
from tests._helpers import assert_bits_equal, bf16_to_device
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
    hosts = [inputs.random_bf16(shape, seed, outliers=3, factor=40) for shape, seed in cases]
    Xs = [bf16_to_device(h) for h in hosts]
    refs = [awq.act_stats(X) for X in Xs]
    # the workspace entry point is itself pinned to the oracle; check that link here too
    for h, r in zip(hosts, refs):
        assert_bits_equal(r, orc.act_mean(h), "act_stats against the oracle")
    # two calls in a row on the same input, then other shapes (the larger first call leaves stale
    # partial sums in the shared scratch that the smaller ones must not pick up), then the first again
    order = [0, 0, 1, 2, 0]
    for i in order:
        got = call_noalloc(lib, Xs[i])
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int32), refs[i].view(torch.int32)), f"case {cases[i]}"
        assert_bits_equal(got, orc.act_mean(hosts[i]), f"no-alloc statistic against the oracle, case {cases[i]}")


def test_noalloc_rejects_sizes_beyond_the_scratch(lib):
    # Real device buffers, large enough for the shape the call describes, so that even a call that got
    # past validation would stay inside them. ceil(N/256) * K = 65 * 32768 > 2**21 doubles.
    N, K = 16384 + 256, 32768
    X = torch.zeros((N, K), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(K, dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.awq_act_stats_noalloc(ctypes.c_void_p(X.data_ptr()), N, K, K, ctypes.c_void_p(out.data_ptr()), stream)
    assert rc == 1
    assert "exceed the fixed scratch" in lib.awq_last_error().decode()
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0, "a rejected call launches nothing"


def test_noalloc_binding_checks_its_output_and_makes_no_copy(lib):
    X = bf16_to_device(inputs.random_bf16((512, 256), 5, outliers=2, factor=30))
    with pytest.raises(ValueError):
        awq.act_stats_noalloc(X, torch.empty(255, dtype=torch.float32, device="cuda"))   # too short
    with pytest.raises(ValueError):
        awq.act_stats_noalloc(X, torch.empty(256, dtype=torch.bfloat16, device="cuda"))  # wrong dtype
    with pytest.raises(ValueError):
        awq.act_stats_noalloc(X.t(), torch.empty(512, dtype=torch.float32, device="cuda"))  # strided columns
    out = torch.empty(256, dtype=torch.float32, device="cuda")
    awq.act_stats_noalloc(X, out)
    torch.cuda.synchronize()
    assert torch.equal(out, awq.act_stats(X))
