"""Failure detection without a GPU fault: a wait that nobody satisfies gives up after a short limit,
the status reaches the host, the remaining kernels skip their work, and the context stays usable."""
import numpy as np
import pytest
import torch

from tests._helpers import bf16_to_device
from weight_only_quantization_act_b200 import awq, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    awq.load_library()


def test_injected_stall_reports_timeout_and_context_survives():
    X = inputs.random_bf16((512, 512), seed=1, outliers=2, factor=30)
    W = inputs.random_bf16((512, 512), seed=2, scale=0.02)
    Xd, Wd = bf16_to_device(X), bf16_to_device(W)
    act = awq.act_stats(Xd)
    awq.set_wait_limit_ns(200_000_000)
    try:
        bad = awq.search(Xd, Wd, act, flags=awq.FLAG_INJECT_STALL)
        assert awq.search_status(bad) == 5
        assert "site" in awq.load_library().awq_last_error().decode()
        assert int(bad.best_j.item()) == -1
        assert torch.isnan(bad.losses).all()
    finally:
        awq.set_wait_limit_ns(2_000_000_000)
    good = awq.search(Xd, Wd, act)
    assert awq.search_status(good) == 0
    assert int(good.best_j.item()) >= 0
    assert torch.isfinite(good.losses).all()
    # the same workspace can be reused after a timeout: the status word is cleared per call
    again = awq.search(Xd, Wd, act, workspace=bad.workspace)
    assert awq.search_status(again) == 0
    assert torch.equal(again.losses, good.losses)
