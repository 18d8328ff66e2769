"""The smoke entry point's checks (search, fold, W4A16 prefill and decode, INT8 pack on the workload-1
layer, each against the oracle), run on the library the other GPU tests load."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_smoke_checks():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import __graft_entry__

    __graft_entry__.smoke_checks()
