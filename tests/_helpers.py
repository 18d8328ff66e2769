"""Shared helpers of the test-suite (device transfer of bf16 bit matrices, comparisons)."""
import numpy as np
import torch

LOSS_RTOL = 2e-2   # per-ratio loss tolerance against the fp64 oracle


def bf16_to_device(bits: np.ndarray, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def f32_bits(a) -> np.ndarray:
    if isinstance(a, torch.Tensor):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def assert_bits_equal(got, want, what=""):
    g, w = f32_bits(got), f32_bits(want)
    assert g.shape == w.shape, (what, g.shape, w.shape)
    bad = np.nonzero(g != w)
    assert bad[0].size == 0, (f"{what}: {bad[0].size} of {g.size} differ; first at {tuple(b[0] for b in bad)}: "
                              f"got {g.view(np.float32)[tuple(b[0] for b in bad)]!r} "
                              f"want {w.view(np.float32)[tuple(b[0] for b in bad)]!r}")


def loss_rel_err(got, want) -> np.ndarray:
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    return np.abs(got - want) / np.maximum(np.abs(want), 1e-300)


def check_argmin_rule(gpu_best: int, oracle_losses) -> None:
    """The GPU may pick another ratio only where the oracle's best two losses are within the tolerance."""
    ol = np.asarray(oracle_losses, np.float64)
    ob = int(np.argmin(ol))  # first minimum
    if gpu_best == ob:
        return
    assert 0 <= gpu_best < ol.size
    assert ol[gpu_best] <= ol[ob] * (1 + LOSS_RTOL), (gpu_best, ob, ol[gpu_best], ol[ob])
