"""The multi-rank host path on CPU: two gloo ranks, as torchrun would start them."""
import os

import numpy as np
import pytest
import torch.multiprocessing as mp

from weight_only_quantization_act_b200 import inputs, replicas


def _rank_main(rank, world, port, out):
    import torch.distributed as dist

    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, lr = replicas.rank_env()
        wl = replicas.replica_workload(inputs.workload(1), r)
        X, W, _ = inputs.make_inputs(wl)
        slowest = replicas.max_over_ranks(1.0 + r)      # rank r pretends to take 1 + r seconds
        out[r] = (r, w, lr, wl.seed, inputs.sha256_of(X, W), slowest,
                  replicas.job_throughput(20, w, slowest))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_replicas_and_max_timing():
    port = 29500 + (os.getpid() % 2000)
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    r0, r1 = res[0], res[1]
    assert (r0[0], r0[1], r0[2]) == (0, 2, 0) and (r1[0], r1[1], r1[2]) == (1, 2, 1)
    assert r0[3] != r1[3] and r0[4] != r1[4], "each rank must quantize its own layer"
    assert r0[5] == r1[5] == 2.0, "timing is the max over ranks"
    assert r0[6] == pytest.approx(20 * 2 / 2.0)


def test_single_process_defaults():
    assert replicas.max_over_ranks(3.5) == 3.5
    wl = inputs.workload(2)
    assert replicas.replica_workload(wl, 0) is wl
    assert replicas.replica_workload(wl, 3).seed == wl.seed + 3000
    assert np.isclose(replicas.job_throughput(20, 4, 0.5), 160.0)
