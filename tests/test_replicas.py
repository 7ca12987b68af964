"""Host logic of the multi-GPU path (token-sharded replicas), run as two
gloo ranks on the CPU: the ranks' tokens differ, the timing maximum and
the barrier are collective, and the whole-job rate counts every rank's
units over the slowest rank's time."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    from rank_fp8_residual_b200 import replicas
    from synth_inputs import make_x
    assert replicas.rank_env() == (rank, world, rank)
    replicas.init("gloo", timeout_s=60)
    try:
        assert replicas.world_size() == world
        # each rank's own device time; the job's time is the slowest one
        my_time = 1.0 + 0.25 * rank
        t_max = replicas.max_over_ranks(my_time)
        replicas.barrier()
        x = make_x(8, 32, seed=replicas.token_seed(rank))
        results[rank] = (t_max, x.float().sum().item(),
                         replicas.aggregate_rate(100.0, 4, t_max, replicas.world_size()))
    finally:
        replicas.finalize()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, results), nprocs=world, join=True)
        res = dict(results)
    assert set(res) == {0, 1}
    assert res[0][0] == res[1][0] == 1.25          # max over ranks, seen by every rank
    assert res[0][1] != res[1][1]                  # the ranks' tokens differ
    assert res[0][2] == res[1][2] == pytest.approx(2 * 4 * 100.0 / 1.25)


def test_single_process_defaults():
    from rank_fp8_residual_b200 import replicas
    assert replicas.world_size() == 1
    assert replicas.max_over_ranks(3.5) == 3.5
    replicas.barrier()  # a no-op without a process group
    assert replicas.token_seed(0) == 0 and replicas.token_seed(3) == 1003
    assert replicas.aggregate_rate(10.0, 2, 4.0, 1) == 5.0
