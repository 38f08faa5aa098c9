"""The benchmark's multi-process logic on CPU: two gloo ranks, each with its own
timing, agree on the max over ranks and on the whole-job (weak-scaling) value."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        local_ms = 10.0 + 5.0 * rank                      # rank 1 is slower
        m = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        v = bench.weak_scaling_value(world, n_q=8, n_layers=1, steps=100, tot_ms_max=m)
        bench.barrier(world)
        out[rank] = (m, v)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_value():
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out[0] == out[1]
    m, v = out[0]
    assert m == 15.0
    # 2 ranks x 8 queries x 1 layer x 100 steps in 15 ms
    assert v == pytest.approx(2 * 8 * 100 / 0.015)


def test_single_rank_value_and_max_are_local():
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.weak_scaling_value(1, 4, 4, 10, 2.0) == pytest.approx(4 * 4 * 10 / 0.002)
