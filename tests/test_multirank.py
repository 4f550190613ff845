"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): each rank
draws an independent seeded batch, and the reported time is the maximum
over ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import bench
    from attention_jvp_continuous_b200.inputs import WORKLOADS, make_inputs
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w, r, _ = bench.dist_setup()
        assert (w, r) == (world, rank)
        t = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        wl = WORKLOADS["tiny_tf"]
        (q, *_), _ = make_inputs(wl, seed=bench.rank_seed(wl.seed, rank))
        gathered = [torch.zeros_like(q) for _ in range(world)]
        dist.all_gather(gathered, q)
        out[rank] = (t, bool(torch.equal(gathered[0], gathered[1])))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_independent_inputs():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(worker, args=(world, free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    assert out[0][0] == out[1][0] == 15.0
    assert out[0][1] is False  # ranks draw different inputs


def test_reference_arm_other_ranks_do_nothing(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        ref_rows, steps, warmup = 1, 1, 3
    assert bench.run_reference(A(), None) is None
