"""Ulysses context parallelism on CPU process groups (gloo, world sizes 2
and 4): the token-shard <-> head-group all-to-alls are exact inverses and
place every (head, token) row where the layout says, and the context-parallel
JVP equals the single-process result. The local attention here is the
float64 oracle (on GPUs it is the CUDA kernel, covered by
tests/test_gpu_ulysses.py)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def problem(B=1, H=4, T=6, F=4, d=16, seed=3):
    from oracle import MaskSpec, TEACHER_FORCING
    spec = MaskSpec(TEACHER_FORCING, T, F, 1)
    g = torch.Generator().manual_seed(seed)
    xs = [torch.randn(B, H, spec.length, d, generator=g) for _ in range(6)]
    return spec, xs


def oracle_attn(spec):
    from oracle import jvp_attention

    def attn(q, k, v, dq, dk, dv, mask):
        o, do, lse = jvp_attention(q, k, v, dq, dk, dv, spec)
        return (torch.from_numpy(o).float(), torch.from_numpy(do).float(),
                torch.from_numpy(lse).float())
    return attn


def worker(rank, world, B, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    from attention_jvp_continuous_b200.ulysses import head_to_seq, seq_to_head, ulysses_jvp_attn
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        spec, xs = problem(B=B)
        L, P = spec.length, world
        Ls, Hp = L // P, xs[0].shape[1] // P
        shard = [x[:, :, rank * Ls:(rank + 1) * Ls].contiguous() for x in xs]
        # layout: this rank gets heads [rank Hp, (rank+1) Hp) of every token
        hx = seq_to_head(shard)
        ok_layout = all(torch.equal(hx[i], xs[i][:, rank * Hp:(rank + 1) * Hp]) for i in range(6))
        back = head_to_seq([hx[i] for i in range(6)])
        ok_round = all(torch.equal(back[i], shard[i]) for i in range(6))
        o, do, lse = ulysses_jvp_attn(*shard, None, attn=oracle_attn(spec))
        out[rank] = (ok_layout, ok_round, o.numpy(), do.numpy(), lse.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,B", [(2, 1), (4, 1), (2, 2)])
def test_ulysses_matches_single_process(world, B):
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(worker, args=(world, B, free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    spec, xs = problem(B=B)
    ro, rdo, rl = oracle_attn(spec)(*xs, None)
    Ls = spec.length // world
    for r in range(world):
        ok_layout, ok_round, o, do, lse = out[r]
        assert ok_layout and ok_round
        sl = slice(r * Ls, (r + 1) * Ls)
        np.testing.assert_allclose(o, ro[:, :, sl].numpy(), atol=1e-6)
        np.testing.assert_allclose(do, rdo[:, :, sl].numpy(), atol=1e-6)
        np.testing.assert_allclose(lse, rl[:, :, sl].numpy(), atol=1e-6)
