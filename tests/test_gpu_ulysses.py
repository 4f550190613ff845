"""The context-parallel JVP through NCCL with the CUDA kernel, on the one
GPU a test box has (world size 1: the all-to-alls are identity copies, so
the result equals the kernel called directly, bit for bit, and the float64
oracle within the bf16 parity tolerances). Multi-rank data movement is
covered on CPU process groups by tests/test_ulysses.py."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu


def oracle_mismatch(o, do, lse, xs, w):
    """Whole-sequence outputs against the float64 oracle at the bf16 parity
    tolerances (max|err| <= 2e-2 max|ref|, rel L2 <= 5e-3; LSE within
    1e-3). Returns the failures, empty when all hold."""
    import numpy as np

    from oracle import MaskSpec, jvp_attention
    ref = jvp_attention(*(x.cpu() for x in xs), MaskSpec(w.mode, w.tokens_per_frame,
                                                          w.n_frames, w.chunk))
    bad = []
    for name, got, want in (("O", o, ref[0]), ("dO", do, ref[1])):
        err = got.float().cpu().numpy().astype(np.float64) - want
        rel = np.linalg.norm(err) / np.linalg.norm(want)
        mx = np.abs(err).max() / np.abs(want).max()
        if not (rel <= 5e-3 and mx <= 2e-2):
            bad.append(f"{name}: rel L2 {rel:.3e}, max-abs {mx:.3e}")
    lerr = np.abs(lse.cpu().numpy() - ref[2]).max()
    if not lerr <= 1e-3:
        bad.append(f"LSE: {lerr:.3e}")
    return bad


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def worker(rank, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK="0", WORLD_SIZE="1")
    import datetime

    import torch.distributed as dist

    import attention_jvp_continuous_b200 as ja
    from attention_jvp_continuous_b200.inputs import WORKLOADS, make_inputs
    from attention_jvp_continuous_b200.ulysses import ulysses_jvp_attn
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        w = WORKLOADS["tf"].with_(H=2, tokens_per_frame=96, n_frames=5)
        xs, _ = make_inputs(w, device="cuda")
        mask = ja.Mask(w.mode, w.tokens_per_frame, w.n_frames, w.chunk)
        o1, do1, l1 = ulysses_jvp_attn(*xs, mask)
        o2, do2, l2 = ja.jvp_attn(*xs, mask)
        ja.check_device_error()
        out[0] = bool(torch.equal(o1, o2) and torch.equal(do1, do2) and torch.equal(l1, l2))
        out[1] = oracle_mismatch(o1, do1, l1, xs, w)
    finally:
        dist.destroy_process_group()


def test_ulysses_world_one_equals_kernel():
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(worker, args=(free_port(), out), nprocs=1, start_method="spawn", join=True)
    assert out[0] is True
    assert list(out[1]) == []
