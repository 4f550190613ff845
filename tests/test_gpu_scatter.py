"""The scatter epilogue (jvp_attn_fwd_scatter): the output exchange of Ulysses
context parallelism fused into the JVP kernel. Each of P ranks holds one
head group of all tokens and stores every output row into the token shard
that owns it. On one GPU the P ranks are emulated by P launches, one per
head group, whose destination shards all live on this device; no launch
waits on another. The shards must equal the token slices of the plain
kernel's outputs bit for bit (each output row is computed by the same
instructions, only its address differs), every row must be written exactly
by its own head group, and the fused Ulysses path at world size 1 must equal
the all-to-all path."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import attention_jvp_continuous_b200 as ja
from attention_jvp_continuous_b200.inputs import Workload, make_inputs
from oracle import MaskSpec, jvp_attention

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from attention_jvp_continuous_b200 import build
    build.build()


def oracle_mismatch(o, do, lse, xs, w):
    """Compares whole-sequence outputs with the float64 oracle at the bf16
    parity tolerances (max|err| <= 2e-2 max|ref|, rel L2 <= 5e-3; LSE
    within 1e-3). Returns a list of failures, empty when all hold."""
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


def _shards(B, Ht, L, d, P, fill):
    o = [torch.full((B, Ht, L // P, d), fill, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    do = [torch.full((B, Ht, L // P, d), fill, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    lse = [torch.full((B, Ht, L // P), fill, dtype=torch.float32, device="cuda") for _ in range(P)]
    return o, do, lse


@pytest.mark.parametrize("P", [1, 2, 4, 8])
@pytest.mark.parametrize("mode", [ja.TEACHER_FORCING, ja.FRAME_CAUSAL])
def test_scatter_equals_token_slices(P, mode):
    # 4 heads (8 for 8 shards, the most the epilogue takes), TF: 2 x 3
    # frames x 100 tokens = 600 tokens; frame-causal: 6 x 100. Shards of
    # 600 / P tokens: tile boundaries and shard boundaries do not line up.
    F = 3 if mode == ja.TEACHER_FORCING else 6
    w = Workload("scatter", 2, max(4, P), 128, mode, 100, F, 1, "bf16", 0.1)
    xs, _ = make_inputs(w, device="cuda")
    mask = ja.Mask(w.mode, w.tokens_per_frame, w.n_frames, w.chunk)
    B, Ht, L, d = xs[0].shape
    ref = ja.jvp_attn(*xs, mask)
    o, do, lse = _shards(B, Ht, L, d, P, float("nan"))
    Hl = Ht // P
    for r in range(P):  # rank r: head group [r Hl, (r+1) Hl) of all tokens
        grp = [x[:, r * Hl:(r + 1) * Hl].contiguous() for x in xs]
        ja.jvp_attn_scatter(*grp, mask, o, do, lse, h0=r * Hl)
    ja.check_device_error()
    Ls = L // P
    for s in range(P):
        assert torch.equal(o[s], ref[0][:, :, s * Ls:(s + 1) * Ls]), s
        assert torch.equal(do[s], ref[1][:, :, s * Ls:(s + 1) * Ls]), s
        assert torch.equal(lse[s], ref[2][:, :, s * Ls:(s + 1) * Ls]), s
    # The shards put back in token order, against the oracle on every row
    # (shard and tile boundaries included): the scatter arithmetic of shard
    # r = n // (L/P), row n % (L/P), head h0 + h is checked independently
    # of the plain kernel.
    full = [torch.cat(x, dim=2) for x in (o, do, lse)]
    assert oracle_mismatch(*full, xs, w) == []


def test_scatter_writes_only_its_head_group():
    w = Workload("scatter_one", 1, 4, 128, ja.TEACHER_FORCING, 100, 3, 1, "bf16", 0.1)
    xs, _ = make_inputs(w, device="cuda")
    mask = ja.Mask(w.mode, w.tokens_per_frame, w.n_frames, w.chunk)
    B, Ht, L, d = xs[0].shape
    P = 2
    o, do, lse = _shards(B, Ht, L, d, P, 7.0)
    grp = [x[:, 1:3].contiguous() for x in xs]  # heads 1 and 2 only
    ja.jvp_attn_scatter(*grp, mask, o, do, lse, h0=1)
    ja.check_device_error()
    ref = ja.jvp_attn(*xs, mask)
    Ls = L // P
    for s in range(P):
        for h in range(Ht):
            sl = slice(s * Ls, (s + 1) * Ls)
            if h in (1, 2):
                assert torch.equal(o[s][:, h], ref[0][:, h, sl])
                assert torch.equal(lse[s][:, h], ref[2][:, h, sl])
            else:  # untouched
                assert bool((o[s][:, h] == 7.0).all()) and bool((do[s][:, h] == 7.0).all())
                assert bool((lse[s][:, h] == 7.0).all())


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _fused_worker(rank, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK="0", WORLD_SIZE="1")
    import datetime

    import torch.distributed as dist

    from attention_jvp_continuous_b200.ulysses import (ShardBuffers, ulysses_jvp_attn,
                                                       ulysses_jvp_attn_fused)
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        w = Workload("fused", 1, 2, 128, ja.TEACHER_FORCING, 96, 5, 1, "bf16", 0.1)
        xs, _ = make_inputs(w, device="cuda")
        mask = ja.Mask(w.mode, w.tokens_per_frame, w.n_frames, w.chunk)
        B, H, L, d = xs[0].shape
        bufs = ShardBuffers(B, H, L, d, device="cuda")
        o1, do1, l1 = ulysses_jvp_attn_fused(*xs, mask, bufs)
        o2, do2, l2 = ulysses_jvp_attn(*xs, mask)
        ja.check_device_error()
        out[0] = bool(torch.equal(o1, o2) and torch.equal(do1, do2) and torch.equal(l1, l2))
        out[1] = oracle_mismatch(o1, do1, l1, xs, w)
    finally:
        dist.destroy_process_group()


def test_fused_ulysses_world_one_equals_all_to_all_path():
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_fused_worker, args=(_free_port(), out), nprocs=1, start_method="spawn",
                       join=True)
    assert out[0] is True
    assert list(out[1]) == []
