"""Ulysses-style context parallelism around the masked attention JVP.

The pages shard the flattened video-token sequence across P ranks and,
around attention, switch to a head shard with one all-to-all and back with
another (Causal-rCM report, Sec. 3.2.1 "Parallelisms"); for the JVP the
tangents travel with their primals and the local attention is the JVP
kernel (Sec. 3.2.2 "JVP Ulysses CP"):

  in:   Q, K, V, dQ, dK, dV  [B, H, L/P, d] on every rank (token shard r =
        tokens [r L/P, (r+1) L/P))  --all-to-all-->  [B, H/P, L, d]
        (head group r = heads [r H/P, (r+1) H/P), all tokens)
  local: O, dO, LSE = jvp_attn(...) under the full-sequence mask
  out:  O, dO [B, H/P, L, d], LSE [B, H/P, L]  --all-to-all-->  token shards

The exchanges use torch.distributed.all_to_all_single (NCCL over
NVLink/NVSwitch on GPUs); the six inputs go in one collective, the two
outputs in a second and LSE in a third (it is float32). The local
attention is the CUDA kernel; ``attn`` exists so that the data movement can
be tested with CPU process groups. ``ulysses_jvp_attn_fused`` replaces the
output all-to-alls with the kernel's scatter epilogue, which stores every
row into the owning rank's shard in symmetric memory.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence

import torch
import torch.distributed as dist


def _world(group) -> int:
    return dist.get_world_size(group)


def seq_to_head(xs: Sequence[torch.Tensor], group=None) -> torch.Tensor:
    """Token shards [B, H, L/P, d] of n tensors (one dtype) -> this rank's
    head group of all tokens, [n, B, H/P, L, d]."""
    P = _world(group)
    n = len(xs)
    B, H, Ls, d = xs[0].shape
    if H % P:
        raise ValueError(f"{H} heads do not split over {P} ranks")
    send = torch.stack(list(xs)).reshape(n, B, P, H // P, Ls, d)
    send = send.permute(2, 0, 1, 3, 4, 5).contiguous()  # [P (destination), n, B, H/P, Ls, d]
    recv = torch.empty_like(send)                        # [P (source token shard), ...]
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 2, 3, 0, 4, 5).reshape(n, B, H // P, P * Ls, d)


def head_to_seq(ys: Sequence[torch.Tensor], group=None) -> torch.Tensor:
    """Head groups [B, H/P, L, d] of n tensors (one dtype) -> this rank's
    token shard with all heads, [n, B, H, L/P, d]."""
    P = _world(group)
    n = len(ys)
    B, Hp, L, d = ys[0].shape
    if L % P:
        raise ValueError(f"{L} tokens do not split over {P} ranks")
    send = torch.stack(list(ys)).reshape(n, B, Hp, P, L // P, d)
    send = send.permute(3, 0, 1, 2, 4, 5).contiguous()  # [P (destination token shard), ...]
    recv = torch.empty_like(send)                        # [P (source head group), ...]
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 2, 0, 3, 4, 5).reshape(n, B, P * Hp, L // P, d)


def ulysses_jvp_attn(q, k, v, dq, dk, dv, mask, group=None,
                     attn: Optional[Callable] = None):
    """Context-parallel masked attention JVP. q .. dv: this rank's token shard
    [B, H, L/P, d] of the full [B, H, L, d] problem (contiguous token ranges,
    rank order); mask: the full-sequence mask. Returns this rank's token
    shard of (o, do, lse): [B, H, L/P, d], [B, H, L/P, d], [B, H, L/P]."""
    if attn is None:
        from . import jvp_attn as attn
    x = seq_to_head((q, k, v, dq, dk, dv), group)
    o, do, lse = attn(*(x[i] for i in range(6)), mask)
    od = head_to_seq((o, do), group)
    l_sh = head_to_seq((lse.unsqueeze(-1),), group)[0, ..., 0]
    return od[0], od[1], l_sh


class ShardBuffers:
    """Output token shards of a fused Ulysses JVP, allocated in symmetric
    memory so that every rank can store into every other rank's shard:
    o, do [B, H, L/P, d] bf16 and lse [B, H, L/P] float32 on each rank.
    ``peers_*[r]`` are this process's views of rank r's buffers (its own for
    r == rank); ``o``, ``do``, ``lse`` are this rank's own."""

    def __init__(self, B: int, H: int, L: int, d: int, device, group=None):
        import torch
        import torch.distributed._symmetric_memory as symm_mem
        P = _world(group)
        if L % P:
            raise ValueError(f"{L} tokens do not split over {P} ranks")
        self.rank = dist.get_rank(group)
        self.world = P
        shapes = ((B, H, L // P, d), (B, H, L // P, d), (B, H, L // P))
        dtypes = (torch.bfloat16, torch.bfloat16, torch.float32)
        self._own = []
        self._handles = []
        self.peers_o, self.peers_do, self.peers_lse = [], [], []
        for shape, dtype, peers in zip(shapes, dtypes,
                                       (self.peers_o, self.peers_do, self.peers_lse)):
            t = symm_mem.empty(*shape, dtype=dtype, device=device)
            h = symm_mem.rendezvous(t, group if group is not None else dist.group.WORLD)
            self._own.append(t)
            self._handles.append(h)
            for r in range(P):
                peers.append(t if r == self.rank else h.get_buffer(r, shape, dtype))
        self.o, self.do, self.lse = self._own


def ulysses_jvp_attn_fused(q, k, v, dq, dk, dv, mask, bufs: ShardBuffers, group=None):
    """Context-parallel masked attention JVP whose output exchange is fused
    into the kernel's epilogue: after the input all-to-all, this rank's
    kernel stores each O, dO, LSE row of its head group straight into the
    owning rank's shard (plain stores over NVLink into symmetric memory)
    instead of a second and third all-to-all. q .. dv: this rank's token
    shard [B, H, L/P, d] (bf16, d = 128). Returns this rank's (o, do, lse)
    shard, the views ``bufs.o, bufs.do, bufs.lse``; they stay valid until
    the next call with the same buffers."""
    import torch
    from . import jvp_attn_scatter
    P = _world(group)
    rank = dist.get_rank(group)
    B, H, Ls, d = q.shape
    x = seq_to_head((q, k, v, dq, dk, dv), group)
    # Every rank has finished reading its previous outputs before any rank
    # stores the new ones into it.
    dist.barrier(group=group)
    jvp_attn_scatter(*(x[i] for i in range(6)), mask, bufs.peers_o, bufs.peers_do,
                     bufs.peers_lse, h0=rank * (H // P))
    # Each shard is complete once every rank's kernel has finished.
    torch.cuda.current_stream(q.device).synchronize()
    dist.barrier(group=group)
    return bufs.o, bufs.do, bufs.lse
