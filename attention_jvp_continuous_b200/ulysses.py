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
be tested with CPU process groups.
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
