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

The exchanges move no data through staging buffers: every message is one
contiguous run of a tensor, the L/P tokens of one (tensor, batch, head),
sent straight from the sender's tensor and received straight into its
place in the receiver's tensor, as one group of point-to-point transfers
(NCCL over NVLink/NVSwitch on GPUs). A rank's own run is one strided copy
per tensor. The local attention is the CUDA kernel; ``attn`` exists so
that the data movement can be tested with CPU process groups.
``ulysses_jvp_attn_fused`` replaces the output exchange with the kernel's
scatter epilogue, which stores every row into the owning rank's shard in
symmetric memory.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence

import torch
import torch.distributed as dist


def _world(group) -> int:
    return dist.get_world_size(group)


def _exchange(sends, recvs, group) -> None:
    """One group of point-to-point transfers. sends / recvs: lists of
    (peer rank in ``group``, contiguous tensor), each list in the order that
    the peer posts the matching other half. Runs on the current stream with
    NCCL (the host does not wait); with gloo the host waits."""
    ops = []
    glob = (lambda r: r) if group is None else (lambda r: dist.get_global_rank(group, r))
    for peer, t in sends:
        ops.append(dist.P2POp(dist.isend, t, glob(peer), group))
    for peer, t in recvs:
        ops.append(dist.P2POp(dist.irecv, t, glob(peer), group))
    if ops:
        for w in dist.batch_isend_irecv(ops):
            w.wait()


def seq_to_head(xs: Sequence[torch.Tensor], group=None) -> torch.Tensor:
    """Token shards [B, H, L/P, ...] of n tensors (one dtype) -> this rank's
    head group of all tokens, [n, B, H/P, L, ...]. Rank r's shard holds
    tokens [r L/P, (r+1) L/P); head group g is heads [g H/P, (g+1) H/P)."""
    P = _world(group)
    me = dist.get_rank(group)
    n = len(xs)
    B, H, Ls = xs[0].shape[:3]
    tail = tuple(xs[0].shape[3:])
    if H % P:
        raise ValueError(f"{H} heads do not split over {P} ranks")
    Hp = H // P
    for x in xs:
        if not x.is_contiguous() or x.shape != xs[0].shape:
            raise ValueError("token shards must be contiguous and of one shape")
    out = torch.empty((n, B, Hp, P * Ls) + tail, dtype=xs[0].dtype, device=xs[0].device)
    mine = slice(me * Ls, (me + 1) * Ls)
    for i, x in enumerate(xs):
        out[i, :, :, mine].copy_(x[:, me * Hp:(me + 1) * Hp])
    sends, recvs = [], []
    for peer in range(P):
        if peer == me:
            continue
        for i, x in enumerate(xs):
            for b in range(B):
                for h in range(Hp):
                    sends.append((peer, x[b, peer * Hp + h]))
                    recvs.append((peer, out[i, b, h, peer * Ls:(peer + 1) * Ls]))
    _exchange(sends, recvs, group)
    return out


def head_to_seq(ys: Sequence[torch.Tensor], group=None) -> torch.Tensor:
    """Head groups [B, H/P, L, ...] of n tensors (one dtype) -> this rank's
    token shard with all heads, [n, B, H, L/P, ...]."""
    P = _world(group)
    me = dist.get_rank(group)
    n = len(ys)
    B, Hp, L = ys[0].shape[:3]
    tail = tuple(ys[0].shape[3:])
    if L % P:
        raise ValueError(f"{L} tokens do not split over {P} ranks")
    Ls = L // P
    for y in ys:
        if not y.is_contiguous() or y.shape != ys[0].shape:
            raise ValueError("head groups must be contiguous and of one shape")
    out = torch.empty((n, B, P * Hp, Ls) + tail, dtype=ys[0].dtype, device=ys[0].device)
    for i, y in enumerate(ys):
        out[i, :, me * Hp:(me + 1) * Hp].copy_(y[:, :, me * Ls:(me + 1) * Ls])
    sends, recvs = [], []
    for peer in range(P):
        if peer == me:
            continue
        for i, y in enumerate(ys):
            for b in range(B):
                for h in range(Hp):
                    sends.append((peer, y[b, h, peer * Ls:(peer + 1) * Ls]))
                    recvs.append((peer, out[i, b, peer * Hp + h]))
    _exchange(sends, recvs, group)
    return out


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
    l_sh = head_to_seq((lse,), group)[0]
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
        # Flag words of the ranks' barrier (jvp_attn_signal_barrier), zeroed
        # on every rank before any rank can use them.
        f = symm_mem.empty(P, dtype=torch.int32, device=device)
        hf = symm_mem.rendezvous(f, group if group is not None else dist.group.WORLD)
        f.zero_()
        torch.cuda.current_stream(f.device).synchronize()
        dist.barrier(group=group)
        self._own.append(f)
        self._handles.append(hf)
        self.flags = [f if r == self.rank else hf.get_buffer(r, (P,), torch.int32)
                      for r in range(P)]
        self.epoch = 0

    def barrier(self) -> None:
        """Device-side barrier of the ranks on the current stream (the
        library's signal barrier): a rank's stream passes it once every
        rank's stream has reached it, so all work enqueued before it on every
        rank is complete. The wait is bounded by the library's wait limit; a
        rank that never arrives is reported as JVP_ERR_DEVICE_TIMEOUT by
        check_device_error instead of hanging."""
        from . import signal_barrier
        self.epoch += 1
        signal_barrier(self.flags, self.rank, self.epoch)


def ulysses_jvp_attn_fused(q, k, v, dq, dk, dv, mask, bufs: ShardBuffers, group=None):
    """Context-parallel masked attention JVP whose output exchange is fused
    into the kernel's epilogue: after the input all-to-all, this rank's
    kernel stores each O, dO, LSE row of its head group straight into the
    owning rank's shard (plain stores over NVLink into symmetric memory)
    instead of a second and third all-to-all. q .. dv: this rank's token
    shard [B, H, L/P, d] (bf16, d = 128). Returns this rank's (o, do, lse)
    shard, the views ``bufs.o, bufs.do, bufs.lse``, complete in stream
    order (work enqueued after this call on the current stream sees them);
    they stay valid until the next call with the same buffers."""
    from . import jvp_attn_scatter
    P = _world(group)
    rank = dist.get_rank(group)
    B, H, Ls, d = q.shape
    x = seq_to_head((q, k, v, dq, dk, dv), group)
    # Stream-ordered device barriers (flag words in symmetric memory, bounded
    # waits): before the launch, every rank's stream has passed its reads
    # of the previous outputs; after it, every rank's kernel has finished
    # storing into every shard. The host never waits.
    bufs.barrier()
    jvp_attn_scatter(*(x[i] for i in range(6)), mask, bufs.peers_o, bufs.peers_do,
                     bufs.peers_lse, h0=rank * (H // P))
    bufs.barrier()
    return bufs.o, bufs.do, bufs.lse
