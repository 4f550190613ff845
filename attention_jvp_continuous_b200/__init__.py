"""B200-native masked attention JVP (Causal-rCM report, Appendix B).

``jvp_attn(q, k, v, dq, dk, dv, mask)`` returns (O, dO, LSE) for softmax
attention under a temporal mask and its forward-mode tangent along
(dQ, dK, dV), computed by the CUDA kernels of ``libjvpattn.so``. PyTorch is
used for device memory and streams only.
"""
from __future__ import annotations

import ctypes
import dataclasses
from typing import Optional, Tuple

from . import _lib
from ._lib import JvpAttnError, MaskDesc

DENSE = 0
FRAME_CAUSAL = 1
CHUNK_CAUSAL = 2
TEACHER_FORCING = 3

__all__ = ["Mask", "jvp_attn", "jvp_attn_fwd", "jvp_attn_scatter", "signal_barrier", "attn_bwd",
           "jvp_attn_bwd", "bwd_scratch_len", "cache_attn", "rope_copy", "qkv_prologue", "mask_stats", "tile_classes",
           "schedule", "schedule_kv", "check_device_error", "set_wait_limit", "set_stall_test", "release",
           "JvpAttnError",
           "DENSE", "FRAME_CAUSAL", "CHUNK_CAUSAL", "TEACHER_FORCING"]


@dataclasses.dataclass(frozen=True)
class Mask:
    """Temporal mask descriptor {mode, tokens_per_frame, n_frames, chunk}."""
    mode: int
    tokens_per_frame: int
    n_frames: int
    chunk: int = 1

    def desc(self) -> MaskDesc:
        return MaskDesc(self.mode, self.tokens_per_frame, self.n_frames, self.chunk)

    @property
    def length(self) -> int:
        ft = self.tokens_per_frame * self.n_frames
        return 2 * ft if self.mode == TEACHER_FORCING else ft


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return _lib.JVP_BF16
    if t.dtype == torch.float32:
        return _lib.JVP_FP32
    raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16 or float32")


def jvp_attn_fwd(q, k, v, dq, dk, dv, o, d_o, lse, mask: Mask,
                 scale: Optional[float] = None, stream: Optional[int] = None) -> None:
    """Raw call of the C ABI on caller-allocated device tensors (no checks
    beyond those the library makes). ``stream`` is a cudaStream_t as int;
    default: the current torch stream of q's device."""
    import torch
    B, H, L, d = q.shape
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    rc = _lib.lib().jvp_attn_fwd(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), dq.data_ptr(), dk.data_ptr(),
        dv.data_ptr(), o.data_ptr(), d_o.data_ptr(),
        ctypes.cast(lse.data_ptr(), ctypes.POINTER(ctypes.c_float)),
        B, H, L, d, _dtype_code(q), mask.desc(),
        0.0 if scale is None else float(scale), ctypes.c_void_p(stream))
    _lib.check(rc, "jvp_attn_fwd")


def jvp_attn_scatter(q, k, v, dq, dk, dv, mask: Mask, o_dst, do_dst, lse_dst, h0: int,
                     scale: Optional[float] = None) -> None:
    """Masked attention JVP of this rank's head group whose epilogue writes
    every output row into the token shard that owns it (the output exchange
    of Ulysses context parallelism, fused into the kernel).

    q, k, v, dq, dk, dv: CUDA bf16 [B, H, L, d] (d = 128), the head group
    h0 .. h0 + H - 1 of all L tokens. o_dst, do_dst: sequences of P bf16
    tensors [B, H_total, L/P, d]; lse_dst: P float32 tensors [B, H_total,
    L/P]. Entry r may be a view of another GPU's memory (a symmetric-memory
    buffer); row n goes to entry n // (L/P). Rows of heads outside this
    group are not written. Enqueued on the current stream; peers see the
    rows after this launch completes and the ranks synchronise.
    """
    import torch
    ts = (q, k, v, dq, dk, dv)
    for t in ts:
        if not t.is_cuda or t.dtype != torch.bfloat16 or t.shape != q.shape or not t.is_contiguous():
            raise ValueError("q, k, v, dq, dk, dv must be contiguous CUDA bf16 [B, H, L, d]")
    B, H, L, d = q.shape
    P = len(o_dst)
    if not (len(do_dst) == P == len(lse_dst)) or P < 1:
        raise ValueError("o_dst, do_dst and lse_dst must list the same number of shards")
    if L % P:
        raise ValueError(f"{L} tokens do not split over {P} shards")
    Ht = o_dst[0].shape[1]
    for o_, do_, l_ in zip(o_dst, do_dst, lse_dst):
        if (o_.shape != (B, Ht, L // P, d) or do_.shape != o_.shape or o_.dtype != torch.bfloat16
                or do_.dtype != torch.bfloat16 or not o_.is_contiguous() or not do_.is_contiguous()):
            raise ValueError("o_dst / do_dst entries must be contiguous bf16 [B, H_total, L/P, d]")
        if l_.shape != (B, Ht, L // P) or l_.dtype != torch.float32 or not l_.is_contiguous():
            raise ValueError("lse_dst entries must be contiguous float32 [B, H_total, L/P]")
    arr = lambda ts_: (ctypes.c_void_p * P)(*[t.data_ptr() for t in ts_])
    stream = torch.cuda.current_stream(q.device).cuda_stream
    rc = _lib.lib().jvp_attn_fwd_scatter(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
        arr(o_dst), arr(do_dst), arr(lse_dst), P, int(h0), Ht,
        B, H, L, d, _dtype_code(q), mask.desc(),
        0.0 if scale is None else float(scale), ctypes.c_void_p(stream))
    _lib.check(rc, "jvp_attn_fwd_scatter")


def signal_barrier(flags, rank: int, epoch: int, stream: Optional[int] = None) -> None:
    """Device-side barrier of the ranks of a context-parallel group on the
    current stream (jvp_attn_signal_barrier). flags: one int32 CUDA tensor
    view per rank of that rank's n_ranks flag words (this process's address
    of it), zero before the first barrier; epoch: 1, 2, ... per barrier."""
    import torch
    n = len(flags)
    for t in flags:
        if not t.is_cuda or t.dtype != torch.int32 or t.numel() < n:
            raise ValueError("flags must be int32 CUDA tensors of at least n_ranks words")
    if stream is None:
        stream = torch.cuda.current_stream(flags[0].device).cuda_stream
    arr = (ctypes.c_void_p * n)(*[t.data_ptr() for t in flags])
    rc = _lib.lib().jvp_attn_signal_barrier(arr, n, int(rank), ctypes.c_uint32(epoch & 0xFFFFFFFF),
                                            ctypes.c_void_p(stream))
    _lib.check(rc, "jvp_attn_signal_barrier")


def jvp_attn(q, k, v, dq, dk, dv, mask: Mask, scale: Optional[float] = None,
             out: Optional[Tuple] = None):
    """O, dO, LSE of masked attention and its JVP.

    q, k, v, dq, dk, dv: CUDA tensors [B, H, L, d], all bfloat16 or all
    float32, contiguous. Returns (o, do, lse) with o, do like q and lse
    float32 [B, H, L]. ``out`` may supply preallocated (o, do, lse).
    """
    import torch
    ts = (q, k, v, dq, dk, dv)
    for t in ts:
        if not t.is_cuda:
            raise ValueError("jvp_attn expects CUDA tensors")
        if t.shape != q.shape or t.dtype != q.dtype or t.device != q.device:
            raise ValueError("q, k, v, dq, dk, dv must share shape, dtype and device")
        if not t.is_contiguous():
            raise ValueError("inputs must be contiguous [B, H, L, d]")
    if q.dim() != 4:
        raise ValueError("inputs must be [B, H, L, d]")
    B, H, L, d = q.shape
    if out is None:
        o = torch.empty_like(q)
        d_o = torch.empty_like(q)
        lse = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    else:
        o, d_o, lse = out
    jvp_attn_fwd(q, k, v, dq, dk, dv, o, d_o, lse, mask, scale)
    return o, d_o, lse


def bwd_scratch_len(B: int, H: int, L: int) -> int:
    """float32 elements of scratch jvp_attn_bwd needs (jvp_attn_bwd_scratch_len)."""
    n = _lib.lib().jvp_attn_bwd_scratch_len(B, H, L)
    if n < 0:
        raise ValueError("invalid shape for jvp_attn_bwd")
    return int(n)


def jvp_attn_bwd(q, k, v, o, g, lse, gq, gk, gv, scratch, mask: Mask,
                 scale: Optional[float] = None, stream: Optional[int] = None) -> None:
    """Into preallocated outputs: (gq, gk, gv) = gradients of sum <g, o> for
    o = masked attention of (q, k, v). bf16 CUDA tensors [B, H, L, 128]; o and
    lse as returned by jvp_attn; scratch a float32 CUDA tensor of at least
    bwd_scratch_len(B, H, L) elements. Allocates nothing."""
    import torch
    for t in (q, k, v, o, g, gq, gk, gv):
        if not t.is_cuda or t.shape != q.shape or t.dtype != q.dtype or not t.is_contiguous():
            raise ValueError("q, k, v, o, g, gq, gk, gv must be contiguous CUDA tensors of "
                             "one shape and dtype")
    for t, name in ((lse, "lse"), (scratch, "scratch")):
        if not t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous float32 CUDA tensor")
    B, H, L, d = q.shape
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    fp = ctypes.POINTER(ctypes.c_float)
    rc = _lib.lib().jvp_attn_bwd(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), g.data_ptr(),
        ctypes.cast(lse.data_ptr(), fp), gq.data_ptr(), gk.data_ptr(), gv.data_ptr(),
        ctypes.cast(scratch.data_ptr(), fp), scratch.numel(), B, H, L, d, _dtype_code(q),
        mask.desc(), 0.0 if scale is None else float(scale), ctypes.c_void_p(stream))
    _lib.check(rc, "jvp_attn_bwd")


def attn_bwd(q, k, v, o, g, lse, mask: Mask, scale: Optional[float] = None,
             stream: Optional[int] = None):
    """Gradients (g_q, g_k, g_v) of sum <g, o> for o = masked attention of
    (q, k, v); o and lse as returned by jvp_attn. bf16 CUDA tensors, d = 128.
    Allocates the outputs and the scratch, then calls jvp_attn_bwd."""
    import torch
    B, H, L, d = q.shape
    gq, gk, gv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    scratch = torch.empty((bwd_scratch_len(B, H, L),), dtype=torch.float32, device=q.device)
    jvp_attn_bwd(q, k, v, o, g, lse, gq, gk, gv, scratch, mask, scale, stream)
    return gq, gk, gv


def cache_attn(q, k_cache, v_cache, n_keys: int, o=None, lse=None,
               scale: Optional[float] = None, stream: Optional[int] = None):
    """Chunk attention over a key/value cache (jvp_attn_cache_fwd): the
    queries q [B, H, Lq, 128] attend to rows [0, n_keys) of k_cache, v_cache
    [B, H, Lcache, 128] (bf16, CUDA). Returns (o [B, H, Lq, 128] bf16,
    lse [B, H, Lq] float32), into o / lse when given."""
    import torch
    B, H, Lq, d = q.shape
    for t in (q, k_cache, v_cache):
        if not t.is_cuda or t.dtype != q.dtype or not t.is_contiguous():
            raise ValueError("q, k_cache, v_cache must be contiguous CUDA tensors of one dtype")
    if k_cache.shape != v_cache.shape or k_cache.shape[:2] != (B, H) or k_cache.shape[3] != d:
        raise ValueError("k_cache and v_cache must be [B, H, Lcache, d] matching q")
    Lcache = k_cache.shape[2]
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device)
    if o.shape != q.shape or o.dtype != q.dtype or not o.is_contiguous():
        raise ValueError("o must be a contiguous tensor like q")
    if lse.shape != (B, H, Lq) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 tensor [B, H, Lq]")
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    fp = ctypes.POINTER(ctypes.c_float)
    rc = _lib.lib().jvp_attn_cache_fwd(
        q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), o.data_ptr(),
        ctypes.cast(lse.data_ptr(), fp), B, H, Lq, int(n_keys), Lcache, d, _dtype_code(q),
        0.0 if scale is None else float(scale), ctypes.c_void_p(stream))
    _lib.check(rc, "jvp_attn_cache_fwd")
    return o, lse


def rope_copy(src, dst, rows: int, src_row0: int = 0, dst_row0: int = 0, cos=None, sin=None,
              rope_row0: int = 0, stream: Optional[int] = None) -> None:
    """Copies rows [src_row0, src_row0 + rows) of src [B, H, Ls, d] to rows
    [dst_row0, ...) of dst [B, H, Ld, d] (jvp_attn_rope_copy), rotating row j
    by table row rope_row0 + j of cos / sin (float32 [n, d/2]) when given."""
    import torch
    for t in (src, dst):
        if not t.is_cuda or t.dtype != src.dtype or not t.is_contiguous() or t.dim() != 4:
            raise ValueError("src and dst must be contiguous 4-D CUDA tensors of one dtype")
    B, H, Ls, d = src.shape
    if dst.shape[:2] != (B, H) or dst.shape[3] != d:
        raise ValueError("dst must be [B, H, Ld, d] matching src")
    fp = ctypes.POINTER(ctypes.c_float)
    cp = sp = None
    n_rope = 0
    if (cos is None) != (sin is None):
        raise ValueError("give both cos and sin, or neither")
    if cos is not None:
        for t in (cos, sin):
            if not t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
                raise ValueError("cos / sin must be contiguous float32 CUDA tensors [n, d/2]")
        if cos.shape != sin.shape or cos.dim() != 2 or cos.shape[1] * 2 != d:
            raise ValueError("cos / sin must both be [n, d/2]")
        cp, sp = ctypes.cast(cos.data_ptr(), fp), ctypes.cast(sin.data_ptr(), fp)
        n_rope = cos.shape[0]
    if stream is None:
        stream = torch.cuda.current_stream(src.device).cuda_stream
    rc = _lib.lib().jvp_attn_rope_copy(
        src.data_ptr(), dst.data_ptr(), B, H, Ls, dst.shape[2], int(rows), int(src_row0),
        int(dst_row0), d, _dtype_code(src), cp, sp, n_rope, int(rope_row0),
        ctypes.c_void_p(stream))
    _lib.check(rc, "jvp_attn_rope_copy")


def qkv_prologue(qkv, d_qkv, H: int, norm_q=None, norm_k=None, norm_group: Optional[int] = None,
                 eps: float = 1e-6, cos=None, sin=None, out=None, stream: Optional[int] = None):
    """Attention-layer tangent prologue (jvp_attn_qkv_prologue): from the fused
    projections qkv, d_qkv [B, L, 3*H*d] (bf16, CUDA) of x and its tangent,
    QK-norm (weights norm_q / norm_k, float32 [norm_group]; norm_group H*d or
    d) with its derivative, RoPE by token row (cos / sin float32 [>= L, d/2])
    and the [B, H, L, d] layout. Returns (q, k, v, dq, dk, dv), into `out`
    (six tensors) when given."""
    import torch
    for t in (qkv, d_qkv):
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 3:
            raise ValueError("qkv and d_qkv must be contiguous bf16 CUDA tensors [B, L, 3 H d]")
    if d_qkv.shape != qkv.shape or qkv.shape[2] % (3 * H):
        raise ValueError("qkv and d_qkv must share one shape [B, L, 3 H d]")
    B, L, C3 = qkv.shape
    d = C3 // (3 * H)
    if out is None:
        out = [torch.empty((B, H, L, d), dtype=qkv.dtype, device=qkv.device) for _ in range(6)]
    for t in out:
        if t.shape != (B, H, L, d) or t.dtype != qkv.dtype or not t.is_contiguous() or not t.is_cuda:
            raise ValueError("outputs must be contiguous bf16 CUDA tensors [B, H, L, d]")
    fp = ctypes.POINTER(ctypes.c_float)

    def fptr(t):
        if t is None:
            return None
        if not t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError("norm weights and rotation tables must be contiguous float32 CUDA tensors")
        return ctypes.cast(t.data_ptr(), fp)

    n_rope = 0 if cos is None else cos.shape[0]
    group = (H * d if norm_group is None else int(norm_group)) if norm_q is not None else 0
    if stream is None:
        stream = torch.cuda.current_stream(qkv.device).cuda_stream
    rc = _lib.lib().jvp_attn_qkv_prologue(
        qkv.data_ptr(), d_qkv.data_ptr(), *[t.data_ptr() for t in out], fptr(norm_q),
        fptr(norm_k), group, float(eps), fptr(cos), fptr(sin), n_rope, B, L, H, d,
        _lib.JVP_BF16, ctypes.c_void_p(stream))
    _lib.check(rc, "jvp_attn_qkv_prologue")
    return tuple(out)


def mask_stats(mask: Mask, L: Optional[int] = None, bm: int = 128, bn: int = 64):
    """(pairs, full, partial, empty) for the mask on a bm x bn tile grid."""
    L = mask.length if L is None else L
    vals = [ctypes.c_int64() for _ in range(4)]
    rc = _lib.lib().jvp_attn_mask_stats(mask.desc(), L, bm, bn,
                                         *[ctypes.byref(x) for x in vals])
    _lib.check(rc, "jvp_attn_mask_stats")
    return tuple(x.value for x in vals)


def tile_classes(mask: Mask, L: Optional[int] = None, bm: int = 128, bn: int = 64):
    """numpy int8 [n_qt, n_kt] of tile classes (0 empty, 1 full, 2 partial)."""
    import numpy as np
    L = mask.length if L is None else L
    nq, nk = -(-L // bm), -(-L // bn)
    out = np.zeros((nq, nk), dtype=np.int8)
    rc = _lib.lib().jvp_attn_tile_classes(
        mask.desc(), L, bm, bn, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int8)), out.size)
    _lib.check(rc, "jvp_attn_tile_classes")
    return out


def schedule(mask: Mask, L: Optional[int] = None, bm: int = 128, bn: int = 64):
    """(qtiles [n, 4], segs [m, 3]) int32 arrays of the tensor-core work list."""
    import numpy as np
    L = mask.length if L is None else L
    nq, ns = ctypes.c_int(), ctypes.c_int()
    lib = _lib.lib()
    lib.jvp_attn_schedule(mask.desc(), L, bm, bn, None, 0, None, 0,
                          ctypes.byref(nq), ctypes.byref(ns))
    qt = np.zeros((nq.value, 4), dtype=np.int32)
    sg = np.zeros((ns.value, 3), dtype=np.int32)
    p32 = ctypes.POINTER(ctypes.c_int32)
    rc = lib.jvp_attn_schedule(mask.desc(), L, bm, bn, qt.ctypes.data_as(p32), nq.value,
                               sg.ctypes.data_as(p32), ns.value, ctypes.byref(nq),
                               ctypes.byref(ns))
    _lib.check(rc, "jvp_attn_schedule")
    return qt, sg


def schedule_kv(mask: Mask, L: Optional[int] = None, bq: int = 64, bk: int = 128):
    """(ktiles [n, 4], segs [m, 3]) int32 arrays of the backward key-pass work list."""
    import numpy as np
    L = mask.length if L is None else L
    nk, ns = ctypes.c_int(), ctypes.c_int()
    lib = _lib.lib()
    lib.jvp_attn_schedule_kv(mask.desc(), L, bq, bk, None, 0, None, 0,
                             ctypes.byref(nk), ctypes.byref(ns))
    kt = np.zeros((nk.value, 4), dtype=np.int32)
    sg = np.zeros((ns.value, 3), dtype=np.int32)
    p32 = ctypes.POINTER(ctypes.c_int32)
    rc = lib.jvp_attn_schedule_kv(mask.desc(), L, bq, bk, kt.ctypes.data_as(p32), nk.value,
                                  sg.ctypes.data_as(p32), ns.value, ctypes.byref(nk),
                                  ctypes.byref(ns))
    _lib.check(rc, "jvp_attn_schedule_kv")
    return kt, sg


def check_device_error(stream: Optional[int] = None) -> None:
    """Synchronise ``stream`` and raise if a kernel recorded a device error."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    _lib.check(_lib.lib().jvp_attn_check_device_error(ctypes.c_void_p(stream)),
               "jvp_attn_check_device_error")


def set_wait_limit(ns: int) -> None:
    """Per-wait limit of the tensor-core kernels in ns (0 = default, 2 s)."""
    _lib.check(_lib.lib().jvp_attn_set_wait_limit(int(ns)), "jvp_attn_set_wait_limit")


def set_stall_test(enable: bool) -> None:
    """Failure-detection test switch: while on, every tensor-core launch ends
    through its bounded-wait timeout path (JVP_ERR_DEVICE_TIMEOUT)."""
    _lib.check(_lib.lib().jvp_attn_set_stall_test(1 if enable else 0), "jvp_attn_set_stall_test")


def release() -> None:
    _lib.check(_lib.lib().jvp_attn_release(), "jvp_attn_release")
