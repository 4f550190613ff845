"""Float64 CPU oracle for KV-cache chunk attention and key rotation.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py): never imported by the
product package; shares no code with the CUDA path.

Causal rollout and inference (Causal-rCM report, Sec. 3.2.1 "KV Cache")
keep the keys and values of committed chunks in a cache. A read-only
forward generates the current chunk while attending to the committed
prefix the chunk needs; an append commits a chunk's keys and values. With
noisy context (Sec. 3.1.3) the committed entries are those of the last
denoising forward instead of a separate clean pass. Keys may be cached
after rotary position embedding (RoPE) or before it, in which case they
are rotated when read (Sec. 3.2.1, pre- and post-RoPE key caching).

Readings (the pages give no formulas here):
  * the current chunk's queries attend to every key of the exposed cache
    prefix, their own chunk's keys included (placed at the chunk's cache
    position): plain softmax attention over the first Lk cache rows;
  * RoPE rotates consecutive pairs (x_2i, x_2i+1) of a row by the angle of
    its position: (x_2i c - x_2i+1 s, x_2i s + x_2i+1 c) with c, s from
    caller-supplied tables cos[p, i], sin[p, i].
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np

from .jvp_attention import _as64


def rope_rows(x, cos, sin):
    """Rotates every row r of x ([..., R, d]) by table row r of cos / sin
    ([R, d/2]): pairs (x[2i], x[2i+1]) -> (x0 c - x1 s, x0 s + x1 c)."""
    x = _as64(x)
    c, s = _as64(cos), _as64(sin)
    if x.shape[-1] % 2 or c.shape != (x.shape[-2], x.shape[-1] // 2) or s.shape != c.shape:
        raise ValueError("tables must be [rows, d/2] for rows x d inputs with even d")
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


def cache_attention_head(q, k_cache, v_cache, n_keys: int, scale: Optional[float] = None):
    """Attention of the Lq query rows q [Lq, d] over the first n_keys rows of
    k_cache / v_cache [Lcache, d]. Returns float64 (o [Lq, d], lse [Lq])."""
    q = _as64(q)
    k = _as64(k_cache)[:n_keys]
    v = _as64(v_cache)[:n_keys]
    if n_keys < 1 or k.shape[0] != n_keys:
        raise ValueError("need 1 <= n_keys <= cache rows")
    c = 1.0 / math.sqrt(q.shape[1]) if scale is None else float(scale)
    s = c * (q @ k.T)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    ell = e.sum(axis=1, keepdims=True)
    o = (e / ell) @ v
    lse = (m + np.log(ell))[:, 0]
    return o, lse


def cache_attention(q, k_cache, v_cache, n_keys: int, scale: Optional[float] = None):
    """Over [B, H, Lq, d] queries and [B, H, Lcache, d] caches: float64
    (o [B, H, Lq, d], lse [B, H, Lq])."""
    B, H, Lq, d = q.shape
    o = np.zeros((B, H, Lq, d))
    lse = np.zeros((B, H, Lq))
    for b in range(B):
        for h in range(H):
            o[b, h], lse[b, h] = cache_attention_head(q[b, h], k_cache[b, h], v_cache[b, h],
                                                      n_keys, scale)
    return o, lse
