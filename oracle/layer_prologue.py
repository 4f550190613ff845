"""Float64 CPU oracle for the tangent prologue of an attention layer.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py): never imported by the
product package; shares no code with the CUDA path.

The JVP is taken layer by layer: every layer exposes a paired
primal-tangent interface, (x, dx) in, (y, dy) out (Causal-rCM report,
Sec. 3.2.2 "JVP FSDP2"). Around attention the layer computes, for every
token, the fused projection [q | k | v] = x W (the weights are the
stop-gradient parameters, so the tangent is dx W), an RMS normalisation of
q and k (QK-norm) and rotary position embedding, then hands q, k, v and
their tangents to the attention JVP. Given the projections of x and dx this
module computes that hand-off:

  rms(a)   = sqrt(mean over the norm group of a^2 + eps)
  y        = a / rms(a) * w                     (w: norm weights)
  dy       = w / rms(a) * (da - a * <a, da>_group / (n * rms(a)^2))
  rope(y)  on pairs (y_2i, y_2i+1) of each head, tables of the token's row
  q, dq    = rope(y_q), rope(dy_q); k, dk likewise; v, dv unchanged

(dy is the derivative of y along da; RoPE is linear, so the tangent is
rotated like the primal.) Readings: the norm group is either all H*d
channels of a token or each head's d channels; the projections are laid
out [B, L, 3, H, d] (q, k, v blocks of H*d channels, head-major inside);
outputs are [B, H, L, d], the attention JVP's input layout.
"""
from __future__ import annotations

from typing import Optional

import numpy as np

from .jvp_attention import _as64
from .kv_cache import rope_rows


def rms_norm_jvp(a, da, w, group: int, eps: float):
    """RMS norm of a [..., C] over consecutive groups of `group` channels with
    weights w [group] (or [C]) and its derivative along da: float64 (y, dy)."""
    a, da = _as64(a), _as64(da)
    C = a.shape[-1]
    if C % group:
        raise ValueError("the channel count must be a multiple of the norm group")
    w = _as64(w)
    g = a.reshape(*a.shape[:-1], C // group, group)
    dg = da.reshape(g.shape)
    ms = (g * g).mean(axis=-1, keepdims=True) + eps
    r = 1.0 / np.sqrt(ms)
    dot = (g * dg).mean(axis=-1, keepdims=True)
    y = g * r
    dy = r * (dg - g * dot / ms)
    y = y.reshape(a.shape)
    dy = dy.reshape(a.shape)
    wb = np.tile(w, C // w.shape[0]) if w.shape[0] != C else w
    return y * wb, dy * wb


def qkv_prologue(qkv, d_qkv, H: int, d: int, norm_q=None, norm_k=None, norm_group: int = 0,
                 eps: float = 1e-6, cos=None, sin=None):
    """qkv, d_qkv: [B, L, 3*H*d] projections of x and dx. norm_q / norm_k:
    weights (None: no QK-norm); norm_group: H*d or d. cos / sin: [L, d/2]
    rotation tables (None: no rotation). Returns float64 (q, k, v, dq, dk,
    dv), each [B, H, L, d]."""
    P, dP = _as64(qkv), _as64(d_qkv)
    B, L, C3 = P.shape
    C = H * d
    if C3 != 3 * C:
        raise ValueError("projections must hold 3 * H * d channels")
    parts = []
    for blk, w in ((0, norm_q), (1, norm_k), (2, None)):
        a = P[:, :, blk * C:(blk + 1) * C]
        da = dP[:, :, blk * C:(blk + 1) * C]
        if w is not None:
            a, da = rms_norm_jvp(a, da, w, norm_group, eps)
        a = a.reshape(B, L, H, d).transpose(0, 2, 1, 3)
        da = da.reshape(B, L, H, d).transpose(0, 2, 1, 3)
        if blk < 2 and cos is not None:
            a, da = rope_rows(a, cos, sin), rope_rows(da, cos, sin)
        parts.append((np.ascontiguousarray(a), np.ascontiguousarray(da)))
    (q, dq), (k, dk), (v, dv) = parts
    return q, k, v, dq, dk, dv
