"""Float64 CPU oracle for the backward pass of masked softmax attention.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py): never imported by the
product package; shares no code with the CUDA path.

The consistency-model loss of the Causal-rCM report is differentiated
through the primal attention output only: the JVP is taken at the
stop-gradient parameters (report, Appendix A, discussion around Eq. 26-28),
so a training step needs, next to the forward JVP, the ordinary gradient of
O = softmax(c QK^T + M) V (Eq. 42) under the same temporal mask.

Given the cotangent G = dL/dO, for every query row i with admissible keys
A_i (masked keys take no part, as in the forward):

  p_ij  = softmax over j in A_i of c <q_i, k_j>
  gV_j  = sum_i p_ij g_i
  dp_ij = <g_i, v_j>
  ds_ij = p_ij (dp_ij - sum_j' p_ij' dp_ij')
  gQ_i  = c sum_j ds_ij k_j
  gK_j  = c sum_i ds_ij q_i

This is the chain rule for L = sum_i <g_i, o_i> written out; it needs no
saved O or LSE (a kernel may use them, the definition does not). Rows that
share an admissible key set are evaluated together with whole-row float64
softmax; no blocking beyond that.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

from .jvp_attention import _as64, _group_rows
from .masks import MaskSpec


def attention_backward_head(q, k, v, g, spec: MaskSpec, scale: Optional[float] = None,
                            row_block: int = 128, rows: Optional[Sequence[int]] = None):
    """Gradients (gq, gk, gv) of sum <g, O> for one (batch, head) slice.

    q, k, v, g: [L, d]. Returns float64 arrays [L, d] each. Every query row
    contributes to gk and gv, so by default all rows are evaluated. With
    ``rows``, only those query rows contribute: gq is exact on them and zero
    elsewhere, gk and gv are the sums of their contributions (the loss
    restricted to those rows of O). Used to time a bounded sample.
    """
    q, k, v, g = (_as64(t) for t in (q, k, v, g))
    L, d = q.shape
    if spec.length != L:
        raise ValueError(f"mask describes {spec.length} tokens, tensors hold {L}")
    c = 1.0 / math.sqrt(d) if scale is None else float(scale)
    gq = np.zeros((L, d))
    gk = np.zeros((L, d))
    gv = np.zeros((L, d))
    for ivs, grp in _group_rows(spec, range(L) if rows is None else rows).items():
        if not ivs:
            continue
        grp = np.asarray(grp)
        for s0 in range(0, len(grp), row_block):
            rr = grp[s0:s0 + row_block]
            Q, G = q[rr], g[rr]
            s = [c * (Q @ k[a:b].T) for a, b in ivs]
            m = np.max([x.max(axis=1) for x in s], axis=0)[:, None]
            e = [np.exp(x - m) for x in s]
            ell = sum(x.sum(axis=1, keepdims=True) for x in e)
            p = [x / ell for x in e]
            dp = [G @ v[a:b].T for a, b in ivs]
            rowdot = sum((pi * dpi).sum(axis=1, keepdims=True) for pi, dpi in zip(p, dp))
            for (a, b), pi, dpi in zip(ivs, p, dp):
                ds = pi * (dpi - rowdot)
                gv[a:b] += pi.T @ G
                gk[a:b] += c * (ds.T @ Q)
                gq[rr] += c * (ds @ k[a:b])
    return gq, gk, gv


def attention_backward(q, k, v, g, spec: MaskSpec, scale: Optional[float] = None,
                       rows: Optional[Sequence[int]] = None):
    """Oracle over [B, H, L, d] inputs: float64 (gq, gk, gv), each [B, H, L, d].
    ``rows`` as in attention_backward_head, for every (batch, head)."""
    B, H, L, d = q.shape
    out = [np.zeros((B, H, L, d)) for _ in range(3)]
    for b in range(B):
        for h in range(H):
            res = attention_backward_head(q[b, h], k[b, h], v[b, h], g[b, h], spec, scale,
                                          rows=rows)
            for o, r in zip(out, res):
                o[b, h] = r
    return tuple(out)
