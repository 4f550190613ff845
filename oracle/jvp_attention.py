"""Float64 CPU oracle for the masked attention JVP.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls or
links this module: it is used by ``tests/``, by ``__graft_entry__.smoke()``
and by the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``.
It shares no code with the CUDA path.

What it computes (Causal-rCM tech report, Appendix B "FlashAttention-2 JVP
Kernel with Custom Masks", Eq. 42-44), for every query row i and its set
A_i of admissible keys:

  s_j   = c * <q_i, k_j>                               (Eq. 42, scores)
  ds_j  = c * (<dq_i, k_j> + <q_i, dk_j>)              (Eq. 43, score tangent)
  p     = softmax over j in A_i of s_j                 (Eq. 42)
  o_i   = sum_j p_j v_j                                (Eq. 42)
  mu_i  = sum_j p_j ds_j
  do_i  = sum_j p_j (ds_j - mu_i) v_j + sum_j p_j dv_j (Eq. 44)
  lse_i = log sum_j exp(s_j)

with c = 1/sqrt(d) unless a scale is given. Masked keys take no part in
any sum: the mask is a fixed routing object with no tangent (Appendix B,
text after Eq. 43). The score tangent uses the same scale c as the score,
the plainest reading of Eq. 43 when its body is missing from the page.

This is the direct dense definition, not the online (streamed) softmax
that a kernel uses: each group of rows that share one admissible key set
is evaluated with whole-row softmax in float64. Rows are processed in
blocks so that no L x L matrix is formed.

Parity pins: the test suite checks this module against torch autodiff of
scaled-dot-product attention, central finite differences, closed-form
pair counts, invariants and brute force (see tests/test_oracle.py).
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

from .masks import MaskSpec, key_intervals

Array = np.ndarray


def _as64(x) -> Array:
    """Exact float64 copy of a numpy array or a (CPU) torch tensor."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def _group_rows(spec: MaskSpec, rows: Sequence[int]):
    """Group query rows by identical admissible key-interval lists."""
    groups: Dict[Tuple[Tuple[int, int], ...], List[int]] = {}
    for r in rows:
        iv = tuple(key_intervals(spec, int(r)))
        groups.setdefault(iv, []).append(int(r))
    return groups


def jvp_attention_head(q, k, v, dq, dk, dv, spec: MaskSpec,
                       scale: Optional[float] = None,
                       rows: Optional[Sequence[int]] = None,
                       row_block: int = 128):
    """Oracle for one (batch, head) slice.

    q, k, v, dq, dk, dv: [L, d] arrays (any float dtype; read exactly and
    upcast to float64). ``rows`` selects query rows (default: all).
    Returns (o, do, lse) as float64 arrays of shapes [n, d], [n, d], [n]
    for the selected rows, in the order given.

    A row with no admissible key gets o = do = 0 and lse = -inf (a
    convention: no descriptor of the four modes produces such a row).
    """
    q, k, v, dq, dk, dv = (_as64(t) for t in (q, k, v, dq, dk, dv))
    L, d = q.shape
    if spec.length != L:
        raise ValueError(f"mask describes {spec.length} tokens, tensors hold {L}")
    c = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rows = np.arange(L) if rows is None else np.asarray(rows, dtype=np.int64)
    pos = {int(r): n for n, r in enumerate(rows)}
    o = np.zeros((len(rows), d))
    do = np.zeros((len(rows), d))
    lse = np.full((len(rows),), -np.inf)

    for ivs, grp in _group_rows(spec, rows).items():
        if not ivs:
            continue
        # The admissible keys are the union of the intervals; each interval
        # is a contiguous slice (a view), and sums over the union are sums
        # of the per-interval sums.
        Ks = [k[a:b] for a, b in ivs]
        Vs = [v[a:b] for a, b in ivs]
        dKs = [dk[a:b] for a, b in ivs]
        dVs = [dv[a:b] for a, b in ivs]
        grp = np.asarray(grp)
        for s0 in range(0, len(grp), row_block):
            rr = grp[s0:s0 + row_block]
            Q, dQ = q[rr], dq[rr]
            s = [c * (Q @ K.T) for K in Ks]                    # Eq. 42
            ds = [c * (dQ @ K.T + Q @ dK.T) for K, dK in zip(Ks, dKs)]  # Eq. 43
            m = np.max([x.max(axis=1) for x in s], axis=0)[:, None]
            e = [np.exp(x - m) for x in s]
            ell = sum(x.sum(axis=1, keepdims=True) for x in e)
            p = [x / ell for x in e]                           # masked softmax
            out_o = sum(pi @ V for pi, V in zip(p, Vs))
            mu = sum((pi * dsi).sum(axis=1, keepdims=True) for pi, dsi in zip(p, ds))
            out_do = sum((pi * (dsi - mu)) @ V + pi @ dV       # Eq. 44
                         for pi, dsi, V, dV in zip(p, ds, Vs, dVs))
            idx = [pos[int(r)] for r in rr]
            o[idx] = out_o
            do[idx] = out_do
            lse[idx] = (m + np.log(ell))[:, 0]
    return o, do, lse


def jvp_attention(q, k, v, dq, dk, dv, spec: MaskSpec,
                  scale: Optional[float] = None,
                  rows: Optional[Sequence[int]] = None):
    """Oracle over [B, H, L, d] inputs.

    Returns float64 (o, do, lse) of shapes [B, H, n, d], [B, H, n, d],
    [B, H, n], where n = L or len(rows).
    """
    B, H, L, d = q.shape
    n = L if rows is None else len(rows)
    o = np.zeros((B, H, n, d))
    do = np.zeros((B, H, n, d))
    lse = np.zeros((B, H, n))
    for b in range(B):
        for h in range(H):
            o[b, h], do[b, h], lse[b, h] = jvp_attention_head(
                q[b, h], k[b, h], v[b, h], dq[b, h], dk[b, h], dv[b, h],
                spec, scale=scale, rows=rows)
    return o, do, lse
