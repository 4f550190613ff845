"""Seeded synthetic workloads for the masked attention JVP.

This module is shared by the tests, the benchmark and the CPU oracle's
callers. It holds workload shapes and random draws only: no attention,
softmax or mask arithmetic lives here.

Workloads follow the Causal-rCM report (Section 4.1, Setup): Wan2.1 at 480p
gives 21 latent frames, and 104x60 latents patchified 2x2 give 52x30 = 1560
tokens per frame (the third-party reading notes on that report, "worked
example of the spatial axis"). The frame-wise (c1-1) and chunk-wise (c3-3)
patterns are the report's two causal settings.

Draw recipe (one generator per workload, seeded once):
  1. Q, K, V, dQ, dK, dV are drawn in that order as float32 standard normals
     of shape [B, H, L, d];
  2. the tangents dQ, dK, dV are multiplied by ``tangent_std``;
  3. if ``head_scale`` is set, one factor s_h ~ U(lo, hi) per head is drawn
     after the six tensors and multiplies both Q[:, h] and K[:, h];
  4. everything is cast to the workload dtype. The cast values are the
     inputs: kernels and the oracle both read exactly these numbers.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Tuple

import torch

# Mask modes, numbered as in the C header.
DENSE = 0
FRAME_CAUSAL = 1
CHUNK_CAUSAL = 2
TEACHER_FORCING = 3

MODE_NAMES = {
    DENSE: "dense",
    FRAME_CAUSAL: "frame_causal",
    CHUNK_CAUSAL: "chunk_causal",
    TEACHER_FORCING: "teacher_forcing",
}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    mode: int
    tokens_per_frame: int
    n_frames: int
    chunk: int
    dtype: str  # "fp32" or "bf16"
    tangent_std: float
    head_scale: Optional[Tuple[float, float]] = None
    seed: int = 0

    @property
    def L(self) -> int:
        ft = self.tokens_per_frame * self.n_frames
        return 2 * ft if self.mode == TEACHER_FORCING else ft

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads: a tiny fp32 case the oracle finishes in well under a
# second, and four bf16 Wan2.1-480p-shaped cases.
WORKLOADS = {
    "tiny_tf": Workload("tiny_tf", B=1, H=2, d=64, mode=TEACHER_FORCING,
                        tokens_per_frame=16, n_frames=4, chunk=1,
                        dtype="fp32", tangent_std=1.0),
    "frame_causal": Workload("frame_causal", B=1, H=12, d=128,
                             mode=FRAME_CAUSAL, tokens_per_frame=1560,
                             n_frames=21, chunk=1, dtype="bf16",
                             tangent_std=0.1),
    "tf": Workload("tf", B=1, H=12, d=128, mode=TEACHER_FORCING,
                   tokens_per_frame=1560, n_frames=21, chunk=1, dtype="bf16",
                   tangent_std=0.1),
    "chunk_tf": Workload("chunk_tf", B=1, H=12, d=128, mode=TEACHER_FORCING,
                         tokens_per_frame=1560, n_frames=21, chunk=3,
                         dtype="bf16", tangent_std=0.1),
    "tf_long": Workload("tf_long", B=2, H=16, d=128, mode=TEACHER_FORCING,
                        tokens_per_frame=1560, n_frames=33, chunk=1,
                        dtype="bf16", tangent_std=0.1, head_scale=(0.5, 2.0)),
}

# The workload the headline throughput is quoted on: the 65,520-token
# teacher-forcing mask.
HEADLINE = "tf"


def make_inputs(w: Workload, device="cpu", seed: Optional[int] = None):
    """Draw (q, k, v, dq, dk, dv) for workload ``w`` on ``device``.

    Returns a tuple of six contiguous [B, H, L, d] tensors of the workload
    dtype, plus the per-head scale draws (or None). CPU and CUDA generators
    give different streams for the same seed; each stream is reproducible.
    """
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(w.seed if seed is None else seed)
    shape = (w.B, w.H, w.L, w.d)
    out = []
    for _ in range(6):
        out.append(torch.randn(shape, generator=g, device=device,
                               dtype=torch.float32))
    q, k, v, dq, dk, dv = out
    if w.tangent_std != 1.0:
        dq.mul_(w.tangent_std)
        dk.mul_(w.tangent_std)
        dv.mul_(w.tangent_std)
    s = None
    if w.head_scale is not None:
        lo, hi = w.head_scale
        s = torch.rand((w.H,), generator=g, device=device,
                       dtype=torch.float32) * (hi - lo) + lo
        q.mul_(s.view(1, -1, 1, 1))
        k.mul_(s.view(1, -1, 1, 1))
    dt = w.torch_dtype
    res = tuple(t.to(dt).contiguous() for t in (q, k, v, dq, dk, dv))
    return res, s


def sample_rows(L: int, n: int, seed: int = 1234):
    """Seeded sorted sample of ``n`` distinct query rows out of ``L``."""
    import numpy as np
    rng = np.random.default_rng(seed)
    n = min(n, L)
    return np.sort(rng.choice(L, size=n, replace=False)).astype(np.int64)


def rope_table(n_pos: int, d: int, base: float = 10000.0, pos0: int = 0, device="cpu"):
    """cos / sin tables [n_pos, d/2] (float32) for rotary position embedding:
    row p, pair i holds the angle (pos0 + p) * base^(-2i/d). Built in float64
    and rounded once; the rotation itself is the caller's (or kernel's)."""
    import numpy as np
    i = np.arange(d // 2, dtype=np.float64)
    ang = (pos0 + np.arange(n_pos, dtype=np.float64))[:, None] * base ** (-2.0 * i / d)[None, :]
    cos = torch.from_numpy(np.cos(ang).astype(np.float32)).to(device)
    sin = torch.from_numpy(np.sin(ang).astype(np.float32)).to(device)
    return cos.contiguous(), sin.contiguous()
