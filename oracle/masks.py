"""Temporal attention masks, oracle side (test infrastructure only).

Token layout: frame-major, the tokens_per_frame (T) spatial tokens of one
frame contiguous; a chunk is ``chunk`` consecutive frames, the last chunk
possibly shorter. Spatial attention inside a frame is always full; only
the temporal axis is masked (third-party reading notes on the Causal-rCM
report, mask-pattern table and the note under it).

Modes (token index n, frame f(n) = n // T, chunk c(n) = f(n) // chunk):

* DENSE: every key (bidirectional; the reading notes' "full" row).
* FRAME_CAUSAL (L = F*T): key j allowed iff f(j) <= f(i). The notes' table
  says "only strictly past frames" for the frame-level row, while the note
  under it says a frame's own spatial tokens are always visible; the own
  frame is therefore included (frame-wise AR, c1-1).
* CHUNK_CAUSAL (L = F*T): allowed iff c(j) <= c(i): full inside a chunk,
  causal across chunks (Causal-rCM report, Section 2.3, diffusion forcing
  "block-causal attention mask"; c3-3 chunk pattern, Section 4.1).
* TEACHER_FORCING (L = 2*F*T): the packed sequence is [clean ; noisy]
  (report, Table 2 notes: "[clean frames, noisy frames] concatenation").
  Clean query i sees clean keys with c(j) <= c(i) and no noisy key.
  Noisy query with local index i' sees clean keys with c(j) < c(i') and
  the noisy keys of its own chunk (report, Section 3.1.1 after Eq. 8:
  each noisy block sees only its allowed clean history and its own noisy
  tokens).

This module writes the admissible set of each query row as a short list of
half-open key intervals, the "query group -> key ranges" form of Appendix B
("Sparse custom-mask representation").
"""
from __future__ import annotations

import dataclasses
from typing import List, Tuple

DENSE = 0
FRAME_CAUSAL = 1
CHUNK_CAUSAL = 2
TEACHER_FORCING = 3


@dataclasses.dataclass(frozen=True)
class MaskSpec:
    mode: int
    tokens_per_frame: int
    n_frames: int
    chunk: int = 1

    def __post_init__(self):
        if self.mode not in (DENSE, FRAME_CAUSAL, CHUNK_CAUSAL, TEACHER_FORCING):
            raise ValueError(f"unknown mask mode {self.mode}")
        if self.tokens_per_frame < 1 or self.n_frames < 1 or self.chunk < 1:
            raise ValueError("tokens_per_frame, n_frames and chunk must be >= 1")

    @property
    def frame_tokens(self) -> int:
        """F*T: tokens in one copy of the video (clean or noisy)."""
        return self.tokens_per_frame * self.n_frames

    @property
    def length(self) -> int:
        ft = self.frame_tokens
        return 2 * ft if self.mode == TEACHER_FORCING else ft

    @property
    def chunk_tokens(self) -> int:
        c = 1 if self.mode == FRAME_CAUSAL else self.chunk
        return c * self.tokens_per_frame


def key_intervals(spec: MaskSpec, i: int) -> List[Tuple[int, int]]:
    """Admissible keys of query token i as sorted, disjoint [a, b) intervals."""
    L = spec.length
    if not 0 <= i < L:
        raise IndexError(i)
    FT = spec.frame_tokens
    if spec.mode == DENSE:
        return [(0, L)]
    S = spec.chunk_tokens
    if spec.mode in (FRAME_CAUSAL, CHUNK_CAUSAL):
        end = min((i // S + 1) * S, FT)
        return [(0, end)]
    # teacher forcing
    if i < FT:
        return [(0, min((i // S + 1) * S, FT))]
    ii = i - FT
    c0 = (ii // S) * S           # first token of the query's own chunk
    c1 = min(c0 + S, FT)         # one past its last token
    out = []
    if c0 > 0:
        out.append((0, c0))      # clean chunks strictly before
    out.append((FT + c0, FT + c1))  # own noisy chunk
    return out


def allowed_pairs(spec: MaskSpec) -> int:
    """Number of admissible (query, key) pairs, summed row by row."""
    return sum(b - a for i in range(spec.length)
               for a, b in key_intervals(spec, i))
