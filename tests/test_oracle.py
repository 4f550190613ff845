"""Pins for the float64 oracle (CPU only).

Nothing here compares the oracle with itself. Each check ties it to
something fixed from outside: hand-written frame-level masks taken from the
pages' prose (tests/golden), closed-form pair counts, torch autodiff of
PyTorch's own scaled-dot-product attention, central finite differences,
algebraic invariants of the JVP, and textbook special cases.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from torch.nn.attention import SDPBackend, sdpa_kernel

from oracle import (CHUNK_CAUSAL, DENSE, FRAME_CAUSAL, TEACHER_FORCING,
                    MaskSpec, allowed_pairs, jvp_attention, jvp_attention_head,
                    key_intervals)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def dense_mask(spec):
    L = spec.length
    m = np.zeros((L, L), dtype=bool)
    for i in range(L):
        for a, b in key_intervals(spec, i):
            m[i, a:b] = True
    return m


def load_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([int(x) for x in line.split()])
    return np.array(rows, dtype=bool)


# --------------------------------------------------------------- masks ----

@pytest.mark.parametrize("fname,spec", [
    ("frame_causal_F4.txt", MaskSpec(FRAME_CAUSAL, 3, 4)),
    ("chunk_causal_F5_c2.txt", MaskSpec(CHUNK_CAUSAL, 3, 5, 2)),
    ("teacher_forcing_F4_c1.txt", MaskSpec(TEACHER_FORCING, 3, 4, 1)),
    ("teacher_forcing_F5_c2.txt", MaskSpec(TEACHER_FORCING, 2, 5, 2)),
    ("dense_F3.txt", MaskSpec(DENSE, 4, 3)),
])
def test_mask_matches_hand_written_frame_pattern(fname, spec):
    gold = load_golden(fname)
    T = spec.tokens_per_frame
    m = dense_mask(spec)
    nf = spec.length // T
    assert gold.shape == (nf, nf)
    for fi in range(nf):
        for fj in range(nf):
            blk = m[fi * T:(fi + 1) * T, fj * T:(fj + 1) * T]
            # spatial attention is full: each frame block is all-or-nothing
            assert blk.all() or not blk.any(), (fi, fj)
            assert bool(blk.all()) == bool(gold[fi, fj]), (fi, fj)


def literal_predicate(spec, i, j):
    """Per-pair predicate in frame/chunk terms, straight from the prose."""
    T, Fn, ch = spec.tokens_per_frame, spec.n_frames, spec.chunk
    if spec.mode == DENSE:
        return True
    if spec.mode == FRAME_CAUSAL:
        return j // T <= i // T
    if spec.mode == CHUNK_CAUSAL:
        return (j // T) // ch <= (i // T) // ch
    FT = T * Fn
    qi_noisy, kj_noisy = i >= FT, j >= FT
    fi, fj = (i % FT) // T, (j % FT) // T
    ci, cj = fi // ch, fj // ch
    if not qi_noisy:
        return (not kj_noisy) and cj <= ci
    if kj_noisy:
        return cj == ci
    return cj < ci


@pytest.mark.parametrize("seed", range(12))
def test_mask_matches_literal_predicate(seed):
    rng = np.random.default_rng(seed)
    mode = [DENSE, FRAME_CAUSAL, CHUNK_CAUSAL, TEACHER_FORCING][seed % 4]
    spec = MaskSpec(mode, int(rng.integers(1, 6)), int(rng.integers(1, 7)),
                    int(rng.integers(1, 4)))
    m = dense_mask(spec)
    L = spec.length
    lit = np.array([[literal_predicate(spec, i, j) for j in range(L)]
                    for i in range(L)])
    np.testing.assert_array_equal(m, lit)
    # every row admits at least its own token
    assert m[np.arange(L), np.arange(L)].all()


def test_pair_counts_closed_forms_workloads():
    # Wan2.1 480p: 21 latent frames of 1560 tokens; 33 frames for the long one.
    T = 1560
    assert allowed_pairs(MaskSpec(FRAME_CAUSAL, T, 21)) == T * T * 21 * 22 // 2 == 562_161_600
    assert allowed_pairs(MaskSpec(TEACHER_FORCING, T, 21, 1)) == T * T * 21 * 22 == 1_124_323_200
    S, K = 3 * T, 7
    assert allowed_pairs(MaskSpec(TEACHER_FORCING, T, 21, 3)) == S * S * K * (K + 1) == 1_226_534_400
    assert allowed_pairs(MaskSpec(TEACHER_FORCING, T, 33, 1)) == T * T * 33 * 34 == 2_730_499_200
    assert allowed_pairs(MaskSpec(TEACHER_FORCING, 16, 4, 1)) == 16 * 16 * 4 * 5 == 5_120


@pytest.mark.parametrize("T,Fn,ch", [(1, 1, 1), (2, 6, 3), (5, 4, 2), (7, 9, 3), (3, 8, 4)])
def test_pair_counts_closed_forms_small(T, Fn, ch):
    L = T * Fn
    assert allowed_pairs(MaskSpec(DENSE, T, Fn)) == L * L
    assert allowed_pairs(MaskSpec(FRAME_CAUSAL, T, Fn)) == T * T * Fn * (Fn + 1) // 2
    S, K = ch * T, Fn // ch  # Fn divisible by ch in these cases
    assert allowed_pairs(MaskSpec(CHUNK_CAUSAL, T, Fn, ch)) == S * S * K * (K + 1) // 2
    assert allowed_pairs(MaskSpec(TEACHER_FORCING, T, Fn, ch)) == S * S * K * (K + 1)


# ------------------------------------------------------------ numerics ----

def rand_inputs(seed, B, H, L, d, tscale=1.0):
    g = torch.Generator().manual_seed(seed)
    xs = [torch.randn(B, H, L, d, generator=g, dtype=torch.float64) for _ in range(6)]
    for t in xs[3:]:
        t.mul_(tscale)
    return xs


def torch_reference(q, k, v, dq, dk, dv, spec, scale=None):
    """O, dO via forward-mode autodiff of PyTorch's own attention; LSE via
    torch.logsumexp over the masked scores."""
    mask = torch.from_numpy(dense_mask(spec))

    def f(q, k, v):
        with sdpa_kernel([SDPBackend.MATH]):
            return F.scaled_dot_product_attention(q, k, v, attn_mask=mask,
                                                  scale=scale)
    o, do = torch.func.jvp(f, (q, k, v), (dq, dk, dv))
    c = 1 / math.sqrt(q.shape[-1]) if scale is None else scale
    s = (q @ k.transpose(-1, -2)) * c
    s = s.masked_fill(~mask, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    return o.numpy(), do.numpy(), lse.numpy()


SPECS = [
    MaskSpec(DENSE, 5, 4),
    MaskSpec(FRAME_CAUSAL, 6, 5),
    MaskSpec(CHUNK_CAUSAL, 4, 7, 3),
    MaskSpec(TEACHER_FORCING, 5, 4, 1),
    MaskSpec(TEACHER_FORCING, 3, 5, 2),
    MaskSpec(TEACHER_FORCING, 16, 4, 1),
]


@pytest.mark.parametrize("spec", SPECS, ids=lambda s: f"m{s.mode}T{s.tokens_per_frame}F{s.n_frames}c{s.chunk}")
@pytest.mark.parametrize("d", [8, 64])
def test_oracle_matches_torch_autodiff(spec, d):
    q, k, v, dq, dk, dv = rand_inputs(7 + d, 2, 2, spec.length, d)
    o_ref, do_ref, lse_ref = torch_reference(q, k, v, dq, dk, dv, spec)
    o, do, lse = jvp_attention(q, k, v, dq, dk, dv, spec)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(do, do_ref, rtol=0, atol=1e-11)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


def test_oracle_explicit_scale_matches_torch():
    spec = MaskSpec(TEACHER_FORCING, 4, 3, 1)
    q, k, v, dq, dk, dv = rand_inputs(3, 1, 2, spec.length, 16)
    o_ref, do_ref, lse_ref = torch_reference(q, k, v, dq, dk, dv, spec, scale=0.37)
    o, do, lse = jvp_attention(q, k, v, dq, dk, dv, spec, scale=0.37)
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(do, do_ref, atol=1e-11)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12)


@pytest.mark.parametrize("spec", SPECS[1:5], ids=str)
def test_central_finite_differences(spec):
    q, k, v, dq, dk, dv = rand_inputs(11, 1, 1, spec.length, 16)
    h = 1e-5
    args = [t.numpy() for t in (q, k, v)]
    tang = [t.numpy() for t in (dq, dk, dv)]
    plus = [a + h * t for a, t in zip(args, tang)]
    minus = [a - h * t for a, t in zip(args, tang)]
    zeros = [np.zeros_like(a) for a in args]
    op, _, lp = jvp_attention(*plus, *zeros, spec)
    om, _, lm = jvp_attention(*minus, *zeros, spec)
    _, do, _ = jvp_attention(*args, *tang, spec)
    fd = (op - om) / (2 * h)
    rel = np.linalg.norm(fd - do) / np.linalg.norm(do)
    assert rel < 1e-8, rel


def test_zero_tangent_gives_zero():
    spec = MaskSpec(TEACHER_FORCING, 4, 4, 1)
    q, k, v, *_ = rand_inputs(1, 1, 2, spec.length, 8)
    z = torch.zeros_like(q)
    _, do, _ = jvp_attention(q, k, v, z, z, z, spec)
    assert np.all(do == 0.0)


def test_value_direction_gives_output():
    # O is linear in V, so the tangent (0, 0, V) reproduces O.
    spec = MaskSpec(CHUNK_CAUSAL, 3, 6, 2)
    q, k, v, *_ = rand_inputs(2, 1, 2, spec.length, 8)
    z = torch.zeros_like(q)
    o, do, _ = jvp_attention(q, k, v, z, z, v, spec)
    np.testing.assert_allclose(do, o, atol=1e-13)


def test_constant_value_tangent_rows():
    # Softmax weights sum to one: dV with every row = w gives dO rows = w.
    spec = MaskSpec(TEACHER_FORCING, 3, 5, 1)
    q, k, v, *_ = rand_inputs(3, 1, 1, spec.length, 8)
    w = torch.randn(8, dtype=torch.float64)
    dv = w.expand_as(v).clone()
    z = torch.zeros_like(q)
    _, do, _ = jvp_attention(q, k, v, z, z, dv, spec)
    np.testing.assert_allclose(do[0, 0], np.broadcast_to(w.numpy(), do[0, 0].shape), atol=1e-13)


@pytest.mark.parametrize("mode", [DENSE, FRAME_CAUSAL, CHUNK_CAUSAL, TEACHER_FORCING])
def test_constant_key_tangent_is_shift_invariant(mode):
    # dK rows all = u shifts every admissible score of a row by the same
    # amount; softmax is shift invariant, so dO = 0 under any mask.
    spec = MaskSpec(mode, 3, 4, 2)
    q, k, v, *_ = rand_inputs(4, 1, 2, spec.length, 8)
    u = torch.randn(8, dtype=torch.float64)
    dk = u.expand_as(k).clone()
    z = torch.zeros_like(q)
    _, do, _ = jvp_attention(q, k, v, z, dk, z, spec)
    assert np.abs(do).max() < 1e-13


def test_query_and_key_directions_agree_with_temperature_derivative():
    # Tangents (Q,0,0) and (0,K,0) both scale the scores by (1+eps): each
    # equals d/dbeta softmax(beta S) V at beta = 1.
    spec = MaskSpec(TEACHER_FORCING, 4, 3, 1)
    q, k, v, *_ = rand_inputs(5, 1, 1, spec.length, 8)
    z = torch.zeros_like(q)
    _, do_q, _ = jvp_attention(q, k, v, q, z, z, spec)
    _, do_k, _ = jvp_attention(q, k, v, z, k, z, spec)
    np.testing.assert_allclose(do_q, do_k, atol=1e-13)
    h = 1e-6
    c = 1 / math.sqrt(8)
    op, _, _ = jvp_attention(q, k, v, z, z, z, spec, scale=c * (1 + h))
    om, _, _ = jvp_attention(q, k, v, z, z, z, spec, scale=c * (1 - h))
    np.testing.assert_allclose(do_q, (op - om) / (2 * h), atol=1e-7)


def test_linearity_in_tangent():
    spec = MaskSpec(FRAME_CAUSAL, 4, 4)
    q, k, v, *t1 = rand_inputs(6, 1, 1, spec.length, 8)
    *_, t2a, t2b, t2c = rand_inputs(60, 1, 1, spec.length, 8)
    t2 = [t2a, t2b, t2c]
    a, b = 0.7, -1.9
    _, d1, _ = jvp_attention(q, k, v, *t1, spec)
    _, d2, _ = jvp_attention(q, k, v, *t2, spec)
    _, d12, _ = jvp_attention(q, k, v, *[a * x + b * y for x, y in zip(t1, t2)], spec)
    np.testing.assert_allclose(d12, a * d1 + b * d2, atol=1e-12)


def test_dense_equals_full_chunk_and_unmasked_attention():
    T, Fn, d = 4, 5, 8
    q, k, v, dq, dk, dv = rand_inputs(8, 1, 2, T * Fn, d)
    r_dense = jvp_attention(q, k, v, dq, dk, dv, MaskSpec(DENSE, T, Fn))
    r_chunk = jvp_attention(q, k, v, dq, dk, dv, MaskSpec(CHUNK_CAUSAL, T, Fn, Fn))
    for a, b in zip(r_dense, r_chunk):
        np.testing.assert_array_equal(a, b)

    def f(q, k, v):
        with sdpa_kernel([SDPBackend.MATH]):
            return F.scaled_dot_product_attention(q, k, v)
    o, do = torch.func.jvp(f, (q, k, v), (dq, dk, dv))
    np.testing.assert_allclose(r_dense[0], o.numpy(), atol=1e-12)
    np.testing.assert_allclose(r_dense[1], do.numpy(), atol=1e-11)


def test_frame_causal_single_token_frames_is_token_causal():
    L, d = 12, 8
    q, k, v, dq, dk, dv = rand_inputs(9, 1, 2, L, d)
    o, do, _ = jvp_attention(q, k, v, dq, dk, dv, MaskSpec(FRAME_CAUSAL, 1, L))

    def f(q, k, v):
        with sdpa_kernel([SDPBackend.MATH]):
            return F.scaled_dot_product_attention(q, k, v, is_causal=True)
    o_t, do_t = torch.func.jvp(f, (q, k, v), (dq, dk, dv))
    np.testing.assert_allclose(o, o_t.numpy(), atol=1e-12)
    np.testing.assert_allclose(do, do_t.numpy(), atol=1e-11)


def test_teacher_forcing_clean_rows_ignore_noisy_tangent():
    # TF-sCM: the clean context carries a zero tangent, only the noisy half
    # follows the teacher velocity (Causal-rCM report, Sec. 3.1.2). Clean
    # queries see only clean keys, so their dO must vanish.
    spec = MaskSpec(TEACHER_FORCING, 4, 4, 1)
    FT = spec.frame_tokens
    q, k, v, dq, dk, dv = rand_inputs(10, 1, 2, spec.length, 8)
    for t in (dq, dk, dv):
        t[:, :, :FT] = 0
    _, do, _ = jvp_attention(q, k, v, dq, dk, dv, spec)
    assert np.all(do[:, :, :FT] == 0.0)
    assert np.abs(do[:, :, FT:]).max() > 1e-3


def test_first_noisy_frame_sees_only_itself():
    # Noisy frame 0 has no clean history: it is plain attention over its own
    # T tokens.
    T, Fn, d = 5, 3, 8
    spec = MaskSpec(TEACHER_FORCING, T, Fn, 1)
    FT = T * Fn
    q, k, v, dq, dk, dv = rand_inputs(12, 1, 1, spec.length, d)
    rows = np.arange(FT, FT + T)
    o, do, _ = jvp_attention(q, k, v, dq, dk, dv, spec, rows=rows)
    sl = slice(FT, FT + T)

    def f(q, k, v):
        with sdpa_kernel([SDPBackend.MATH]):
            return F.scaled_dot_product_attention(q, k, v)
    o_t, do_t = torch.func.jvp(f, (q[:, :, sl], k[:, :, sl], v[:, :, sl]),
                               (dq[:, :, sl], dk[:, :, sl], dv[:, :, sl]))
    np.testing.assert_allclose(o, o_t.numpy(), atol=1e-12)
    np.testing.assert_allclose(do, do_t.numpy(), atol=1e-11)


def test_row_subset_matches_full_evaluation():
    spec = MaskSpec(TEACHER_FORCING, 6, 4, 2)
    q, k, v, dq, dk, dv = rand_inputs(13, 1, 1, spec.length, 8)
    full = jvp_attention(q, k, v, dq, dk, dv, spec)
    rows = np.array([0, 5, 17, 30, 47])
    sub = jvp_attention(q, k, v, dq, dk, dv, spec, rows=rows)
    for a, b in zip(full, sub):
        # BLAS may block the two evaluations differently: equal up to rounding
        np.testing.assert_allclose(a[:, :, rows], b, rtol=0, atol=1e-13)


def test_head_function_rejects_length_mismatch():
    spec = MaskSpec(FRAME_CAUSAL, 4, 4)
    x = np.zeros((15, 8))
    with pytest.raises(ValueError):
        jvp_attention_head(x, x, x, x, x, x, spec)


def test_fully_masked_row_convention(monkeypatch):
    # No descriptor of the four modes leaves a query row without keys, so
    # the oracle's empty-row branch is reached by injecting an empty key
    # set for some rows. Their O and dO are sums over no keys (zero) and
    # their LSE is the log-sum-exp of no scores, which torch gives as -inf;
    # every other row must be exactly what the unmodified mask gives.
    import sys
    oj = sys.modules["oracle.jvp_attention"]  # the package re-exports a function of that name
    spec = MaskSpec(TEACHER_FORCING, 4, 3, 1)
    q, k, v, dq, dk, dv = rand_inputs(21, 1, 2, spec.length, 8)
    ref = jvp_attention(q, k, v, dq, dk, dv, spec)
    empty = {0, 5, 13, 20}
    real = oj.key_intervals
    monkeypatch.setattr(oj, "key_intervals",
                        lambda s, i: [] if i in empty else real(s, i))
    o, do, lse = jvp_attention(q, k, v, dq, dk, dv, spec)
    rows = sorted(empty)
    others = [i for i in range(spec.length) if i not in empty]
    assert np.all(o[:, :, rows] == 0) and np.all(do[:, :, rows] == 0)
    lse_empty = torch.logsumexp(torch.full((3,), float("-inf"), dtype=torch.float64), 0)
    assert np.all(lse[:, :, rows] == lse_empty.item())
    for a, b in zip((o, do, lse), ref):
        np.testing.assert_array_equal(a[:, :, others], b[:, :, others])
