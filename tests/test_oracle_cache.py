"""Pins for the KV-cache oracle (CPU only): torch scaled-dot-product
attention and logsumexp, the rollout identity with the packed masked
forward (chunk-causal and teacher forcing), and rotation invariants of RoPE
checked against complex multiplication."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F
from torch.nn.attention import SDPBackend, sdpa_kernel

from attention_jvp_continuous_b200.inputs import rope_table
from oracle import (CHUNK_CAUSAL, FRAME_CAUSAL, TEACHER_FORCING, MaskSpec, cache_attention,
                    jvp_attention, rope_rows)


def rand(seed, *shape, n=3):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(*shape, generator=g, dtype=torch.float64) for _ in range(n)]


@pytest.mark.parametrize("lq,lk,lcache", [(5, 9, 12), (16, 16, 16), (1, 30, 33)])
def test_cache_attention_matches_sdpa(lq, lk, lcache):
    q, = rand(1, 2, 3, lq, 16, n=1)
    k, v = rand(2, 2, 3, lcache, 16, n=2)
    o, lse = cache_attention(q, k, v, lk)
    with sdpa_kernel([SDPBackend.MATH]):
        ref = F.scaled_dot_product_attention(q, k[:, :, :lk], v[:, :, :lk])
    np.testing.assert_allclose(o, ref.numpy(), atol=1e-12)
    s = (q @ k[:, :, :lk].transpose(-1, -2)) / 4.0
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), atol=1e-12)


def test_cache_rows_past_n_keys_are_ignored():
    q, = rand(3, 1, 1, 4, 8, n=1)
    k, v = rand(4, 1, 1, 10, 8, n=2)
    o1, l1 = cache_attention(q, k, v, 6)
    k2, v2 = k.clone(), v.clone()
    k2[:, :, 6:] = 1e6
    v2[:, :, 6:] = float("nan")
    o2, l2 = cache_attention(q, k2, v2, 6)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


@pytest.mark.parametrize("spec", [MaskSpec(CHUNK_CAUSAL, 3, 6, 2), MaskSpec(FRAME_CAUSAL, 4, 5)],
                         ids=str)
def test_rollout_reproduces_packed_chunk_causal(spec):
    # Generating chunk by chunk against a growing cache (each chunk's own
    # keys at its cache position) gives the packed chunk-causal forward.
    L = spec.length
    q, k, v = rand(5, 1, 2, L, 8)
    z = torch.zeros_like(q)
    o_ref, _, lse_ref = jvp_attention(q, k, v, z, z, z, spec)
    S = spec.chunk_tokens
    for c0 in range(0, L, S):
        c1 = min(c0 + S, L)
        o, lse = cache_attention(q[:, :, c0:c1], k, v, c1)
        np.testing.assert_allclose(o, o_ref[:, :, c0:c1], atol=1e-12)
        np.testing.assert_allclose(lse, lse_ref[:, :, c0:c1], atol=1e-12)


@pytest.mark.parametrize("chunk", [1, 2])
def test_rollout_reproduces_teacher_forcing_noisy_rows(chunk):
    # A noisy chunk of the packed teacher-forcing forward sees the clean
    # chunks before it and itself: a cache holding the clean history, with
    # the noisy chunk's own keys appended at its position.
    spec = MaskSpec(TEACHER_FORCING, 3, 4, chunk)
    L, FT, S = spec.length, spec.length // 2, spec.chunk_tokens
    q, k, v = rand(6, 1, 2, L, 8)
    z = torch.zeros_like(q)
    o_ref, _, lse_ref = jvp_attention(q, k, v, z, z, z, spec)
    for c0 in range(0, FT, S):
        c1 = min(c0 + S, FT)
        kc = torch.cat([k[:, :, :c0], k[:, :, FT + c0:FT + c1]], dim=2)
        vc = torch.cat([v[:, :, :c0], v[:, :, FT + c0:FT + c1]], dim=2)
        o, lse = cache_attention(q[:, :, FT + c0:FT + c1], kc, vc, c1)
        np.testing.assert_allclose(o, o_ref[:, :, FT + c0:FT + c1], atol=1e-12)
        np.testing.assert_allclose(lse, lse_ref[:, :, FT + c0:FT + c1], atol=1e-12)


def test_rope_is_complex_multiplication():
    x, = rand(7, 2, 3, 11, 16, n=1)
    cos, sin = rope_table(11, 16, pos0=5)
    y = rope_rows(x, cos, sin)
    z = torch.complex(x[..., 0::2], x[..., 1::2]) * torch.polar(
        torch.ones_like(cos, dtype=torch.float64), torch.atan2(sin.double(), cos.double()))
    # the table rows have |(c, s)| = 1 up to float32 rounding
    scale = torch.sqrt(cos.double() ** 2 + sin.double() ** 2)
    np.testing.assert_allclose(y[..., 0::2], (z.real * scale).numpy(), atol=1e-12)
    np.testing.assert_allclose(y[..., 1::2], (z.imag * scale).numpy(), atol=1e-12)


def test_rope_invariants():
    x, = rand(8, 1, 2, 9, 32, n=1)
    cos, sin = rope_table(9, 32, pos0=3)
    y = rope_rows(x, cos, sin)
    # zero angle is the identity
    np.testing.assert_array_equal(rope_rows(x, torch.ones(9, 16), torch.zeros(9, 16)), x.numpy())
    # each pair keeps its length (table rounding aside)
    n_x = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    n_y = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    np.testing.assert_allclose(n_y, n_x.numpy(), rtol=1e-6)
    # the opposite angle undoes it
    back = rope_rows(y, cos, -sin)
    np.testing.assert_allclose(back, x.numpy(), atol=1e-5)


def test_rope_scores_depend_on_relative_position():
    q, k = rand(9, 1, 1, 1, 64, n=2)
    d = 64

    def score(m, n):
        cq, sq = rope_table(1, d, pos0=m)
        ck, sk = rope_table(1, d, pos0=n)
        return float((rope_rows(q[0, 0], cq, sq) * rope_rows(k[0, 0], ck, sk)).sum())

    for m, n, t in [(3, 1, 7), (10, 20, 100), (0, 0, 50)]:
        assert abs(score(m, n) - score(m + t, n + t)) < 1e-4 * (1 + abs(score(m, n)))
