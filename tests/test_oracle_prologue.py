"""Pins for the attention-layer tangent prologue oracle (CPU only): torch's
rms_norm for the primal, torch.func.jvp (forward-mode autodiff) for the
tangents of the whole chain, finite differences, the scale invariance of
RMS normalisation, and the plain layout when no norm or rotation applies."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from attention_jvp_continuous_b200.inputs import rope_table
from oracle.layer_prologue import qkv_prologue, rms_norm_jvp


def rand(seed, *shape, n=1):
    g = torch.Generator().manual_seed(seed)
    out = [torch.randn(*shape, generator=g, dtype=torch.float64) for _ in range(n)]
    return out if n > 1 else out[0]


@pytest.mark.parametrize("C,group", [(64, 64), (64, 16), (96, 32)])
def test_rms_norm_primal_and_tangent_match_torch(C, group):
    a, da = rand(1, 3, 5, C, n=2)
    w = rand(2, group)
    eps = 1e-5

    def f(x):
        return F.rms_norm(x.reshape(3, 5, C // group, group), (group,), w, eps).reshape(3, 5, C)

    y_ref, dy_ref = torch.func.jvp(f, (a,), (da,))
    y, dy = rms_norm_jvp(a, da, w, group, eps)
    np.testing.assert_allclose(y, y_ref.numpy(), atol=1e-12)
    np.testing.assert_allclose(dy, dy_ref.numpy(), atol=1e-12)


def test_rms_norm_finite_differences():
    a, da = rand(3, 4, 48, n=2)
    w = rand(4, 48)
    h = 1e-6
    yp, _ = rms_norm_jvp(a + h * da, da, w, 48, 1e-6)
    ym, _ = rms_norm_jvp(a - h * da, da, w, 48, 1e-6)
    _, dy = rms_norm_jvp(a, da, w, 48, 1e-6)
    np.testing.assert_allclose((yp - ym) / (2 * h), dy, atol=1e-7)


def test_rms_norm_is_scale_invariant():
    # Without eps the norm ignores the scale of its input, so the tangent
    # along the input itself vanishes, for every group.
    a = rand(5, 2, 64)
    for group in (64, 16):
        _, dy = rms_norm_jvp(a, 3.0 * a, np.ones(group), group, 0.0)
        assert np.abs(dy).max() < 1e-12


def test_prologue_chain_matches_forward_autodiff():
    B, L, H, d = 2, 7, 3, 16
    C = H * d
    P, dP = rand(6, B, L, 3 * C, n=2)
    wq, wk = rand(7, C), rand(8, C)
    cos, sin = rope_table(L, d, pos0=4)
    c64, s64 = cos.double(), sin.double()

    def rot(x):  # [B, H, L, d] by token row, as complex multiplication
        z = torch.complex(x[..., 0::2], x[..., 1::2]) * torch.complex(c64, s64)
        return torch.stack([z.real, z.imag], dim=-1).reshape(x.shape)

    def heads(x):
        return x.reshape(B, L, H, d).transpose(1, 2)

    def f(p):
        q = heads(F.rms_norm(p[..., :C], (C,), wq, 1e-6))
        k = heads(F.rms_norm(p[..., C:2 * C], (C,), wk, 1e-6))
        return rot(q), rot(k), heads(p[..., 2 * C:])

    prim, tang = torch.func.jvp(f, (P,), (dP,))
    out = qkv_prologue(P, dP, H, d, wq, wk, C, 1e-6, cos, sin)
    for got, ref in zip(out, list(prim) + list(tang)):
        np.testing.assert_allclose(got, ref.numpy(), atol=1e-12)


def test_prologue_per_head_norm_matches_autodiff():
    B, L, H, d = 1, 5, 4, 8
    C = H * d
    P, dP = rand(9, B, L, 3 * C, n=2)
    wq, wk = rand(10, d), rand(11, d)

    def f(p):
        q = F.rms_norm(p[..., :C].reshape(B, L, H, d), (d,), wq, 1e-6).transpose(1, 2)
        k = F.rms_norm(p[..., C:2 * C].reshape(B, L, H, d), (d,), wk, 1e-6).transpose(1, 2)
        return q, k

    (q_ref, k_ref), (dq_ref, dk_ref) = torch.func.jvp(f, (P,), (dP,))
    q, k, _, dq, dk, _ = qkv_prologue(P, dP, H, d, wq, wk, d, 1e-6)
    for got, ref in ((q, q_ref), (k, k_ref), (dq, dq_ref), (dk, dk_ref)):
        np.testing.assert_allclose(got, ref.numpy(), atol=1e-12)


def test_prologue_plain_layout():
    B, L, H, d = 2, 3, 2, 4
    P, dP = rand(12, B, L, 3 * H * d, n=2)
    q, k, v, dq, dk, dv = qkv_prologue(P, dP, H, d)
    for b in range(B):
        for h in range(H):
            for t in range(L):
                for j in range(d):
                    c = h * d + j
                    assert q[b, h, t, j] == P[b, t, c] and k[b, h, t, j] == P[b, t, H * d + c]
                    assert v[b, h, t, j] == P[b, t, 2 * H * d + c]
                    assert dv[b, h, t, j] == dP[b, t, 2 * H * d + c]
