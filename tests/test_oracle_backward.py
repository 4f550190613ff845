"""Pins for the float64 backward oracle (CPU only): torch autograd of PyTorch's
scaled-dot-product attention, central finite differences, the adjoint
identity with the (separately pinned) forward-mode JVP oracle, and
invariants of the gradient."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from torch.nn.attention import SDPBackend, sdpa_kernel

from oracle import (CHUNK_CAUSAL, DENSE, FRAME_CAUSAL, TEACHER_FORCING, MaskSpec,
                    jvp_attention, key_intervals)
from oracle.attention_backward import attention_backward

SPECS = [
    MaskSpec(DENSE, 5, 4),
    MaskSpec(FRAME_CAUSAL, 6, 5),
    MaskSpec(CHUNK_CAUSAL, 4, 7, 3),
    MaskSpec(TEACHER_FORCING, 5, 4, 1),
    MaskSpec(TEACHER_FORCING, 3, 5, 2),
]


def dense_mask(spec):
    L = spec.length
    m = np.zeros((L, L), dtype=bool)
    for i in range(L):
        for a, b in key_intervals(spec, i):
            m[i, a:b] = True
    return torch.from_numpy(m)


def rand(seed, *shape):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(*shape, generator=g, dtype=torch.float64) for _ in range(4)]


@pytest.mark.parametrize("spec", SPECS, ids=str)
def test_backward_matches_torch_autograd(spec):
    q, k, v, g = rand(1, 2, 2, spec.length, 16)
    mask = dense_mask(spec)
    qa, ka, va = (t.clone().requires_grad_(True) for t in (q, k, v))
    with sdpa_kernel([SDPBackend.MATH]):
        o = F.scaled_dot_product_attention(qa, ka, va, attn_mask=mask)
    (o * g).sum().backward()
    gq, gk, gv = attention_backward(q, k, v, g, spec)
    np.testing.assert_allclose(gq, qa.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(gk, ka.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(gv, va.grad.numpy(), atol=1e-11)


@pytest.mark.parametrize("spec", SPECS[1:4], ids=str)
def test_backward_adjoint_of_jvp(spec):
    # <G, J t> = <J^T G, t>: the backward oracle against the forward-mode one.
    q, k, v, g = rand(2, 1, 2, spec.length, 8)
    dq, dk, dv, _ = rand(3, 1, 2, spec.length, 8)
    _, do, _ = jvp_attention(q, k, v, dq, dk, dv, spec)
    gq, gk, gv = attention_backward(q, k, v, g, spec)
    lhs = float((g.numpy() * do).sum())
    rhs = float((gq * dq.numpy()).sum() + (gk * dk.numpy()).sum() + (gv * dv.numpy()).sum())
    assert abs(lhs - rhs) <= 1e-11 * max(1.0, abs(lhs))


def test_backward_finite_differences():
    spec = MaskSpec(TEACHER_FORCING, 4, 3, 1)
    q, k, v, g = rand(4, 1, 1, spec.length, 8)
    gq, gk, gv = attention_backward(q, k, v, g, spec)
    h = 1e-6

    def loss(q_, k_, v_):
        z = torch.zeros_like(q_)
        o, _, _ = jvp_attention(q_, k_, v_, z, z, z, spec)
        return float((g.numpy() * o).sum())

    for i, (grad, t) in enumerate(((gq, q), (gk, k), (gv, v))):
        dirn = torch.randn(t.shape, generator=torch.Generator().manual_seed(10 + i),
                           dtype=torch.float64)
        args_p = [q, k, v]
        args_m = [q, k, v]
        args_p[i] = t + h * dirn
        args_m[i] = t - h * dirn
        fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
        assert abs(fd - float((grad * dirn.numpy()).sum())) < 1e-7 * max(1.0, abs(fd))


@pytest.mark.parametrize("spec", SPECS, ids=str)
def test_backward_invariants(spec):
    q, k, v, g = rand(5, 1, 1, spec.length, 8)
    gq, gk, gv = attention_backward(q, k, v, g, spec)
    # softmax rows sum to one: the value gradient sums to the total cotangent
    np.testing.assert_allclose(gv.sum(axis=2), g.numpy().sum(axis=2), atol=1e-12)
    # each row's score gradient sums to zero: key gradients sum to zero
    np.testing.assert_allclose(gk.sum(axis=2), 0.0, atol=1e-12)
    zq, zk, zv = attention_backward(q, k, v, torch.zeros_like(g), spec)
    assert np.all(zq == 0) and np.all(zk == 0) and np.all(zv == 0)


def test_backward_linear_in_cotangent():
    spec = MaskSpec(FRAME_CAUSAL, 4, 4)
    q, k, v, g1 = rand(6, 1, 1, spec.length, 8)
    *_, g2 = rand(7, 1, 1, spec.length, 8)
    a1 = attention_backward(q, k, v, g1, spec)
    a2 = attention_backward(q, k, v, g2, spec)
    a12 = attention_backward(q, k, v, 0.5 * g1 - 2.0 * g2, spec)
    for x, y, z in zip(a1, a2, a12):
        np.testing.assert_allclose(z, 0.5 * x - 2.0 * y, atol=1e-12)


def test_backward_token_causal_special_case():
    L, d = 10, 8
    q, k, v, g = rand(8, 1, 2, L, d)
    qa, ka, va = (t.clone().requires_grad_(True) for t in (q, k, v))
    with sdpa_kernel([SDPBackend.MATH]):
        o = F.scaled_dot_product_attention(qa, ka, va, is_causal=True)
    (o * g).sum().backward()
    gq, gk, gv = attention_backward(q, k, v, g, MaskSpec(FRAME_CAUSAL, 1, L))
    np.testing.assert_allclose(gq, qa.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(gk, ka.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(gv, va.grad.numpy(), atol=1e-11)


def test_backward_row_subsets_partition():
    # The loss is a sum over query rows, so the contributions of a partition
    # of the rows add up to the full gradient; gq is exact on its own rows.
    spec = MaskSpec(TEACHER_FORCING, 3, 4, 2)
    q, k, v, g = rand(9, 1, 1, spec.length, 8)
    full = attention_backward(q, k, v, g, spec)
    L = spec.length
    perm = np.random.default_rng(3).permutation(L)
    parts = [sorted(perm[:7]), sorted(perm[7:15]), sorted(perm[15:])]
    acc = [np.zeros_like(x) for x in full]
    for rows in parts:
        sub = attention_backward(q, k, v, g, spec, rows=rows)
        rest = np.setdiff1d(np.arange(L), rows)
        np.testing.assert_allclose(sub[0][:, :, rows], full[0][:, :, rows], atol=1e-12)
        assert np.all(sub[0][:, :, rest] == 0)
        for a, x in zip(acc, sub):
            a += x
    for a, x in zip(acc, full):
        np.testing.assert_allclose(a, x, atol=1e-12)


def test_fully_masked_row_contributes_nothing(monkeypatch):
    # A query row without keys (injected: no descriptor of the four modes
    # has one) has O = 0 whatever q, k, v are, so its cotangent reaches
    # nothing: the gradients equal those of the unmodified mask with that
    # row's cotangent set to zero, and its own query gradient is zero.
    import sys
    ob = sys.modules["oracle.attention_backward"]
    oj = sys.modules["oracle.jvp_attention"]  # the package re-exports a function of that name
    spec = MaskSpec(TEACHER_FORCING, 4, 3, 1)
    q, k, v, g = rand(31, 1, 2, spec.length, 8)
    empty = [2, 9, 17]
    g0 = g.clone()
    g0[:, :, empty] = 0
    ref = attention_backward(q, k, v, g0, spec)
    real = oj.key_intervals
    monkeypatch.setattr(oj, "key_intervals",
                        lambda s, i: [] if i in empty else real(s, i))
    assert ob._group_rows is oj._group_rows
    got = attention_backward(q, k, v, g, spec)
    assert np.all(got[0][:, :, empty] == 0)
    for a, b in zip(got, ref):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
