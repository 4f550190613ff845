"""GPU parity of the attention-layer tangent prologue (jvp_attn_qkv_prologue)
against the float64 oracle, alone and chained into the attention JVP
kernel on a teacher-forcing mask."""
import numpy as np
import pytest
import torch

import attention_jvp_continuous_b200 as ja
from attention_jvp_continuous_b200.inputs import rope_table
from oracle import MaskSpec, TEACHER_FORCING, jvp_attention
from oracle.layer_prologue import qkv_prologue

pytestmark = pytest.mark.gpu


def randn(seed, shape, dtype=torch.bfloat16, std=1.0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(dtype).cuda()


def close_bf16(out, ref, what):
    # one bf16 rounding of an fp32 result: half an ulp (2^-8) of the value,
    # plus fp32 cancellation in the tangent (da - a <a, da> r^2)
    got = out.double().cpu().numpy()
    tol = 2.0 ** -8 * 1.01 * np.abs(ref) + 1e-4 * np.abs(ref).max()
    bad = np.abs(got - ref) > tol
    assert not bad.any(), (what, np.abs(got - ref).max(), np.abs(ref).max())


CASES = [  # B, L, H, d, norm group ("C", "d" or None), rotate
    (1, 100, 12, 128, "C", True),
    (2, 37, 4, 64, "d", True),
    (1, 50, 2, 128, "d", False),
    (1, 20, 2, 128, None, True),
    (2, 9, 8, 32, None, False),
    (1, 40, 16, 128, "d", True),   # 8 vectors per lane: the widest register-resident form
    (1, 30, 24, 128, "C", True),   # H*d = 3072: the two-pass loop for wider layers
    (1, 25, 2, 256, "d", True),    # d = 256: a head spans all 32 lanes
    (2, 17, 32, 8, "d", True),     # d = 8: a head is one vector
]


@pytest.mark.parametrize("B,L,H,d,group,rotate", CASES)
def test_prologue_matches_oracle(B, L, H, d, group, rotate):
    C = H * d
    P = randn(1, (B, L, 3 * C), std=2.0)
    dP = randn(2, (B, L, 3 * C), std=0.1)
    ng = {"C": C, "d": d, None: None}[group]
    wq = (randn(3, (ng,), torch.float32) * 0.2 + 1.0) if ng else None
    wk = (randn(4, (ng,), torch.float32) * 0.2 + 1.0) if ng else None
    cos, sin = rope_table(L + 3, d, device="cuda") if rotate else (None, None)
    out = ja.qkv_prologue(P, dP, H, wq, wk, ng, 1e-6, cos, sin)
    torch.cuda.synchronize()
    ref = qkv_prologue(P.cpu(), dP.cpu(), H, d,
                       None if wq is None else wq.cpu(), None if wk is None else wk.cpu(),
                       ng or 0, 1e-6,
                       None if cos is None else cos[:L].cpu(), None if sin is None else sin[:L].cpu())
    for name, o, r in zip(("q", "k", "v", "dq", "dk", "dv"), out, ref):
        close_bf16(o, r, name)
    # v is a pure layout change: bit-exact
    assert torch.equal(out[2], P[:, :, 2 * C:].reshape(B, L, H, d).transpose(1, 2))
    assert torch.equal(out[5], dP[:, :, 2 * C:].reshape(B, L, H, d).transpose(1, 2))


def test_prologue_then_attention_jvp():
    # Layer chain: projections of (x, dx) -> prologue (QK-norm, RoPE, their
    # tangents) -> masked attention JVP, against the chained float64 oracles.
    T, F, chunk, H, d = 64, 4, 1, 2, 128
    spec = MaskSpec(TEACHER_FORCING, T, F, chunk)
    L, C = spec.length, H * d
    P = randn(5, (1, L, 3 * C), std=2.0)
    dP = randn(6, (1, L, 3 * C), std=0.1)
    wq = randn(7, (C,), torch.float32) * 0.2 + 1.0
    wk = randn(8, (C,), torch.float32) * 0.2 + 1.0
    pos_cos, pos_sin = rope_table(L // 2, d, device="cuda")
    cos, sin = torch.cat([pos_cos, pos_cos]).contiguous(), torch.cat([pos_sin, pos_sin]).contiguous()
    q, k, v, dq, dk, dv = ja.qkv_prologue(P, dP, H, wq, wk, C, 1e-6, cos, sin)
    o, do, lse = ja.jvp_attn(q, k, v, dq, dk, dv, ja.Mask(ja.TEACHER_FORCING, T, F, chunk))
    ja.check_device_error()
    # oracle chain on the kernel's own prologue outputs (bf16 values) ...
    ro, rdo, rl = jvp_attention(q.cpu(), k.cpu(), v.cpu(), dq.cpu(), dk.cpu(), dv.cpu(), spec)
    for name, got, ref in (("o", o, ro), ("do", do, rdo)):
        g = got.double().cpu().numpy()
        assert np.abs(g - ref).max() <= 2e-2 * np.abs(ref).max(), name
        assert np.linalg.norm(g - ref) / np.linalg.norm(ref) <= 5e-3, name
    # ... and the prologue outputs themselves against the float64 prologue
    ref_in = qkv_prologue(P.cpu(), dP.cpu(), H, d, wq.cpu(), wk.cpu(), C, 1e-6, cos.cpu(),
                          sin.cpu())
    for name, got, ref in zip(("q", "k", "v", "dq", "dk", "dv"), (q, k, v, dq, dk, dv), ref_in):
        close_bf16(got, ref, name)


@pytest.mark.slow
def test_prologue_full_size_sampled_tokens():
    # The bench's shape: 65,520 tokens, 12 heads of 128, norm over all 1,536
    # channels, RoPE; sampled tokens against the oracle.
    from attention_jvp_continuous_b200.inputs import sample_rows
    B, L, H, d = 1, 65520, 12, 128
    C = H * d
    P = randn(20, (B, L, 3 * C), std=2.0)
    dP = randn(21, (B, L, 3 * C), std=0.1)
    wq = randn(22, (C,), torch.float32) * 0.2 + 1.0
    wk = randn(23, (C,), torch.float32) * 0.2 + 1.0
    cos, sin = rope_table(L, d, device="cuda")
    out = ja.qkv_prologue(P, dP, H, wq, wk, C, 1e-6, cos, sin)
    torch.cuda.synchronize()
    rows = torch.from_numpy(sample_rows(L, 48, seed=3))
    ref = qkv_prologue(P[:, rows].cpu(), dP[:, rows].cpu(), H, d, wq.cpu(), wk.cpu(), C, 1e-6,
                       cos[rows.cuda()].cpu(), sin[rows.cuda()].cpu())
    for name, o, r in zip(("q", "k", "v", "dq", "dk", "dv"), out, ref):
        close_bf16(o[:, :, rows.cuda()], r, name)
