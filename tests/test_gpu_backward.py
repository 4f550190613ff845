"""GPU parity of the masked attention backward (jvp_attn_bwd) against the
float64 oracle, plus full-size checks that need no oracle: the adjoint
identity between the library's own JVP and backward kernels, and gradient
invariants.

Tolerances (bf16 inputs, fp32 accumulation, bf16 outputs), per gradient:
  max|err| <= 2e-2 * max|ref|  and  ||err||_2 <= 1e-2 ||ref||_2
The backward rounds two operands to bf16 per pair (P and dS, where dS holds
a difference dP - D), so its relative L2 bar is twice the forward's.
"""
import numpy as np
import pytest
import torch

import attention_jvp_continuous_b200 as ja
from attention_jvp_continuous_b200.inputs import WORKLOADS, Workload, make_inputs
from oracle import MaskSpec
from oracle.attention_backward import attention_backward

pytestmark = pytest.mark.gpu

MAXABS, RELL2 = 2e-2, 1e-2


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from attention_jvp_continuous_b200 import build
    build.build()


def mask_of(w):
    return ja.Mask(w.mode, w.tokens_per_frame, w.n_frames, w.chunk)


def forward_and_backward(w, q, k, v, g):
    z = torch.zeros_like(q)
    o, _, lse = ja.jvp_attn(q, k, v, z, z, z, mask_of(w))
    grads = ja.attn_bwd(q, k, v, o, g, lse, mask_of(w))
    ja.check_device_error()
    return o, lse, grads


def compare(got, ref, what):
    g = got.float().cpu().numpy().astype(np.float64)
    err = g - ref
    rel = np.linalg.norm(err) / np.linalg.norm(ref)
    mx = np.abs(err).max() / np.abs(ref).max()
    assert rel <= RELL2, f"{what}: rel L2 {rel:.3e}"
    assert mx <= MAXABS, f"{what}: max-abs/max|ref| {mx:.3e}"


CASES = [
    Workload("bwd_tf", 1, 2, 128, ja.TEACHER_FORCING, 200, 3, 1, "bf16", 1.0),
    Workload("bwd_tf_chunk", 1, 2, 128, ja.TEACHER_FORCING, 100, 5, 2, "bf16", 1.0),
    Workload("bwd_frame", 2, 1, 128, ja.FRAME_CAUSAL, 130, 5, 1, "bf16", 1.0),
    Workload("bwd_chunk", 1, 2, 128, ja.CHUNK_CAUSAL, 70, 7, 3, "bf16", 1.0),
    Workload("bwd_dense", 1, 2, 128, ja.DENSE, 64, 4, 1, "bf16", 1.0),
    Workload("bwd_tiny", 1, 1, 128, ja.TEACHER_FORCING, 5, 2, 1, "bf16", 1.0),
    Workload("bwd_medium", 1, 2, 128, ja.TEACHER_FORCING, 400, 4, 1, "bf16", 1.0),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_backward_matches_oracle(w):
    (q, k, v, g, _, _), _ = make_inputs(w, device="cpu")
    spec = MaskSpec(w.mode, w.tokens_per_frame, w.n_frames, w.chunk)
    ref = attention_backward(q, k, v, g, spec)
    _, _, grads = forward_and_backward(w, *(t.cuda() for t in (q, k, v, g)))
    for name, got, want in zip(("gQ", "gK", "gV"), grads, ref):
        compare(got, want, name)


@pytest.mark.parametrize("w", [
    # 2 x 32 heads x 5 query tiles (and 5 key tiles) = 320 work items per
    # pass, more than the 148 SMs: persistent CTAs carry over from one item
    # to the next in both passes. 600 tokens end in a ragged 88-row tile.
    Workload("bwd_many_items_tf", 2, 32, 128, ja.TEACHER_FORCING, 100, 3, 1, "bf16", 1.0),
    Workload("bwd_many_items_chunk", 2, 40, 128, ja.CHUNK_CAUSAL, 90, 6, 2, "bf16", 1.0),
], ids=lambda w: w.name)
def test_backward_more_items_than_sms(w):
    n_items = w.B * w.H * -(-w.L // 128)
    assert n_items > 148
    (q, k, v, g, _, _), _ = make_inputs(w, device="cpu")
    spec = MaskSpec(w.mode, w.tokens_per_frame, w.n_frames, w.chunk)
    ref = attention_backward(q, k, v, g, spec)
    _, _, grads = forward_and_backward(w, *(t.cuda() for t in (q, k, v, g)))
    for name, got, want in zip(("gQ", "gK", "gV"), grads, ref):
        compare(got, want, name)


def parity_rows(w, n_random=96):
    """Seeded random query rows plus the mask's frame, half and tile edges."""
    L, T, F = w.L, w.tokens_per_frame, w.n_frames
    rng = np.random.default_rng(1234)
    rows = set(rng.choice(L, size=n_random, replace=False).tolist())
    FT = T * F
    for base in ([0, FT] if w.mode == ja.TEACHER_FORCING else [0]):
        for f in (0, 1, F // 2, F - 1):
            rows.update({base + f * T, base + f * T + T - 1})
    rows.update({L - 1, L - 2, 127, 128})
    return np.array(sorted(r for r in rows if 0 <= r < L))


def full_size_case(name):
    w = WORKLOADS[name]
    (q, k, v, _, _, _), _ = make_inputs(w, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(99)
    g = torch.randn(q.shape, generator=gen, device="cuda").to(q.dtype)
    _, _, grads = forward_and_backward(w, q, k, v, g)
    spec = MaskSpec(w.mode, w.tokens_per_frame, w.n_frames, w.chunk)
    return w, spec, (q, k, v, g), grads


@pytest.mark.slow
@pytest.mark.parametrize("name", ["frame_causal", "tf", "chunk_tf", "tf_long"])
def test_full_size_gq_on_sampled_rows(name):
    # The launch the backward bench times (all heads, full length); gQ of a
    # row depends only on that row's cotangent, so the oracle restricted to
    # the sampled rows gives gQ exactly there.
    w, spec, ins, (gq, _, _) = full_size_case(name)
    rows = parity_rows(w)
    ref_gq = attention_backward(*(t.cpu() for t in ins), spec, rows=rows)[0]
    idx = torch.as_tensor(rows, device=gq.device)
    compare(gq[:, :, idx], ref_gq[:, :, rows], "gQ")


@pytest.mark.slow
@pytest.mark.parametrize("name,h", [("tf", 7), ("chunk_tf", 2)])
def test_full_size_one_head_all_gradients(name, h):
    # Key and value gradients gather over every query row that sees a key,
    # so one head of the full launch is compared whole: gQ, gK and gV on
    # all 65,520 rows (about a minute of float64 per head).
    from oracle.attention_backward import attention_backward_head
    w, spec, ins, grads = full_size_case(name)
    ref = attention_backward_head(*(t[0, h].cpu() for t in ins), spec)
    for what, got, want in zip(("gQ", "gK", "gV"), grads, ref):
        compare(got[0, h], want, what)


def test_backward_deterministic():
    w = CASES[0]
    (q, k, v, g, _, _), _ = make_inputs(w, device="cuda")
    a = forward_and_backward(w, q, k, v, g)[2]
    b = forward_and_backward(w, q, k, v, g)[2]
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["tf", "chunk_tf"])
def test_full_size_adjoint_and_invariants(name):
    # <G, J t> from the JVP kernel equals <J^T G, t> from the backward
    # kernels; value gradients sum to the total cotangent; key gradients
    # sum to zero.
    w = WORKLOADS[name]
    (q, k, v, dq, dk, dv), _ = make_inputs(w, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(99)
    g = torch.randn(q.shape, generator=gen, device="cuda").to(q.dtype)
    o, d_o, lse = ja.jvp_attn(q, k, v, dq, dk, dv, mask_of(w))
    gq, gk, gv = ja.attn_bwd(q, k, v, o, g, lse, mask_of(w))
    ja.check_device_error()
    f = lambda x: x.double()
    lhs = (f(g) * f(d_o)).sum().item()
    rhs = ((f(gq) * f(dq)).sum() + (f(gk) * f(dk)).sum() + (f(gv) * f(dv)).sum()).item()
    scale = (f(g).abs() * f(d_o).abs()).sum().item()
    assert abs(lhs - rhs) <= 2e-3 * scale, (lhs, rhs, scale)
    tot_g = f(g).sum(dim=2)
    assert ((f(gv).sum(dim=2) - tot_g).abs().max() <= 2e-2 * tot_g.abs().max() + 1.0).item()
    assert ((f(gk).sum(dim=2)).abs().max() <= 2e-2 * f(gk).abs().sum(dim=2).max()).item()
    for t in (gq, gk, gv):
        assert torch.isfinite(t).all()
