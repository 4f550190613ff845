"""GPU parity: the CUDA kernels, called through the C ABI, against the
float64 oracle on the same seeded inputs.

Tolerances (written here, applied to O and dO separately):
  bf16 inputs: max|err| <= 2e-2 * max|ref|  and  ||err||_2 <= 5e-3 ||ref||_2
  fp32 inputs: ||err||_2 <= 1e-4 ||ref||_2
  LSE:         max|err| <= 1e-3 (bf16), 1e-5 (fp32)
"""
import numpy as np
import pytest
import torch

import attention_jvp_continuous_b200 as ja
from attention_jvp_continuous_b200.inputs import WORKLOADS, Workload, make_inputs
from oracle import MaskSpec, jvp_attention

pytestmark = pytest.mark.gpu

BF16_MAXABS, BF16_RELL2, FP32_RELL2 = 2e-2, 5e-3, 1e-4


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from attention_jvp_continuous_b200 import build
    build.build()


def spec_of(w):
    return MaskSpec(w.mode, w.tokens_per_frame, w.n_frames, w.chunk)


def mask_of(w):
    return ja.Mask(w.mode, w.tokens_per_frame, w.n_frames, w.chunk)


def run_gpu(w, inputs):
    o, do, lse = ja.jvp_attn(*inputs, mask_of(w))
    ja.check_device_error()
    return o, do, lse


def compare(got, ref, dtype, what):
    g = got.detach().float().cpu().numpy().astype(np.float64)
    err = g - ref
    rel = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-30)
    mx = np.abs(err).max() / max(np.abs(ref).max(), 1e-30)
    if dtype == "fp32":
        assert rel <= FP32_RELL2, f"{what}: rel L2 {rel:.3e}"
    else:
        assert rel <= BF16_RELL2, f"{what}: rel L2 {rel:.3e}"
        assert mx <= BF16_MAXABS, f"{what}: max-abs/max|ref| {mx:.3e}"
    return rel, mx


def check_full(w, seed=0):
    inputs, _ = make_inputs(w, device="cpu", seed=seed)
    ref = jvp_attention(*inputs, spec_of(w))
    dev = [t.cuda() for t in inputs]
    o, do, lse = run_gpu(w, dev)
    compare(o, ref[0], w.dtype, "O")
    compare(do, ref[1], w.dtype, "dO")
    lse_tol = 1e-5 if w.dtype == "fp32" else 1e-3
    assert np.abs(lse.cpu().numpy() - ref[2]).max() <= lse_tol
    return o, do, lse


def test_tiny_fp32_teacher_forcing():
    check_full(WORKLOADS["tiny_tf"])


SMALL_BF16 = [
    # several query tiles, ragged tails, every mask mode, d = 128 (tensor cores)
    Workload("tf_small", 2, 3, 128, ja.TEACHER_FORCING, 200, 3, 1, "bf16", 0.1),
    Workload("tf_chunk_small", 1, 2, 128, ja.TEACHER_FORCING, 100, 5, 2, "bf16", 0.1),
    Workload("frame_small", 1, 3, 128, ja.FRAME_CAUSAL, 130, 5, 1, "bf16", 0.1),
    Workload("chunk_small", 2, 1, 128, ja.CHUNK_CAUSAL, 70, 7, 3, "bf16", 0.1),
    Workload("dense_small", 1, 2, 128, ja.DENSE, 64, 4, 1, "bf16", 0.1),
    Workload("tiny_L", 1, 1, 128, ja.TEACHER_FORCING, 5, 2, 1, "bf16", 0.1),
    Workload("unit_tangent", 1, 2, 128, ja.TEACHER_FORCING, 96, 4, 1, "bf16", 1.0),
    Workload("head_scale", 1, 4, 128, ja.TEACHER_FORCING, 150, 3, 1, "bf16", 0.1,
             head_scale=(0.5, 2.0)),
]


@pytest.mark.parametrize("w", SMALL_BF16, ids=lambda w: w.name)
def test_tensor_core_small(w):
    check_full(w)


@pytest.mark.parametrize("w", [
    Workload("simt_bf16_d64", 1, 2, 64, ja.TEACHER_FORCING, 40, 3, 1, "bf16", 0.1),
    Workload("simt_fp32_d128", 1, 2, 128, ja.FRAME_CAUSAL, 50, 4, 1, "fp32", 1.0),
    Workload("simt_fp32_d32", 1, 1, 32, ja.CHUNK_CAUSAL, 33, 5, 2, "fp32", 1.0),
], ids=lambda w: w.name)
def test_cuda_core_path(w):
    check_full(w)


def test_more_items_than_sms():
    # 2 * 90 heads x 2 query tiles = 360 work items > 148 SMs
    w = Workload("many_heads", 2, 90, 128, ja.TEACHER_FORCING, 64, 2, 1, "bf16", 0.1)
    check_full(w)


def test_deterministic():
    w = SMALL_BF16[0]
    inputs, _ = make_inputs(w, device="cuda")
    a = run_gpu(w, inputs)
    b = run_gpu(w, inputs)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_zero_tangent_exact_and_value_direction():
    w = SMALL_BF16[0]
    (q, k, v, dq, dk, dv), _ = make_inputs(w, device="cuda")
    z = torch.zeros_like(q)
    o, do, _ = run_gpu(w, (q, k, v, z, z, z))
    assert torch.count_nonzero(do) == 0
    # tangent (0, 0, V): dO equals O (the same products in the same order)
    o2, do2, _ = run_gpu(w, (q, k, v, z, z, v))
    assert torch.equal(o2, o)
    err = (do2.float() - o.float()).abs().max()
    assert err <= 1e-2 * o.float().abs().max()


def test_clean_rows_have_zero_tangent_under_teacher_forcing():
    w = SMALL_BF16[0]
    (q, k, v, dq, dk, dv), _ = make_inputs(w, device="cuda")
    FT = w.tokens_per_frame * w.n_frames
    for t in (dq, dk, dv):
        t[:, :, :FT] = 0
    _, do, _ = run_gpu(w, (q, k, v, dq, dk, dv))
    assert torch.count_nonzero(do[:, :, :FT]) == 0
    assert do[:, :, FT:].abs().max() > 0


def parity_rows(w, n_random=96):
    """Seeded random rows plus the structural edges of the mask."""
    L, T, F = w.L, w.tokens_per_frame, w.n_frames
    rng = np.random.default_rng(1234)
    rows = set(rng.choice(L, size=n_random, replace=False).tolist())
    FT = T * F
    for base in ([0, FT] if w.mode == ja.TEACHER_FORCING else [0]):
        for f in (0, 1, F // 2, F - 1):
            rows.update({base + f * T, base + f * T + T - 1})
    rows.update({L - 1, L - 2, 127, 128})
    return np.array(sorted(r for r in rows if 0 <= r < L))


@pytest.mark.slow
@pytest.mark.parametrize("name", ["frame_causal", "tf", "chunk_tf", "tf_long"])
def test_full_size_sampled_rows(name):
    w = WORKLOADS[name]
    inputs, _ = make_inputs(w, device="cuda")
    o, do, lse = run_gpu(w, inputs)
    rows = parity_rows(w)
    host = [t.cpu() for t in inputs]
    ref = jvp_attention(*host, spec_of(w), rows=rows)
    idx = torch.as_tensor(rows)
    compare(o[:, :, idx], ref[0], "bf16", "O")
    compare(do[:, :, idx], ref[1], "bf16", "dO")
    assert np.abs(lse[:, :, idx].cpu().numpy() - ref[2]).max() <= 1e-3
    assert torch.isfinite(o).all() and torch.isfinite(do).all()
