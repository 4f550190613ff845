"""The allocation-free entry point, jvp_attn_fwd_noalloc, against jvp_attn_fwd.

Some callers cannot let the library cudaMalloc its work-list buffer (their
device memory all belongs to their own pool, or their deployment forbids
device allocation after start-up). jvp_attn_fwd_noalloc keeps that list in
a fixed array inside the library instead. This file is collected last so that a failure here leaves
every other test already run.
"""
import ctypes

import numpy as np
import pytest
import torch

import attention_jvp_continuous_b200 as ja
from attention_jvp_continuous_b200 import _lib
from attention_jvp_continuous_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from attention_jvp_continuous_b200 import build
    build.build()


def call(fn, q, k, v, dq, dk, dv, o, do, lse, w):
    B, H, L, d = q.shape
    return fn(*[ctypes.c_void_p(t.data_ptr()) for t in (q, k, v, dq, dk, dv, o, do)],
              ctypes.cast(lse.data_ptr(), ctypes.POINTER(ctypes.c_float)),
              B, H, L, d, _lib.JVP_BF16,
              _lib.MaskDesc(w.mode, w.tokens_per_frame, w.n_frames, w.chunk), 0.0,
              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def close(a, b):
    # the bf16 parity tolerance used for the tensor-core kernel
    a, b = a.float().cpu().numpy().astype(np.float64), b.float().cpu().numpy().astype(np.float64)
    err = a - b
    assert np.linalg.norm(err) <= 5e-3 * np.linalg.norm(b)
    assert np.abs(err).max() <= 2e-2 * np.abs(b).max()


def test_noalloc_matches_allocating_entry_on_two_calls_in_a_row():
    lib = _lib.lib()
    cases = [
        Workload("na_tf", 1, 3, 128, ja.TEACHER_FORCING, 150, 3, 1, "bf16", 0.1),
        Workload("na_frame", 2, 2, 128, ja.FRAME_CAUSAL, 200, 4, 1, "bf16", 0.1),
    ]
    for w in cases:  # two calls in a row; the second rewrites the shared array
        ins, _ = make_inputs(w, device="cuda")
        outs = []
        for fn in (lib.jvp_attn_fwd, lib.jvp_attn_fwd_noalloc):
            o, do = torch.empty_like(ins[0]), torch.empty_like(ins[0])
            lse = torch.empty(ins[0].shape[:3], dtype=torch.float32, device="cuda")
            assert call(fn, *ins, o, do, lse, w) == 0
            ja.check_device_error()
            outs.append((o, do, lse))
        (o1, do1, l1), (o2, do2, l2) = outs
        close(o2, o1)
        close(do2, do1)
        assert (l2 - l1).abs().max().item() <= 1e-3


def test_noalloc_rejects_oversized_work_list():
    lib = _lib.lib()
    fake = [0x1000] * 9  # never dereferenced: the size check comes first
    rc = lib.jvp_attn_fwd_noalloc(
        *[ctypes.c_void_p(x) for x in fake[:8]],
        ctypes.cast(ctypes.c_void_p(fake[8]), ctypes.POINTER(ctypes.c_float)),
        1, 1, 4096 * 513, 128, _lib.JVP_BF16, _lib.MaskDesc(ja.DENSE, 4096, 513, 1), 0.0, None)
    assert rc == _lib.JVP_ERR_TOO_LARGE


def _outputs_of(fn, ins, w):
    o, do = torch.empty_like(ins[0]), torch.empty_like(ins[0])
    lse = torch.empty(ins[0].shape[:3], dtype=torch.float32, device="cuda")
    assert call(fn, *ins, o, do, lse, w) == 0
    ja.check_device_error()
    return o, do, lse


def test_noalloc_list_kept_and_rewritten_across_masks():
    # Mask A, then B (longer, so its list overwrites more of the shared
    # array), then A twice: the third call must rewrite A's list, the fourth
    # reuses it without a copy. Every call is checked against jvp_attn_fwd.
    lib = _lib.lib()
    wa = Workload("na_a", 1, 2, 128, ja.TEACHER_FORCING, 120, 3, 1, "bf16", 0.1)
    wb = Workload("na_b", 1, 2, 128, ja.FRAME_CAUSAL, 300, 5, 1, "bf16", 0.1)
    ins = {w.name: make_inputs(w, device="cuda")[0] for w in (wa, wb)}
    ref = {w.name: _outputs_of(lib.jvp_attn_fwd, ins[w.name], w) for w in (wa, wb)}
    for w in (wa, wb, wa, wa):
        o, do, lse = _outputs_of(lib.jvp_attn_fwd_noalloc, ins[w.name], w)
        o1, do1, l1 = ref[w.name]
        close(o, o1)
        close(do, do1)
        assert (lse - l1).abs().max().item() <= 1e-3


def test_noalloc_refuses_a_capturing_stream():
    lib = _lib.lib()
    w = Workload("na_cap", 1, 1, 128, ja.TEACHER_FORCING, 64, 2, 1, "bf16", 0.1)
    ins, _ = make_inputs(w, device="cuda")
    o, do, lse = _outputs_of(lib.jvp_attn_fwd_noalloc, ins, w)  # first call: set-up
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=torch.cuda.Stream()):
        rc = call(lib.jvp_attn_fwd_noalloc, *ins, o, do, lse, w)
    assert rc == _lib.JVP_ERR_INVALID_ARG
    # nothing was recorded or left pending: a plain call still works
    o2, do2, l2 = _outputs_of(lib.jvp_attn_fwd_noalloc, ins, w)
    assert torch.equal(o2, o) and torch.equal(do2, do) and torch.equal(l2, lse)


def test_noalloc_at_its_largest_work_list():
    # 255 frames of 1560 tokens under the teacher-forcing mask: 795,600
    # tokens, whose work list takes 64,478 of the array's 65,472 words.
    # Sampled rows (frame and half edges included) against the float64
    # oracle; 260 frames (65,762 words) no longer fit.
    from oracle import MaskSpec, jvp_attention_head
    lib = _lib.lib()
    w = Workload("na_max", 1, 1, 128, ja.TEACHER_FORCING, 1560, 255, 1, "bf16", 0.1)
    ins, _ = make_inputs(w, device="cuda")
    o, do, lse = _outputs_of(lib.jvp_attn_fwd_noalloc, ins, w)
    FT = w.tokens_per_frame * w.n_frames
    rng = np.random.default_rng(5)
    rows = sorted(set(rng.choice(w.L, size=16, replace=False).tolist())
                  | {0, 1559, 1560, FT - 1, FT, FT + 1559, w.L - 1})
    spec = MaskSpec(w.mode, w.tokens_per_frame, w.n_frames, w.chunk)
    ref_o, ref_do, ref_lse = jvp_attention_head(*(t[0, 0].cpu() for t in ins), spec, rows=rows)
    idx = torch.as_tensor(rows, device="cuda")
    for got, want in ((o[0, 0, idx], ref_o), (do[0, 0, idx], ref_do)):
        g = got.float().cpu().numpy().astype(np.float64)
        assert np.linalg.norm(g - want) <= 5e-3 * np.linalg.norm(want)
        assert np.abs(g - want).max() <= 2e-2 * np.abs(want).max()
    assert np.abs(lse[0, 0, idx].cpu().numpy() - ref_lse).max() <= 1e-3
    fake = [0x1000] * 9  # never dereferenced: the size check comes first
    big = w.with_(n_frames=260)
    rc = lib.jvp_attn_fwd_noalloc(
        *[ctypes.c_void_p(x) for x in fake[:8]],
        ctypes.cast(ctypes.c_void_p(fake[8]), ctypes.POINTER(ctypes.c_float)),
        1, 1, big.L, 128, _lib.JVP_BF16,
        _lib.MaskDesc(big.mode, big.tokens_per_frame, big.n_frames, big.chunk), 0.0, None)
    assert rc == _lib.JVP_ERR_TOO_LARGE

