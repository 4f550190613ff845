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
