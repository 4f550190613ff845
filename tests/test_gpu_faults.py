"""Failure detection on the GPU without faulting it: every wait inside the
tensor-core kernels (attention JVP, backward, cache attention) is bounded.
With the stall-test switch on, each launch's MMA warp first waits on a
barrier phase that nothing completes; after the (short) wait limit it
records a timeout in the device error word and aborts, the other roles see
the abort flag and end their own waits, every role drains its own copies and
MMAs, the tensor memory is freed and the kernel exits. The host reads the
error, and the same context then computes correct results again."""
import numpy as np
import pytest
import torch

import attention_jvp_continuous_b200 as ja
from attention_jvp_continuous_b200 import _lib
from attention_jvp_continuous_b200.inputs import Workload, make_inputs
from oracle import MaskSpec, jvp_attention

pytestmark = pytest.mark.gpu

LIMIT_NS = 200_000  # 0.2 ms: far above any wait of a healthy launch of these sizes


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from attention_jvp_continuous_b200 import build
    build.build()


def _timeout_then_recover(run, check):
    ja.check_device_error()  # start clean
    try:
        ja.set_wait_limit(LIMIT_NS)
        ja.set_stall_test(True)
        run()
        with pytest.raises(ja.JvpAttnError) as e:
            ja.check_device_error()
        assert e.value.code == _lib.JVP_ERR_DEVICE_TIMEOUT
    finally:
        ja.set_stall_test(False)
        ja.set_wait_limit(0)
    ja.check_device_error()  # the word was cleared by the read
    check(run())
    ja.check_device_error()


def test_jvp_wait_timeout_is_reported_and_context_recovers():
    w = Workload("fault_tf", 1, 2, 128, ja.TEACHER_FORCING, 100, 3, 1, "bf16", 0.1)
    mask = ja.Mask(w.mode, w.tokens_per_frame, w.n_frames, w.chunk)
    inputs, _ = make_inputs(w, device="cpu")
    dev = [t.cuda() for t in inputs]
    ref = jvp_attention(*inputs, MaskSpec(w.mode, w.tokens_per_frame, w.n_frames, w.chunk))

    def check(res):
        for got, want in zip(res[:2], ref[:2]):
            g = got.float().cpu().numpy().astype(np.float64)
            assert np.linalg.norm(g - want) <= 5e-3 * np.linalg.norm(want)

    _timeout_then_recover(lambda: ja.jvp_attn(*dev, mask), check)


def test_tiny_wait_limit_never_breaks_a_launch():
    # A 1 ns limit makes waits that are not satisfied at once give up, or
    # not, depending on timing; either way the launch ends, and the error
    # word holds a timeout or nothing.
    w = Workload("fault_tiny", 1, 2, 128, ja.TEACHER_FORCING, 100, 3, 1, "bf16", 0.1)
    mask = ja.Mask(w.mode, w.tokens_per_frame, w.n_frames, w.chunk)
    inputs, _ = make_inputs(w, device="cpu")
    dev = [t.cuda() for t in inputs]
    ja.check_device_error()
    try:
        ja.set_wait_limit(1)
        for _ in range(3):
            ja.jvp_attn(*dev, mask)
            try:
                ja.check_device_error()
            except ja.JvpAttnError as e:
                assert e.code == _lib.JVP_ERR_DEVICE_TIMEOUT
    finally:
        ja.set_wait_limit(0)
    ja.check_device_error()


def test_backward_and_cache_waits_are_bounded_too():
    from oracle import cache_attention
    from oracle.attention_backward import attention_backward
    w = Workload("fault_bwd", 1, 2, 128, ja.TEACHER_FORCING, 100, 3, 1, "bf16", 1.0)
    spec = MaskSpec(w.mode, w.tokens_per_frame, w.n_frames, w.chunk)
    mask = ja.Mask(w.mode, w.tokens_per_frame, w.n_frames, w.chunk)
    (q, k, v, g, *_), _ = make_inputs(w, device="cpu")
    dq, dk, dv, dg = (t.cuda() for t in (q, k, v, g))
    o, _, lse = ja.jvp_attn(dq, dk, dv, *(torch.zeros_like(t) for t in (dq, dk, dv)), mask)
    ja.check_device_error()
    ref = attention_backward(q, k, v, g, spec)

    def check_bwd(grads):
        for got, want in zip(grads, ref):
            gg = got.float().cpu().numpy().astype(np.float64)
            assert np.linalg.norm(gg - want) <= 1e-2 * np.linalg.norm(want)

    _timeout_then_recover(lambda: ja.attn_bwd(dq, dk, dv, o, dg, lse, mask), check_bwd)

    Lk = 500
    ref_o, _ = cache_attention(q, k, v, Lk)

    def check_cache(res):
        gg = res[0].float().cpu().numpy().astype(np.float64)
        assert np.linalg.norm(gg - ref_o) <= 5e-3 * np.linalg.norm(ref_o)

    _timeout_then_recover(lambda: ja.cache_attn(dq, dk, dv, Lk), check_cache)
    # split-K cache launch (short query chunk over a long prefix) as well
    qs = dq[:, :, :96].contiguous()
    ref_s, _ = cache_attention(q[:, :, :96], k, v, 600)

    def check_split(res):
        gg = res[0].float().cpu().numpy().astype(np.float64)
        assert np.linalg.norm(gg - ref_s) <= 5e-3 * np.linalg.norm(ref_s)

    _timeout_then_recover(lambda: ja.cache_attn(qs, dk, dv, 600), check_split)
