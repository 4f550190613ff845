"""The ranks' device barrier (jvp_attn_signal_barrier) on one GPU. Kernels
that wait on one another never run as separate launches here, so a second
rank is emulated by its flag words: the peer's arrival is written by the
host before the launch (the barrier must pass and must have announced this
rank's arrival in the peer's words), or never written (the bounded wait
must run out with JVP_ERR_DEVICE_TIMEOUT and leave the context usable)."""
import pytest
import torch

import attention_jvp_continuous_b200 as ja
from attention_jvp_continuous_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from attention_jvp_continuous_b200 import build
    build.build()


def test_single_rank_barrier_passes_every_epoch():
    f = torch.zeros(1, dtype=torch.int32, device="cuda")
    for epoch in range(1, 5):
        ja.signal_barrier([f], 0, epoch)
        ja.check_device_error()
        assert int(f.item()) == epoch


def test_two_ranks_peer_already_arrived():
    mine = torch.zeros(2, dtype=torch.int32, device="cuda")
    peer = torch.zeros(2, dtype=torch.int32, device="cuda")
    mine[1] = 3  # rank 1 reached epoch 3 already
    ja.signal_barrier([mine, peer], 0, 3)
    ja.check_device_error()
    assert mine.tolist() == [3, 3]
    assert peer.tolist() == [3, 0]  # this rank's arrival, announced to rank 1


def test_missing_rank_times_out_and_context_survives():
    mine = torch.zeros(2, dtype=torch.int32, device="cuda")
    peer = torch.zeros(2, dtype=torch.int32, device="cuda")
    ja.set_wait_limit(2_000_000)  # 2 ms
    try:
        ja.signal_barrier([mine, peer], 0, 1)  # rank 1 never arrives
        with pytest.raises(ja.JvpAttnError) as e:
            ja.check_device_error()
        assert e.value.code == ja._lib.JVP_ERR_DEVICE_TIMEOUT
    finally:
        ja.set_wait_limit(0)
    ja.check_device_error()  # the error word was cleared
    w = Workload("after_timeout", 1, 1, 128, ja.TEACHER_FORCING, 64, 2, 1, "bf16", 0.1)
    xs, _ = make_inputs(w, device="cuda")
    o, do, lse = ja.jvp_attn(*xs, ja.Mask(w.mode, w.tokens_per_frame, w.n_frames, w.chunk))
    ja.check_device_error()
    assert torch.isfinite(o).all() and torch.isfinite(do).all()
