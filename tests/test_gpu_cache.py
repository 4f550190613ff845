"""GPU parity of the key/value-cache path against the float64 oracle:
jvp_attn_rope_copy (cache appends, with and without rotary embedding) and
jvp_attn_cache_fwd (chunk attention over the exposed cache prefix, with and
without key splits), a chunk-by-chunk rollout that reproduces the packed
teacher-forcing forward, and sampled rows of the full-size chunk."""
import numpy as np
import pytest
import torch

import attention_jvp_continuous_b200 as ja
from attention_jvp_continuous_b200.inputs import rope_table, sample_rows
from oracle import cache_attention, cache_attention_head, rope_rows

pytestmark = pytest.mark.gpu

MAXABS, RELL2, LSE_ABS = 2e-2, 5e-3, 1e-3  # bf16 tolerances of the forward


def randn(seed, shape, dtype=torch.bfloat16, std=1.0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(dtype).cuda()


def check_close(out, ref, what):
    out = out.double().cpu().numpy()
    err = np.abs(out - ref)
    assert err.max() <= MAXABS * np.abs(ref).max(), (what, err.max())
    rel = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert rel <= RELL2, (what, rel)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rotate", [False, True])
def test_rope_copy_matches_oracle(dtype, rotate):
    B, H, Ls, Ld, d = 2, 3, 50, 80, 128
    src = randn(1, (B, H, Ls, d), dtype)
    dst = randn(2, (B, H, Ld, d), dtype)
    before = dst.clone()
    rows, s0, d0, r0 = 37, 5, 20, 11
    cos, sin = rope_table(64, d, pos0=100, device="cuda")
    if rotate:
        ja.rope_copy(src, dst, rows, s0, d0, cos, sin, rope_row0=r0)
    else:
        ja.rope_copy(src, dst, rows, s0, d0)
    torch.cuda.synchronize()
    got = dst[:, :, d0:d0 + rows]
    if not rotate:
        assert torch.equal(got, src[:, :, s0:s0 + rows])
    else:
        ref = rope_rows(src[:, :, s0:s0 + rows].cpu(), cos[r0:r0 + rows].cpu(),
                        sin[r0:r0 + rows].cpu())
        g = got.double().cpu().numpy()
        half_ulp = 2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -23
        tol = half_ulp * 1.01 * np.abs(ref) + 1e-6 * np.abs(src.double().cpu().numpy()).max()
        assert np.all(np.abs(g - ref) <= tol)
    # rows outside the destination range are untouched
    assert torch.equal(dst[:, :, :d0], before[:, :, :d0])
    assert torch.equal(dst[:, :, d0 + rows:], before[:, :, d0 + rows:])


def test_rope_copy_in_place_and_inverse():
    B, H, L, d = 1, 2, 33, 128
    x = randn(3, (B, H, L, d), torch.float32)
    y = x.clone()
    cos, sin = rope_table(L, d, device="cuda")
    ja.rope_copy(y, y, L, cos=cos, sin=sin)
    ja.rope_copy(y, y, L, cos=cos, sin=-sin)
    torch.cuda.synchronize()
    assert torch.allclose(y, x, atol=1e-5, rtol=1e-5)


CASES = [  # B, H, Lq, Lk, Lcache
    (1, 2, 200, 700, 1024),      # ragged query and key tails, split keys
    (1, 1, 128, 128, 128),       # one tile
    (2, 3, 5, 1000, 1003),       # tiny chunk, many splits
    (1, 2, 1560, 3120, 4000),    # one frame over two frames of context
    (1, 4, 4096, 2000, 2048),    # enough query tiles for no split
    (1, 149, 128, 2000, 2000),   # one whole wave of 148 items, one leftover cut into pieces
    (1, 100, 384, 1000, 1024),   # two whole waves, four leftover items cut in two
]


@pytest.mark.parametrize("B,H,Lq,Lk,Lcache", CASES)
def test_cache_attn_matches_oracle(B, H, Lq, Lk, Lcache):
    q = randn(10, (B, H, Lq, 128))
    k = randn(11, (B, H, Lcache, 128))
    v = randn(12, (B, H, Lcache, 128))
    # cache rows past the exposed prefix must not be read
    k[:, :, Lk:] = float("nan")
    v[:, :, Lk:] = float("nan")
    o, lse = ja.cache_attn(q, k, v, Lk)
    ja.check_device_error()
    ref_o, ref_lse = cache_attention(q.cpu(), k.cpu(), v.cpu(), Lk)
    check_close(o, ref_o, "o")
    assert np.abs(lse.double().cpu().numpy() - ref_lse).max() <= LSE_ABS


def test_cache_attn_is_deterministic():
    q = randn(20, (1, 2, 300, 128))
    k = randn(21, (1, 2, 5000, 128))
    v = randn(22, (1, 2, 5000, 128))
    o1, l1 = ja.cache_attn(q, k, v, 4999)
    o2, l2 = ja.cache_attn(q, k, v, 4999)
    ja.check_device_error()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("prerope", [False, True])
def test_rollout_reproduces_packed_teacher_forcing(prerope):
    # Generate the noisy chunks of a teacher-forcing batch one by one against
    # a cache: the clean history is committed chunk by chunk, the current
    # noisy chunk's keys are written at its cache position, and each chunk's
    # output must equal the packed forward's rows (keys rotated by position;
    # post-RoPE caching rotates at the append, pre-RoPE caching stores raw
    # keys and rotates the exposed prefix into a working buffer).
    T, F, chunk, H = 96, 5, 1, 2
    S, FT = T * chunk, T * F
    L = 2 * FT
    q = randn(30, (1, H, L, 128))
    k = randn(31, (1, H, L, 128))
    v = randn(32, (1, H, L, 128))
    cos, sin = rope_table(FT, 128, device="cuda")
    # packed reference: clean and noisy token i share the position of frame
    # index i mod FT
    pos_cos = torch.cat([cos, cos]).contiguous()
    pos_sin = torch.cat([sin, sin]).contiguous()
    kr = torch.empty_like(k)
    ja.rope_copy(k, kr, L, cos=pos_cos, sin=pos_sin)
    mask = ja.Mask(ja.TEACHER_FORCING, T, F, chunk)
    z = torch.zeros_like(q)
    o_ref, _, lse_ref = ja.jvp_attn(q, kr, v, z, z, z, mask)
    kc = torch.zeros((1, H, FT, 128), dtype=k.dtype, device="cuda")
    vc = torch.zeros_like(kc)
    work = torch.zeros_like(kc)
    for c0 in range(0, FT, S):
        c1 = c0 + S
        # current chunk at its position (uncommitted), then attend
        if prerope:
            ja.rope_copy(k, kc, S, FT + c0, c0)                       # raw noisy keys
            ja.rope_copy(kc, work, c1, 0, 0, cos=cos, sin=sin)       # rotate the prefix
            keys = work
        else:
            ja.rope_copy(k, kc, S, FT + c0, c0, cos=cos, sin=sin, rope_row0=c0)
            keys = kc
        ja.rope_copy(v, vc, S, FT + c0, c0)
        o, lse = ja.cache_attn(q[:, :, FT + c0:FT + c1].contiguous(), keys, vc, c1)
        torch.cuda.synchronize()
        ref = o_ref[:, :, FT + c0:FT + c1].double().cpu().numpy()
        check_close(o, ref, f"chunk {c0 // S}")
        assert (lse - lse_ref[:, :, FT + c0:FT + c1]).abs().max().item() <= LSE_ABS
        # commit the clean chunk (the context of the next chunk)
        if prerope:
            ja.rope_copy(k, kc, S, c0, c0)
        else:
            ja.rope_copy(k, kc, S, c0, c0, cos=cos, sin=sin, rope_row0=c0)
        ja.rope_copy(v, vc, S, c0, c0)
    ja.check_device_error()


@pytest.mark.slow
def test_cache_attn_full_size_sampled_rows():
    # The last chunk of a 21-frame rollout at 1560 tokens per frame: 1560
    # queries over 32,760 cached keys, 12 heads.
    B, H, Lq, Lk = 1, 12, 1560, 32760
    q = randn(40, (B, H, Lq, 128))
    k = randn(41, (B, H, Lk, 128))
    v = randn(42, (B, H, Lk, 128))
    o, lse = ja.cache_attn(q, k, v, Lk)
    ja.check_device_error()
    rows = sample_rows(Lq, 24, seed=7)
    qh, kh, vh = q.cpu(), k.cpu(), v.cpu()
    for h in (0, 5, 11):
        ro, rl = cache_attention_head(qh[0, h, rows], kh[0, h], vh[0, h], Lk)
        check_close(o[0, h, rows], ro, f"head {h}")
        assert np.abs(lse[0, h, rows].double().cpu().numpy() - rl).max() <= LSE_ABS
