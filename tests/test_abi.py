"""C-ABI tests that need no GPU: the library loads, exports every function
declared in include/jvp_attn.h, and rejects bad arguments with the
documented codes before touching a device."""
import ctypes
import os
import re

import pytest

import attention_jvp_continuous_b200 as ja
from attention_jvp_continuous_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from attention_jvp_continuous_b200 import build
    build.build()


def declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            with open(os.path.join(ROOT, "include", h)) as f:
                src = f.read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"\b(jvp_attn_\w+)\s*\(", src)
    return sorted(set(names))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert "jvp_attn_fwd" in names and len(names) >= 8
    lib = ctypes.CDLL(_lib.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(_lib.EXPORTS) <= set(names)


def test_version_and_strerror():
    assert _lib.lib().jvp_attn_version() == 100
    for code in range(0, -11, -1):
        s = _lib.strerror(code)
        assert s and s != "unknown error code"
    assert _lib.strerror(-999) == "unknown error code"


def call_fwd(ptr=0x1000, B=1, H=1, L=64, d=128, dtype=_lib.JVP_BF16,
             mask=(ja.TEACHER_FORCING, 8, 4, 1), scale=0.0, ptrs=None):
    p = [ptr] * 9 if ptrs is None else ptrs
    return _lib.lib().jvp_attn_fwd(
        *[ctypes.c_void_p(x) for x in p[:8]],
        ctypes.cast(ctypes.c_void_p(p[8]), ctypes.POINTER(ctypes.c_float)),
        B, H, L, d, dtype, _lib.MaskDesc(*mask), scale, None)


def test_null_pointer_rejected():
    ptrs = [0x1000] * 9
    ptrs[4] = 0
    assert call_fwd(ptrs=ptrs) == _lib.JVP_ERR_INVALID_ARG


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), _lib.JVP_ERR_INVALID_ARG),
    (dict(d=-4), _lib.JVP_ERR_INVALID_ARG),
    (dict(dtype=7), _lib.JVP_ERR_INVALID_ARG),
    (dict(mask=(9, 8, 4, 1)), _lib.JVP_ERR_INVALID_ARG),
    (dict(mask=(ja.TEACHER_FORCING, 0, 4, 1)), _lib.JVP_ERR_INVALID_ARG),
    (dict(mask=(ja.CHUNK_CAUSAL, 8, 4, 0), L=32), _lib.JVP_ERR_INVALID_ARG),
    (dict(L=63), _lib.JVP_ERR_SHAPE_MISMATCH),
    (dict(mask=(ja.FRAME_CAUSAL, 8, 4, 1), L=64), _lib.JVP_ERR_SHAPE_MISMATCH),
    (dict(d=100), _lib.JVP_ERR_UNSUPPORTED_HEAD_DIM),
    (dict(d=256, dtype=_lib.JVP_FP32), _lib.JVP_ERR_UNSUPPORTED_HEAD_DIM),
    (dict(ptr=0x1008), _lib.JVP_ERR_MISALIGNED),
    (dict(B=70000, H=70000, L=64), _lib.JVP_ERR_TOO_LARGE),
    (dict(scale=float("nan")), _lib.JVP_ERR_INVALID_ARG),
])
def test_argument_errors(kw, code):
    assert call_fwd(**kw) == code


def call_fwd_noalloc(ptr=0x1000, B=1, H=1, L=64, d=128, dtype=_lib.JVP_BF16,
                     mask=(ja.TEACHER_FORCING, 8, 4, 1), scale=0.0):
    return _lib.lib().jvp_attn_fwd_noalloc(
        *[ctypes.c_void_p(ptr) for _ in range(8)],
        ctypes.cast(ctypes.c_void_p(ptr), ctypes.POINTER(ctypes.c_float)),
        B, H, L, d, dtype, _lib.MaskDesc(*mask), scale, None)


@pytest.mark.parametrize("kw,code", [
    (dict(ptr=0), _lib.JVP_ERR_INVALID_ARG),
    (dict(B=0), _lib.JVP_ERR_INVALID_ARG),
    (dict(dtype=_lib.JVP_FP32), _lib.JVP_ERR_INVALID_ARG),       # tensor-core configuration only
    (dict(d=64), _lib.JVP_ERR_UNSUPPORTED_HEAD_DIM),
    (dict(scale=float("nan")), _lib.JVP_ERR_INVALID_ARG),
    (dict(L=63), _lib.JVP_ERR_SHAPE_MISMATCH),
    (dict(ptr=0x1008), _lib.JVP_ERR_MISALIGNED),
    (dict(B=70000, H=70000), _lib.JVP_ERR_TOO_LARGE),
    # a work list larger than the fixed array: rejected before any device work
    (dict(L=4096 * 513, mask=(ja.DENSE, 4096, 513, 1)), _lib.JVP_ERR_TOO_LARGE),
])
def test_noalloc_argument_errors(kw, code):
    assert call_fwd_noalloc(**kw) == code


def test_valid_call_without_gpu_fails_cleanly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    rc = call_fwd()
    assert rc in (_lib.JVP_ERR_LAUNCH_FAILED, _lib.JVP_ERR_UNSUPPORTED_DEVICE)


def test_python_wrapper_rejects_cpu_tensors():
    import torch
    x = torch.zeros(1, 1, 64, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ja.jvp_attn(x, x, x, x, x, x, ja.Mask(ja.TEACHER_FORCING, 8, 4, 1))


def test_error_type_carries_code():
    e = _lib.JvpAttnError(_lib.JVP_ERR_SHAPE_MISMATCH, "where")
    assert e.code == -2 and "mask descriptor" in str(e)


FAKE = 1 << 20  # 16-byte aligned dummy device address; never dereferenced on error paths


def call_cache(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, H=2, Lq=100, Lk=500, Lcache=512,
             d=128, dtype=_lib.JVP_BF16, scale=0.0)
    a.update(kw)
    fp = ctypes.POINTER(ctypes.c_float)
    return _lib.lib().jvp_attn_cache_fwd(a["q"], a["k"], a["v"], a["o"],
                                         ctypes.cast(a["lse"], fp), a["B"], a["H"], a["Lq"],
                                         a["Lk"], a["Lcache"], a["d"], a["dtype"], a["scale"],
                                         None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), _lib.JVP_ERR_INVALID_ARG),
    (dict(Lk=0), _lib.JVP_ERR_INVALID_ARG),
    (dict(Lk=513), _lib.JVP_ERR_INVALID_ARG),
    (dict(Lq=0), _lib.JVP_ERR_INVALID_ARG),
    (dict(dtype=_lib.JVP_FP32), _lib.JVP_ERR_INVALID_ARG),
    (dict(d=64), _lib.JVP_ERR_UNSUPPORTED_HEAD_DIM),
    (dict(scale=float("inf")), _lib.JVP_ERR_INVALID_ARG),
    (dict(o=FAKE + 8), _lib.JVP_ERR_MISALIGNED),
])
def test_cache_fwd_argument_errors(kw, code):
    assert call_cache(**kw) == code


def call_rope(**kw):
    a = dict(src=FAKE, dst=FAKE + (1 << 16), B=1, H=2, src_rows=64, dst_rows=128, rows=32,
             src_row0=0, dst_row0=96, d=128, dtype=_lib.JVP_BF16, cos=FAKE, sin=FAKE,
             rope_rows=40, rope_row0=8)
    a.update(kw)
    fp = ctypes.POINTER(ctypes.c_float)
    cvt = lambda x: ctypes.cast(x, fp) if x else None  # noqa: E731
    return _lib.lib().jvp_attn_rope_copy(a["src"], a["dst"], a["B"], a["H"], a["src_rows"],
                                         a["dst_rows"], a["rows"], a["src_row0"],
                                         a["dst_row0"], a["d"], a["dtype"], cvt(a["cos"]),
                                         cvt(a["sin"]), a["rope_rows"], a["rope_row0"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(dst_row0=97), _lib.JVP_ERR_INVALID_ARG),           # past the destination rows
    (dict(src_row0=33), _lib.JVP_ERR_INVALID_ARG),           # past the source rows
    (dict(rope_row0=9), _lib.JVP_ERR_INVALID_ARG),           # past the table
    (dict(sin=0), _lib.JVP_ERR_INVALID_ARG),                 # one table only
    (dict(d=100), _lib.JVP_ERR_INVALID_ARG),                 # bf16 rows of 16-byte vectors
    (dict(rows=-1), _lib.JVP_ERR_INVALID_ARG),
    (dict(dst=FAKE, dst_row0=90), _lib.JVP_ERR_INVALID_ARG),  # overlapping, not in place
    (dict(src=FAKE + 4), _lib.JVP_ERR_MISALIGNED),
    (dict(rows=0), _lib.JVP_OK),                              # nothing to do, no device touched
])
def test_rope_copy_argument_errors(kw, code):
    assert call_rope(**kw) == code


def call_bwd(B=1, H=2, L=64, d=128, dtype=_lib.JVP_BF16, mask=(ja.TEACHER_FORCING, 8, 4, 1),
             scale=0.0, scratch_len=None, ptrs=None):
    p = [FAKE] * 10 if ptrs is None else ptrs
    if scratch_len is None:
        scratch_len = max(_lib.lib().jvp_attn_bwd_scratch_len(B, H, L), 0)
    fp = ctypes.POINTER(ctypes.c_float)
    vp = [ctypes.c_void_p(x) for x in p]
    return _lib.lib().jvp_attn_bwd(*vp[:5], ctypes.cast(vp[5], fp), *vp[6:9],
                                   ctypes.cast(vp[9], fp), scratch_len, B, H, L, d, dtype,
                                   _lib.MaskDesc(*mask), scale, None)


@pytest.mark.parametrize("kw,code", [
    (dict(ptrs=[FAKE] * 9 + [0]), _lib.JVP_ERR_INVALID_ARG),            # no scratch
    (dict(ptrs=[FAKE] * 5 + [0] + [FAKE] * 4), _lib.JVP_ERR_INVALID_ARG),  # no lse
    (dict(L=0), _lib.JVP_ERR_INVALID_ARG),
    (dict(dtype=_lib.JVP_FP32), _lib.JVP_ERR_INVALID_ARG),               # bf16 only
    (dict(scale=float("inf")), _lib.JVP_ERR_INVALID_ARG),
    (dict(d=64), _lib.JVP_ERR_UNSUPPORTED_HEAD_DIM),
    (dict(L=63), _lib.JVP_ERR_SHAPE_MISMATCH),                           # mask covers 64
    (dict(mask=(9, 8, 4, 1)), _lib.JVP_ERR_INVALID_ARG),
    (dict(B=70000, H=70000), _lib.JVP_ERR_TOO_LARGE),
    (dict(scratch_len=2 * 2 * 128 - 1), _lib.JVP_ERR_INVALID_ARG),      # one float short
    (dict(ptrs=[FAKE] * 6 + [FAKE + 8] + [FAKE] * 3), _lib.JVP_ERR_MISALIGNED),
])
def test_bwd_argument_errors(kw, code):
    assert call_bwd(**kw) == code


def test_bwd_valid_call_without_gpu_fails_cleanly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert call_bwd() in (_lib.JVP_ERR_LAUNCH_FAILED, _lib.JVP_ERR_UNSUPPORTED_DEVICE)


def test_bwd_scratch_len():
    assert _lib.lib().jvp_attn_bwd_scratch_len(1, 12, 65520) == 2 * 12 * 65536
    assert _lib.lib().jvp_attn_bwd_scratch_len(2, 3, 1) == 2 * 6 * 128
    assert _lib.lib().jvp_attn_bwd_scratch_len(0, 1, 1) == -1


def call_prologue(**kw):
    a = dict(qkv=FAKE, dqkv=FAKE, outs=[FAKE] * 6, nq=FAKE, nk=FAKE, group=1536, eps=1e-6,
             cos=FAKE, sin=FAKE, rope_rows=100, B=1, L=100, H=12, d=128, dtype=_lib.JVP_BF16)
    a.update(kw)
    fp = ctypes.POINTER(ctypes.c_float)
    cvt = lambda x: ctypes.cast(x, fp) if x else None  # noqa: E731
    return _lib.lib().jvp_attn_qkv_prologue(a["qkv"], a["dqkv"], *a["outs"], cvt(a["nq"]),
                                            cvt(a["nk"]), a["group"], a["eps"], cvt(a["cos"]),
                                            cvt(a["sin"]), a["rope_rows"], a["B"], a["L"],
                                            a["H"], a["d"], a["dtype"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(qkv=0), _lib.JVP_ERR_INVALID_ARG),
    (dict(nk=0), _lib.JVP_ERR_INVALID_ARG),                   # one norm weight only
    (dict(group=64), _lib.JVP_ERR_INVALID_ARG),               # neither H*d nor d
    (dict(rope_rows=99), _lib.JVP_ERR_INVALID_ARG),           # table shorter than L
    (dict(H=3, d=32), _lib.JVP_ERR_INVALID_ARG),              # H*d not a multiple of 256
    (dict(d=96, H=8), _lib.JVP_ERR_UNSUPPORTED_HEAD_DIM),
    (dict(dtype=_lib.JVP_FP32), _lib.JVP_ERR_INVALID_ARG),
    (dict(eps=float("nan")), _lib.JVP_ERR_INVALID_ARG),
    (dict(outs=[FAKE] * 5 + [FAKE + 8]), _lib.JVP_ERR_MISALIGNED),
])
def test_prologue_argument_errors(kw, code):
    assert call_prologue(**kw) == code


def test_size_limits():
    # index ranges of the kernels: rejected before any device work
    assert call_cache(B=70000, H=70000, Lq=1, Lk=1, Lcache=1) == _lib.JVP_ERR_TOO_LARGE
    fp = ctypes.POINTER(ctypes.c_float)
    rc = _lib.lib().jvp_attn_bwd(*[FAKE] * 5, ctypes.cast(FAKE, fp), *[FAKE] * 3,
                                 ctypes.cast(FAKE, fp), 1 << 40, 70000, 70000, 64, 128,
                                 _lib.JVP_BF16, _lib.MaskDesc(ja.TEACHER_FORCING, 8, 4, 1), 0.0,
                                 None)
    assert rc == _lib.JVP_ERR_TOO_LARGE
    assert call_prologue(B=1 << 20, L=1 << 15, rope_rows=1 << 15) == _lib.JVP_ERR_TOO_LARGE


def call_scatter(ptr=0x1000, dst=0x2000, P=2, h0=0, Ht=2, B=1, H=1, L=64, d=128,
                 dtype=_lib.JVP_BF16, mask=(ja.TEACHER_FORCING, 8, 4, 1), scale=0.0,
                 o_dst=None, null_arrays=False):
    arr = lambda xs: (ctypes.c_void_p * max(1, len(xs)))(*xs)
    o = arr([dst] * P if o_dst is None else o_dst)
    do = arr([dst + 0x1000] * P)
    ls = arr([dst + 0x2000] * P)
    if null_arrays:
        o = None
    return _lib.lib().jvp_attn_fwd_scatter(
        *[ctypes.c_void_p(ptr)] * 6, o, do, ls, P, h0, Ht,
        B, H, L, d, dtype, _lib.MaskDesc(*mask), scale, None)


@pytest.mark.parametrize("kw,code", [
    (dict(null_arrays=True), _lib.JVP_ERR_INVALID_ARG),
    (dict(P=0), _lib.JVP_ERR_INVALID_ARG),
    (dict(P=9), _lib.JVP_ERR_INVALID_ARG),          # more shards than the kernel's table
    (dict(P=3), _lib.JVP_ERR_INVALID_ARG),          # 64 tokens do not split in 3
    (dict(h0=2, Ht=2), _lib.JVP_ERR_INVALID_ARG),   # head group past the total
    (dict(h0=-1), _lib.JVP_ERR_INVALID_ARG),
    (dict(Ht=0), _lib.JVP_ERR_INVALID_ARG),
    (dict(o_dst=[0x2000, 0]), _lib.JVP_ERR_INVALID_ARG),
    (dict(o_dst=[0x2000, 0x2008]), _lib.JVP_ERR_MISALIGNED),
    (dict(d=64), _lib.JVP_ERR_UNSUPPORTED_HEAD_DIM),  # tensor-core kernel only
    (dict(dtype=_lib.JVP_FP32), _lib.JVP_ERR_UNSUPPORTED_HEAD_DIM),
    (dict(ptr=0x1008), _lib.JVP_ERR_MISALIGNED),
    (dict(L=63), _lib.JVP_ERR_INVALID_ARG),
])
def test_scatter_argument_errors(kw, code):
    assert call_scatter(**kw) == code


def test_scatter_valid_call_without_gpu_fails_cleanly():
    rc = call_scatter()
    assert rc in (_lib.JVP_ERR_LAUNCH_FAILED, _lib.JVP_ERR_UNSUPPORTED_DEVICE)


def call_barrier(flags=(0x1000, 0x2000), n=None, rank=0, epoch=1):
    n = len(flags) if n is None else n
    arr = (ctypes.c_void_p * max(len(flags), 1))(*flags) if flags is not None else None
    return _lib.lib().jvp_attn_signal_barrier(arr, n, rank, epoch, None)


@pytest.mark.parametrize("kw,code", [
    (dict(flags=None, n=2), _lib.JVP_ERR_INVALID_ARG),
    (dict(n=0), _lib.JVP_ERR_INVALID_ARG),
    (dict(flags=tuple(0x1000 * (i + 1) for i in range(9))), _lib.JVP_ERR_INVALID_ARG),
    (dict(rank=2), _lib.JVP_ERR_INVALID_ARG),
    (dict(rank=-1), _lib.JVP_ERR_INVALID_ARG),
    (dict(flags=(0x1000, 0)), _lib.JVP_ERR_INVALID_ARG),
    (dict(flags=(0x1000, 0x2002)), _lib.JVP_ERR_MISALIGNED),
])
def test_signal_barrier_argument_errors(kw, code):
    assert call_barrier(**kw) == code


def test_signal_barrier_valid_call_without_gpu_fails_cleanly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    # valid arguments reach the device query, which fails without a GPU
    rc = call_barrier()
    assert rc in (_lib.JVP_ERR_UNSUPPORTED_DEVICE, _lib.JVP_ERR_LAUNCH_FAILED)
