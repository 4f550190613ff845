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
            src = open(os.path.join(ROOT, "include", h)).read()
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
