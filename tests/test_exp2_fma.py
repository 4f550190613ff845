"""The cache kernel computes a quarter of its exponentials on the FMA pipe
(ex2_fma2: Cody-Waite range reduction, a fitted cubic, 2^n assembled in the
exponent field). This test reads the constants from the kernel source and
replays the same float32 steps on the CPU: the relative error against
exp2 stays below the documented 8e-5 over the whole input range, and
-inf, -127 and anything below give exactly 0 (masked keys)."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(__file__), "..", "attention_jvp_continuous_b200", "csrc",
                   "attn_cache_sm100.cu")


def _constants():
    with open(SRC) as f:
        src = f.read()
    body = src[src.index("uint64_t ex2_fma2("):]
    body = body[:body.index("\n}\n")]
    shift = float(re.search(r"kShift = ([0-9.]+)f", body).group(1))
    coef = [float(c) for c in re.findall(r"f2pack\(([0-9.]+)f, \1f\)", body)]
    # Horner order in the source: c3 (times f) + c2, then c1, then c0.
    assert len(coef) == 4, coef
    return shift, coef


def _emulate(x, shift, coef):
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-127.0))
    t = (x + f32(shift)).astype(f32)
    n = (t - f32(shift)).astype(f32)
    f = (x - n).astype(f32)
    c3, c2, c1, c0 = (f32(c) for c in coef)
    q = (c3 * f + c2).astype(f32)
    q = (q * f + c1).astype(f32)
    q = (q * f + c0).astype(f32)
    s = ((t.view(np.uint32) << np.uint32(23)) + np.uint32(0x3F800000)).astype(np.uint32)
    return (q * s.view(f32)).astype(f32)


def test_shift_rounds_to_integers():
    shift, _ = _constants()
    assert shift == 1.5 * 2 ** 23


def test_relative_error_bound():
    shift, coef = _constants()
    x = np.linspace(-126.0, 127.0, 2_000_001).astype(np.float32)
    y = _emulate(x, shift, coef).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 8e-5, rel.max()


def test_masked_and_underflow_give_exact_zero():
    shift, coef = _constants()
    x = np.array([-np.inf, -127.0, -200.0, -1e30], dtype=np.float32)
    assert (_emulate(x, shift, coef) == 0.0).all()


def test_integer_powers():
    shift, coef = _constants()
    x = np.arange(-120, 121, dtype=np.float32)
    y = _emulate(x, shift, coef).astype(np.float64)
    # 2^n exactly, times the cubic at f = 0 (its constant term)
    assert np.allclose(y, np.exp2(x.astype(np.float64)) * np.float32(coef[3]), rtol=1e-7)
