"""The FMA-pipe exponential of the attention kernels' softmax (csrc/exp2x2.cuh), checked on the CPU.

The kernels compute 2^x for some scores without the SFU: x is clamped at -125, rounded to the
nearest integer n by adding and subtracting 1.5 * 2^23, f = x - n is put through a cubic, and n
is added into the exponent field. This test reads the cubic's constants from the header, redoes
those fp32 steps in numpy (each operation rounded to fp32, a fused multiply-add rounded once),
and compares with 2^x in fp64 -- the mathematical definition, not the kernel's own formula:
- relative error at most 7.5e-5 over x in [-125, 8], the range the softmax feeds it (scores
  minus a running maximum, at most 8 above it);
- exact powers of two at integers (f = 0 gives c0, within the same bound);
- masked scores (-inf) and anything below -125 give 2^-125, which is zero after bf16 rounding
  relative to a row maximum of at least 1;
- the constants are what the committed fitting script prints, and a plausible slip (a dropped
  term, a transposed pair of coefficients) breaks the bound.
"""
import pathlib
import re

import numpy as np
import pytest

CSRC = pathlib.Path(__file__).resolve().parents[1] / "sliding_window_attention_chunked_b200" / "csrc"


def _constants():
    text = (CSRC / "exp2x2.cuh").read_text()
    return [np.float32(float(re.search(rf"kExpC{i} = ([0-9.eE+-]+)f;", text).group(1))) for i in range(4)]


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def emulate(x, c):
    """the kernel's steps in fp32"""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    shifter = np.float32(12582912.0)
    j = (x + shifter).astype(np.float32)
    fr = (x - (j - shifter).astype(np.float32)).astype(np.float32)
    q = _fma32(np.full_like(fr, c[3]), fr, np.full_like(fr, c[2]))
    q = _fma32(q, fr, np.full_like(fr, c[1]))
    q = _fma32(q, fr, np.full_like(fr, c[0]))
    bits = q.view(np.uint32).astype(np.uint64) + (j.view(np.uint32).astype(np.uint64) << np.uint64(23))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def _max_rel_err(c):
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), np.arange(-125, 9) + 0.5]).astype(np.float32)
    y = emulate(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    return np.max(np.abs(y / ref - 1))


def test_cubic_relative_error_bound():
    assert _max_rel_err(_constants()) <= 7.5e-5


def test_integers_and_clamp():
    c = _constants()
    n = np.arange(-125, 9, dtype=np.float32)
    assert np.allclose(emulate(n, c) / np.exp2(n.astype(np.float64)), 1.0, rtol=7.5e-5, atol=0)
    low = emulate(np.array([-np.inf, -1e30, -200.0, -125.0], np.float32), c)
    assert np.allclose(low.astype(np.float64), 2.0 ** -125, rtol=7.5e-5, atol=0)


def test_constants_match_fitting_script():
    import importlib.util
    spec = importlib.util.spec_from_file_location("fit_exp2_cubic", CSRC / "fit_exp2_cubic.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    fitted = mod.fit(grid=4001, passes=1500)
    assert np.allclose(fitted, _constants(), rtol=2e-5, atol=0)


@pytest.mark.parametrize("slip", ["drop_cubic", "swap_c1_c2", "c0_one"])
def test_planted_slips_break_the_bound(slip):
    c = list(_constants())
    if slip == "drop_cubic":
        c[3] = np.float32(0.0)
    elif slip == "swap_c1_c2":
        c[1], c[2] = c[2], c[1]
    else:
        c[0] = np.float32(1.0)
    assert _max_rel_err(c) > 7.5e-5
