"""The FMA-pipe exp2 of the attention kernel, checked on the CPU.

seg_attn.cu computes part of the softmax exponentials as 2^x = 2^n * p(f),
x = n + f, n = rint(x), with a cubic p fitted for minimax relative error on
[-1/2, 1/2]. These tests tie the constants in the kernel source to a fresh fit
(exp2_poly_fit.py) and bound the error of the whole computation, range
reduction and exponent insertion included, emulated step by step in fp32 over
the range the softmax feeds it (x = s * scale * log2(e) - m <= 8 because the
running max is raised once a tile exceeds it by more than 8).
"""

import os
import re
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "segment_causal_kv_b200", "csrc")


def kernel_constants():
    src = open(os.path.join(CSRC, "seg_attn.cu")).read()
    c = [float(re.search(rf"constexpr float kExp2C{k} = ([0-9.eE+-]+)f;", src).group(1)) for k in range(4)]
    return np.array(c, dtype=np.float32)


def exp2_fma2_emulated(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """The kernel's sequence in fp32: clamp, shift by 1.5 * 2^23, cubic, add n to the exponent field."""
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    nf = (t - magic).astype(np.float32)
    f = (x - nf).astype(np.float32)  # fma(nf, -1, x) is exact
    q = np.full_like(f, c[3])
    for k in (2, 1, 0):
        q = (q.astype(np.float64) * f.astype(np.float64) + np.float64(c[k])).astype(np.float32)
    bits = (q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_kernel_constants_are_the_minimax_fit():
    pytest.importorskip("scipy")
    tools = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tools")
    sys.path.insert(0, tools)
    try:
        import exp2_poly_fit
    finally:
        sys.path.remove(tools)
    fitted, bound = exp2_poly_fit.fit()
    np.testing.assert_allclose(kernel_constants(), fitted, rtol=0, atol=2e-6)
    assert bound < 8e-5


def test_relative_error_over_the_softmax_range():
    c = kernel_constants()
    x = np.concatenate([np.linspace(-125.0, 8.5, 2_000_001, dtype=np.float64),
                        np.arange(-125, 9, dtype=np.float64) + 0.5,  # ties of the rounding to n
                        np.arange(-125, 9, dtype=np.float64)])
    x = x.astype(np.float32)
    got = exp2_fma2_emulated(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    # 7.5e-5 from the cubic plus a few fp32 roundings
    assert rel.max() < 8e-5, rel.max()
    # far below the 2^-9 relative rounding of the BF16 P the kernel stores
    assert rel.max() < 2.0 ** -9 / 20


def test_clamp_and_exponent_edges():
    c = kernel_constants()
    x = np.array([-1e30, -200.0, -125.0, -124.5, 0.0, 8.0, 8.49], dtype=np.float32)
    got = exp2_fma2_emulated(x, c).astype(np.float64)
    assert np.all(np.isfinite(got)) and np.all(got > 0)
    # clamped inputs give 2^-125 (normal), not a wrapped exponent
    np.testing.assert_allclose(got[:3], 2.0 ** -125, rtol=1e-4)
    np.testing.assert_allclose(got[3:], np.exp2(x[3:].astype(np.float64)), rtol=1e-4)
