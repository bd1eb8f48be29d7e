"""The FMA-pipe exponential of the forward kernel (ex2_poly in csrc/ptx.cuh), checked on the CPU.

The kernel evaluates a share of its exponentials 2^x as p(f) * 2^j with j = round(x), f = x - j in
[-1/2, 1/2] (Cody and Waite's range reduction) and p a degree-3 polynomial with p(0) = 1. These
tests read the constants from the shipped source, re-derive them (minimax in relative error on
[-1/2, 1/2] by Lawson's iteration), and emulate the kernel's fp32 steps to bound the error.
"""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PTX = os.path.join(ROOT, "exact_attention_161_b200", "csrc", "ptx.cuh")


def shipped_coefficients():
    src = open(PTX).read()
    body = src[src.index("float ex2_poly(float x)"):]
    body = body[:body.index("}")]
    hexf = re.findall(r"(0x1\.[0-9a-f]+p-?\d+)f", body)
    c3, c2, c1 = (float.fromhex(h) for h in hexf[:3])
    return c1, c2, c3


def test_packed_pair_uses_the_same_coefficients():
    # ex2_poly2 (FP8's pairs on f32x2 instructions) must evaluate the same polynomial
    src = open(PTX).read()
    body = src[src.index("float2 ex2_poly2(float2 x)"):]
    body = body[:body.index("\n}")]
    hexf = [float.fromhex(h) for h in re.findall(r"(0x1\.[0-9a-f]+p-?\d+)f", body)]
    c1, c2, c3 = shipped_coefficients()
    assert sorted(set(hexf)) == sorted({c1, c2, c3}), (hexf, (c1, c2, c3))


def lawson_fit(deg=3, iters=200):
    f = np.linspace(-0.5, 0.5, 20001)
    y = 2.0 ** f
    A = np.stack([f ** k for k in range(1, deg + 1)], axis=1) / y[:, None]
    b = (y - 1.0) / y
    w = np.ones_like(f)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        w = w * np.abs(A @ c - b)
        w /= w.sum()
    return c


def f32(x):
    return np.asarray(x, dtype=np.float32)


def fma32(a, b, c):
    # fp32 fused multiply-add: the product of two fp32 values is exact in fp64; one rounding to fp32
    return f32(np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.asarray(c, np.float64))


def ex2_poly_emulated(x):
    c1, c2, c3 = shipped_coefficients()
    x = np.maximum(f32(x), f32(-127.0))
    t = f32(x + f32(12582912.0))
    f = f32(x - f32(t - f32(12582912.0)))
    q = fma32(f32(c3), f, f32(c2))
    q = fma32(q, f, f32(c1))
    q = fma32(q, f, f32(1.0))
    bits = (q.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_coefficients_are_the_minimax_fit():
    shipped = np.array(shipped_coefficients())
    fit = lawson_fit()
    assert np.allclose(shipped, fit.astype(np.float32), rtol=1e-6, atol=0), (shipped, fit)


def test_relative_error_bound_over_the_range_the_kernel_uses():
    # exponents the softmax takes: s * scale * log2(e) - m, at most 8 above 0 (lazy rescale), down to
    # where the result is below fp32's normal range
    x = np.linspace(-126.0, 9.0, 2_000_001)
    got = ex2_poly_emulated(x).astype(np.float64)
    ref = 2.0 ** f32(x).astype(np.float64)
    rel = np.abs(got / ref - 1.0)
    assert rel.max() <= 1.1e-4, rel.max()


def test_integers_are_exact_and_masked_scores_give_zero():
    j = np.arange(-126, 10)
    assert np.array_equal(ex2_poly_emulated(j.astype(np.float32)), (2.0 ** j).astype(np.float32))
    assert ex2_poly_emulated(np.array([-np.inf], np.float32))[0] == 0.0
    assert ex2_poly_emulated(np.array([-127.0], np.float32))[0] == 0.0
    assert ex2_poly_emulated(np.array([0.0], np.float32))[0] == 1.0
