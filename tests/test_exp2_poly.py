"""The FMA-pipe 2^x of the attention kernel (exp2_poly2 in
csrc/attn_sm100.cu), restated step by step in fp32 and checked against the
exact 2^x.

The softmax evaluates part of every row's exponentials without the exp2
unit: x = n + r with n = rint(x) (adding 1.5 * 2^23), r = x - n, 2^r by a
degree-5 polynomial, 2^n added into the exponent field.  Its relative error
must stay at the level of ex2.approx.f32 (about 2^-22), so that the operand
codes of P~ stay decided the same way as with the exp2 unit.  The
coefficients are read from the kernel source, so the test checks what the
kernel uses."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "quantized_attention_08_b200", "csrc", "attn_sm100.cu")
F32 = np.float32
MAGIC = F32(12582912.0)


def kernel_coefficients():
    src = open(SRC, encoding="utf-8").read()
    c = {int(m.group(1)): float(m.group(2).rstrip("f"))
         for m in re.finditer(r"constexpr float kExpC(\d) = ([0-9.eE+-]+f);", src)}
    assert sorted(c) == list(range(6)), c
    return [F32(c[i]) for i in range(6)]


def fma32(a, b, c):
    # product exact in fp64; one rounding of the sum (to fp64, then fp32)
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(F32)


def exp2_poly(x, clamp=False):
    x = np.asarray(x, F32)
    if clamp:
        x = np.maximum(x, F32(-125.0))
    t = (x + MAGIC).astype(F32)
    n = (t - MAGIC).astype(F32)
    r = fma32(n, np.full_like(n, -1.0), x)
    c = kernel_coefficients()
    q = fma32(r, np.full_like(r, c[5]), np.full_like(r, c[4]))
    for k in (3, 2, 1, 0):
        q = fma32(q, r, np.full_like(r, c[k]))
    bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(F32), n, r


def test_range_reduction_is_exact():
    x = np.random.default_rng(0).uniform(-124, 9, 200000).astype(F32)
    _, n, r = exp2_poly(x)
    assert np.all(n == np.rint(x.astype(np.float64)))
    assert np.all(np.abs(r) <= 0.5)
    assert np.all(n.astype(np.float64) + r.astype(np.float64) == x.astype(np.float64))


def test_relative_error_matches_the_exp2_unit():
    rng = np.random.default_rng(1)
    x = np.concatenate([np.linspace(-124, 9, 1_000_003), rng.uniform(-30, 9, 500_000),
                        np.arange(-124, 10), np.arange(-124, 9) + 0.5]).astype(F32)
    y, _, _ = exp2_poly(x)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(y.astype(np.float64) - exact) / exact
    assert rel.max() <= 2.0 ** -21.9, float(np.log2(rel.max()))
    # integers are exact up to the polynomial's value at r = 0
    xi = np.arange(-124, 10).astype(F32)
    yi, _, _ = exp2_poly(xi)
    assert np.all(np.abs(yi.astype(np.float64) / np.exp2(xi.astype(np.float64)) - 1) <= 2.0 ** -22)


def test_clamp_keeps_tiny_results_positive_and_tiny():
    x = np.array([-125.0, -126.5, -200.0, -1e6, -3e7], F32)
    y, _, _ = exp2_poly(x, clamp=True)
    assert np.all(y > 0) and np.all(y <= 2.0 ** -124.9)
    # e4m3(448 * y) and fp16(y) are zero codes for all of them
    assert np.all(448.0 * y.astype(np.float64) < 2.0 ** -10)


def test_polynomial_fit_reproduces_the_kernel_constants():
    from quantized_attention_08_b200.fit_exp2_poly import remez_relative
    c, lev = remez_relative(5)
    assert lev < 2.0 ** -23.5
    assert [F32(v) for v in c] == kernel_coefficients()
