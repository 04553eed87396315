"""Pins for the oracle's pre-pass: Smooth K and the per-block quantizers.

Checks are brute force in exact rational arithmetic (Python fractions),
closed-form invariants of the quantizer, and special cases."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads


def rn32(fr: Fraction) -> Fraction:
    """Round an exact rational to the nearest binary32 value (ties to even)."""
    if fr == 0:
        return Fraction(0)
    sgn = -1 if fr < 0 else 1
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    q = Fraction(2) ** (max(e, -126) - 23)
    m, r = divmod(a, q)
    m = int(m)
    if r * 2 > q or (r * 2 == q and m % 2 == 1):
        m += 1
    return sgn * m * q


def rne_int(fr: Fraction) -> int:
    f = int(fr // 1)
    r = fr - f
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and f % 2 == 1):
        f += 1
    return f


def test_rn32_helper_agrees_with_numpy_float32():
    rng = np.random.default_rng(0)
    for v in rng.standard_normal(2000) * 1e3:
        assert float(rn32(Fraction(float(v)))) == float(np.float32(v))


@pytest.mark.parametrize("shape,scale", [((1, 2, 256, 64), 1.0), ((1, 1, 300, 64), 500.0)])
def test_mean_k_equals_exact_rational_mean(shape, scale):
    rng = np.random.default_rng(11)
    k = (rng.standard_normal(shape) * scale + 3.0).astype(np.float16)
    got = oracle.mean_k(k)
    B, H, N, d = shape
    for b in range(B):
        for h in range(H):
            for c in range(0, d, 7):
                s = sum(Fraction(float(x)) for x in k[b, h, :, c])
                exact = s / N
                # the defined route: exact sum -> fp64 -> /N in fp64 -> fp32;
                # the sum is exact in fp64 here, so it is RN64(exact) -> fp32
                expect = np.float32(float(exact))
                assert got[b, h, c] == expect


def test_mean_k_is_order_free():
    w = workloads.get("small_b_n256_d64")
    _, k, _ = workloads.generate(w)
    perm = np.random.default_rng(5).permutation(k.shape[2])
    assert np.array_equal(oracle.mean_k(k), oracle.mean_k(k[:, :, perm]))


def test_quant_q_brute_force_rational():
    w = workloads.get("small_b_n256_d64")
    q, _, _ = workloads.generate(w)
    q = q[:, :1, :160, :16]          # one full block + a ragged tail, 16 channels
    scale = 0.125 * 1.1
    qh, dq = oracle.quant_q(q, scale)
    s32 = rn32(Fraction(float(np.float32(scale))))
    x = [[rn32(Fraction(float(v)) * s32) for v in row] for row in q[0, 0]]
    for bi, (r0, r1) in enumerate([(0, 128), (128, 160)]):
        amax = max(abs(v) for row in x[r0:r1] for v in row)
        delta = rn32(amax / 127)
        assert Fraction(float(dq[0, 0, bi])) == delta
        for r in range(r0, r1):
            for c in range(16):
                expect = max(-127, min(127, rne_int(rn32(x[r][c] / delta))))
                assert int(qh[0, 0, r, c]) == expect


def test_smooth_k_brute_force_rational():
    w = workloads.get("small_b_n256_d64")
    _, k, _ = workloads.generate(w)
    k = k[:, :1, :, :8]
    kh, dk, mk = oracle.smooth_quant_k(k)
    x = [[rn32(Fraction(float(v)) - Fraction(float(mk[0, 0, c]))) for c, v in enumerate(row)]
         for row in k[0, 0]]
    for bi in range(2):
        blk = x[bi * 128:(bi + 1) * 128]
        delta = rn32(max(abs(v) for row in blk for v in row) / 127)
        assert Fraction(float(dk[0, 0, bi])) == delta
        for r, row in enumerate(blk):
            for c, v in enumerate(row):
                assert int(kh[0, 0, bi * 128 + r, c]) == max(-127, min(127, rne_int(rn32(v / delta))))


@pytest.mark.parametrize("N", [256, 300, 1])
def test_quantizer_invariants(N):
    rng = np.random.default_rng(N)
    x = (rng.standard_normal((2, 3, N, 64)) * rng.uniform(0.01, 50, (2, 3, 1, 1))).astype(np.float32)
    xh, dl = oracle.quant_blocks(x)
    nb = dl.shape[-1]
    assert nb == (N + 127) // 128
    assert np.abs(xh.astype(np.int32)).max() <= 127
    for bi in range(nb):
        sl = slice(bi * 128, min(N, bi * 128 + 128))
        blk = x[..., sl, :].astype(np.float64)
        hb = xh[..., sl, :].astype(np.float64)
        d = dl[..., bi].astype(np.float64)[..., None, None]
        amax = np.abs(blk).max(axis=(-2, -1))
        assert np.array_equal(dl[..., bi], (amax.astype(np.float32) / np.float32(127)).astype(np.float32))
        # every non-empty block uses the full code range
        assert np.all(np.abs(hb).max(axis=(-2, -1)) == 127)
        # dequantization error within half a step (plus fp32 division rounding)
        assert np.all(np.abs(blk - d * hb) <= d / 2 * (1 + 2.0 ** -20))


def test_zero_block_quantizes_to_zero():
    x = np.zeros((1, 1, 256, 64), np.float32)
    x[..., 128:, :] = 1.5
    xh, dl = oracle.quant_blocks(x)
    assert dl[0, 0, 0] == 0 and np.all(xh[..., :128, :] == 0)
    assert np.all(xh[..., 128:, :] == 127)


def test_quant_v_fp8_rational_and_invariants():
    w = workloads.get("llm_8p8_b2_h16_n4096_d128").with_(B=1, H=2, H_kv=2, N=200)
    _, _, v = workloads.generate(w)
    for v_r in (448.0, 9.0):
        vh, dv = oracle.quant_v_fp8(v, v_r)
        for c in range(0, 128, 17):
            col = v[0, 1, :, c]
            amax = max(abs(Fraction(float(t))) for t in col)
            delta = rn32(amax / Fraction(v_r))
            assert Fraction(float(dv[0, 1, c])) == delta
            y = np.array([float(rn32(Fraction(float(t)) / delta)) for t in col])
            assert np.array_equal(vh[0, 1, :, c], oracle.e4m3_encode(y))
        dec = oracle.e4m3_decode(vh)
        # the column maximum lands on the top of the range
        assert np.allclose(np.abs(dec).max(axis=2), v_r, rtol=2 ** -3)
        err = np.abs(v.astype(np.float64) - dv[:, :, None, :] * dec)
        bound = dv[:, :, None, :] * np.maximum(np.abs(v / dv[:, :, None, :]) * 2.0 ** -4, 2.0 ** -10)
        assert np.all(err <= bound * (1 + 2.0 ** -20))


def test_quant_v_fp8_zero_column():
    v = np.zeros((1, 1, 64, 64), np.float16)
    v[..., 1] = 2.0
    vh, dv = oracle.quant_v_fp8(v)
    assert dv[0, 0, 0] == 0 and np.all(vh[..., 0] == 0)
    assert np.all(oracle.e4m3_decode(vh[..., 1]) == 448.0)
