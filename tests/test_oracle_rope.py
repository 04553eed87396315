"""Pins of the oracle's rotary embedding (rotate-half pairing, fp32
products and sum, fp16 result) against closed forms."""
import numpy as np

import oracle
import workloads


def _rand(shape, seed, scale=3.0):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(shape) * scale).astype(np.float16)


def test_identity_rotation_is_exact():
    x = _rand((1, 2, 37, 64), 0)
    cos = np.ones((37, 32), np.float32)
    sin = np.zeros((37, 32), np.float32)
    assert np.array_equal(oracle.rope(x, cos, sin).view(np.uint16), x.view(np.uint16))


def test_quarter_turn_swaps_halves():
    # c = 0, s = 1: y1 = -x2, y2 = x1 exactly
    x = _rand((1, 1, 5, 128), 1)
    cos = np.zeros((5, 64), np.float32)
    sin = np.ones((5, 64), np.float32)
    y = oracle.rope(x, cos, sin)
    assert np.array_equal(y[..., :64], -x[..., 64:])
    assert np.array_equal(y[..., 64:], x[..., :64])


def test_matches_complex_multiplication_within_one_fp16_ulp():
    # (x_i + j x_{i+d/2}) * exp(j angle): the pairing and signs of the formula
    for d in (64, 128):
        N = 300
        x = _rand((2, 3, N, d), d)
        cos, sin = workloads.rope_tables(N, d)
        y = oracle.rope(x, cos, sin).astype(np.float64)
        h = d // 2
        z = (x[..., :h].astype(np.float64) + 1j * x[..., h:].astype(np.float64)) * \
            (cos.astype(np.float64) + 1j * sin.astype(np.float64))
        exact = np.concatenate([z.real, z.imag], axis=-1)
        # one fp16 ulp of the result, plus the fp32 rounding of the two
        # products and their sum (which can move the result across a fp16
        # rounding boundary when the sum cancels)
        ulp16 = np.spacing(np.abs(exact).astype(np.float16)).astype(np.float64)
        x1, x2 = x[..., :h].astype(np.float64), x[..., h:].astype(np.float64)
        c, s = cos.astype(np.float64), sin.astype(np.float64)
        mag = np.abs(x1 * c) + np.abs(x2 * s) + np.abs(x2 * c) + np.abs(x1 * s)
        f32err = 2.0 ** -23 * np.concatenate([mag, mag], axis=-1)
        assert np.all(np.abs(y - exact) <= ulp16 + f32err)
        # and a transposed pairing (interleaved channels) is far off
        xi = x.reshape(*x.shape[:-1], h, 2)
        zi = (xi[..., 0].astype(np.float64) + 1j * xi[..., 1].astype(np.float64)) * (c + 1j * s)
        wrong = np.stack([zi.real, zi.imag], axis=-1).reshape(x.shape)
        assert np.abs(y - wrong).max() > 0.1


def test_pair_norm_preserved():
    d, N = 128, 64
    x = _rand((1, 1, N, d), 7)
    cos, sin = workloads.rope_tables(N, d)
    y = oracle.rope(x, cos, sin).astype(np.float64)
    xf = x.astype(np.float64)
    h = d // 2
    nx = np.hypot(xf[..., :h], xf[..., h:])
    ny = np.hypot(y[..., :h], y[..., h:])
    assert np.allclose(nx, ny, rtol=2e-3, atol=1e-3)


def test_scores_depend_on_relative_position():
    # <rope(q, t1), rope(k, t2)> depends on t1 - t2 only (up to fp16 rounding)
    d, N = 64, 96
    cos, sin = workloads.rope_tables(N, d)
    rng = np.random.default_rng(3)
    qv = rng.standard_normal(d).astype(np.float16)
    kv = rng.standard_normal(d).astype(np.float16)
    q = np.broadcast_to(qv, (1, 1, N, d)).copy()
    k = np.broadcast_to(kv, (1, 1, N, d)).copy()
    rq = oracle.rope(q, cos, sin)[0, 0].astype(np.float64)
    rk = oracle.rope(k, cos, sin)[0, 0].astype(np.float64)
    for delta in (0, 5, 31):
        s = np.array([rq[t + delta] @ rk[t] for t in range(N - delta)])
        assert np.ptp(s) < 2e-2 * max(1.0, np.abs(s).max())


def test_tables():
    cos, sin = workloads.rope_tables(1000, 128)
    assert cos.shape == (1000, 64) and cos.dtype == np.float32
    assert np.allclose(cos.astype(np.float64) ** 2 + sin.astype(np.float64) ** 2, 1.0, atol=1e-6)
    assert np.all(cos[0] == 1) and np.all(sin[0] == 0)
