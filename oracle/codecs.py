"""Number formats used by the oracle: fp16 and FP8 E4M3 (OCP "fn" flavour).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module.

E4M3 ("fn"): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits, no
infinities, NaN = S.1111.111, largest finite magnitude 1.75 * 2^8 = 448,
smallest subnormal 2^-9.  The SageAttention2++ review (section "核心公式",
the delta formulas) quantizes P~ and V to this format with round-to-nearest
("⌈·⌋"); values beyond the range saturate to +-448 here ("satfinite").

Both codecs are written from the bit-format definition; the tests pin them
against torch's CPU float8_e4m3fn / float16 casts (library routines).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
FP16_MAX = 65504.0


def fp16_rne(x) -> np.ndarray:
    """Round float32/float64 values to the nearest fp16 (ties to even)."""
    with np.errstate(over="ignore"):
        return np.asarray(x).astype(np.float16)


def e4m3_decode(codes) -> np.ndarray:
    """uint8 E4M3 codes -> float64 values (NaN for S.1111.111)."""
    c = np.asarray(codes).astype(np.int64) & 0xFF
    sign = np.where(c & 0x80, -1.0, 1.0)
    mag = c & 0x7F
    e = mag >> 3
    m = mag & 7
    val = np.where(e == 0, m * 2.0 ** -9, (8 + m) * np.exp2(e.astype(np.float64) - 10.0))
    val = np.where(mag == 0x7F, np.nan, val)
    return sign * val


def e4m3_encode(x) -> np.ndarray:
    """float32/float64 -> uint8 E4M3 code: round to nearest, ties to even
    mantissa, magnitudes above 448 saturate to 448, NaN -> 0x7F.

    For |x| >= 2^-6 with binade e (2^e <= |x| < 2^(e+1)) the code is
    (e+6)*8 + rne(|x| * 2^(3-e)); the same formula with e clamped to -6
    covers the subnormals (code = rne(|x| * 2^9)), and a mantissa that
    rounds up to 16 rolls over into the next binade automatically."""
    xf = np.asarray(x, dtype=np.float64)
    neg = np.signbit(xf)
    a = np.abs(xf)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, a)
    a = np.minimum(a, 1024.0)       # anything >= 464 saturates; keeps inf finite
    with np.errstate(divide="ignore"):
        _, ex = np.frexp(a)          # a = f * 2^ex, f in [0.5, 1)
    e = np.maximum(ex.astype(np.int64) - 1, -6)
    scaled = a * np.exp2((3 - e).astype(np.float64))   # exact: power-of-two scaling
    M = np.rint(scaled).astype(np.int64)                # half-to-even
    code = (e + 6) * 8 + M
    code = np.where(a == 0, 0, code)
    code = np.minimum(code, 0x7E)                        # satfinite
    code = np.where(nan, 0x7F, code)
    code = np.where(neg & ~nan, code | 0x80, code)
    return code.astype(np.uint8)


def e4m3_round(x) -> np.ndarray:
    """Value of e4m3_encode(x), as float64."""
    return e4m3_decode(e4m3_encode(x))
