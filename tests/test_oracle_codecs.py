"""Pins for the oracle's number formats (CPU only).

The E4M3 codec is written from the OCP bit format; here it is checked
against torch's CPU float8_e4m3fn casts (a library routine) exhaustively
over every fp16 value inside the finite range, plus the saturation and
tie rules that torch does not share (torch maps overflow to NaN)."""
import numpy as np
import pytest
import torch

from oracle import codecs


def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = codecs.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # largest finite magnitude 448, the static 1/448 P~ scale of the 8+8 variant
    assert np.nanmax(ours) == 448.0 and codecs.E4M3_MAX == 448.0
    assert ours[1] == 2.0 ** -9          # smallest subnormal


def test_e4m3_encode_matches_torch_on_every_fp16_in_range():
    h = np.arange(65536, dtype=np.uint16).view(np.float16)
    f = h.astype(np.float32)
    ok = np.isfinite(f) & (np.abs(f) <= 448.0)
    f = f[ok]
    ours = codecs.e4m3_encode(f)
    ref = torch.from_numpy(f).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # -0.0 and +0.0 both allowed to keep their sign
    assert np.array_equal(ours, ref)


def test_e4m3_encode_matches_torch_random_fp32():
    rng = np.random.default_rng(7)
    f = (rng.standard_normal(200000) * np.exp2(rng.uniform(-14, 8, 200000))).astype(np.float32)
    f = f[np.abs(f) <= 448.0]
    ours = codecs.e4m3_encode(f)
    ref = torch.from_numpy(f).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_saturation_and_nan():
    big = np.array([448.0, 448.5, 463.9, 464.0, 480.0, 1e6, 65504.0, np.inf], np.float32)
    assert np.all(codecs.e4m3_encode(big) == 0x7E)
    assert np.all(codecs.e4m3_encode(-big) == 0xFE)
    assert codecs.e4m3_encode(np.array([np.nan], np.float32))[0] == 0x7F


def test_e4m3_ties_go_to_even_mantissa():
    vals = codecs.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    mids = (vals[:-1] + vals[1:]) / 2.0        # exact in fp64
    codes = codecs.e4m3_encode(mids)
    lo = np.arange(0, 0x7E)
    expect = np.where(lo % 2 == 0, lo, lo + 1)  # even code = even mantissa LSB
    assert np.array_equal(codes.astype(np.int64), expect)


def test_fp16_rne_matches_torch():
    rng = np.random.default_rng(3)
    f = (rng.standard_normal(100000) * np.exp2(rng.uniform(-20, 15, 100000))).astype(np.float32)
    ours = codecs.fp16_rne(f).view(np.uint16)
    ref = torch.from_numpy(f).to(torch.float16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
