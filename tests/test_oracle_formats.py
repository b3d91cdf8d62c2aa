"""Pins for the oracle's number-format routines (CPU only).

The oracle decodes fp16 / bf16 / fp32 / E4M3 storage from the published
format definitions and encodes with round-to-nearest-even.  These tests check
it against independent library conversions (NumPy float16/float32, torch
bfloat16 / float8_e4m3fn) exhaustively where the code space is small, and
against values that follow from the OCP E4M3 definition itself.
"""
import math

import numpy as np
import pytest
import torch

import oracle as orc


def _same(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nan_a, nan_b = np.isnan(a), np.isnan(b)
    assert np.array_equal(nan_a, nan_b)
    assert np.array_equal(a[~nan_a], b[~nan_b])
    # signed zeros too
    assert np.array_equal(np.signbit(a[~nan_a]), np.signbit(b[~nan_b]))


def test_f16_decode_exhaustive_vs_numpy():
    codes = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    _same(orc.decode_values(codes, orc.F16), codes.view(np.float16).astype(np.float64))


def test_bf16_decode_exhaustive_vs_torch():
    codes = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    _same(orc.decode_values(codes, orc.BF16), ref)


def test_f32_decode_vs_numpy():
    rng = np.random.default_rng(0)
    codes = rng.integers(0, 1 << 32, size=200_000, dtype=np.uint64).astype(np.uint32)
    special = np.array([0, 0x80000000, 1, 0x807fffff, 0x00800000, 0x7f7fffff, 0x7f800000,
                        0xff800000, 0x7fc00000, 0x3f800000], dtype=np.uint32)
    codes = np.concatenate([codes, special])
    _same(orc.decode_values(codes, orc.F32), codes.view(np.float32).astype(np.float64))


def test_e4m3_decode_exhaustive_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    _same(orc.decode_values(codes, orc.FP8_E4M3), ref)


def test_e4m3_decode_definition_values():
    # OCP 8-bit FP, E4M3: bias 7, S.1111.111 is NaN, no infinities.
    dec = orc.decode_values(np.array([0x7E, 0x01, 0x08, 0x38, 0x00, 0x80, 0x07, 0x77],
                                     dtype=np.uint8), orc.FP8_E4M3)
    assert list(dec[:4]) == [448.0, 2.0 ** -9, 2.0 ** -6, 1.0]
    assert dec[4] == 0.0 and not np.signbit(dec[4])
    assert dec[5] == 0.0 and np.signbit(dec[5])
    assert dec[6] == 7 * 2.0 ** -9          # largest subnormal
    assert dec[7] == 1.875 * 2.0 ** 7       # 240
    nan = orc.decode_values(np.array([0x7F, 0xFF], dtype=np.uint8), orc.FP8_E4M3)
    assert np.isnan(nan).all()


def test_e4m3_encode_roundtrip_all_finite_codes():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = orc.decode_values(codes, orc.FP8_E4M3).astype(np.float32)
    assert np.array_equal(orc.encode_e4m3(vals), codes)


def test_e4m3_encode_vs_torch_in_range():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(100_000) * 40.0,
        rng.uniform(-448, 448, 100_000),
        rng.standard_normal(50_000) * 2.0 ** -7,   # subnormal region
    ]).astype(np.float32)
    # every midpoint between two adjacent finite codes (ties -> even)
    pos = np.sort(orc.decode_values(np.arange(0x7F, dtype=np.uint8), orc.FP8_E4M3))
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (pos[1:] + pos[:-1]) / 2)
    x = np.concatenate([x, mids, -mids])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(orc.encode_e4m3(x), ref)


def test_e4m3_encode_ties_and_saturation():
    enc = lambda v: int(orc.encode_e4m3(np.array([v], dtype=np.float32))[0])
    # ties to even: 1 + 1/16 lies halfway between 1.0 (0x38) and 1.125 (0x39)
    assert enc(1.0625) == 0x38
    assert enc(1.1875) == 0x3A       # between 1.125 (odd) and 1.25 (even)
    assert enc(2.0 ** -10) == 0x00   # half the smallest subnormal -> 0 (even)
    assert enc(3 * 2.0 ** -11) == 0x01
    assert enc(-(2.0 ** -10)) == 0x80
    # satfinite: everything beyond 448 clamps to 448
    for v in (448.0, 449.0, 464.0, 479.0, 480.0, 1e6, math.inf):
        assert enc(v) == 0x7E
        assert enc(-v) == 0xFE
    assert enc(math.nan) & 0x7F == 0x7F


def test_bf16_encode_vs_torch():
    rng = np.random.default_rng(2)
    x32 = np.concatenate([rng.standard_normal(200_000), rng.standard_normal(1000) * 1e-39,
                          [0.0, -0.0, 3.3e38, -3.4e38]]).astype(np.float32)
    ref = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.encode_bf16(x32.astype(np.float64)), ref)


def test_f16_encode_vs_numpy():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(200_000) * 100, rng.standard_normal(1000) * 1e-6,
                        [0.0, -0.0, 65504.0, 65519.9, 65520.0, 1e6]])
    assert np.array_equal(orc.encode_f16(x), x.astype(np.float16).view(np.uint16))
