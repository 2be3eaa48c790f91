"""Pins for the oracle's number formats: library routines, closed forms and
printed points of the format definitions (CPU only)."""
import json
import os

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import (bf16_bits_to_f64, bf16_round, e4m3_decode, e4m3_encode,
                    f32_round, f64_to_bf16_bits)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _lib_e4m3(x):
    """E4M3 codes from ml_dtypes (round-to-nearest-even, no saturation)."""
    return np.asarray(x, dtype=np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)


def test_e4m3_decode_matches_library_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = e4m3_decode(codes)
    lib = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    ok = ~np.isnan(lib)
    assert np.array_equal(ours[ok], lib[ok])
    assert np.array_equal(np.signbit(ours[ok]), np.signbit(lib[ok]))
    # the same through torch's float8 type
    lt = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(ours[ok], lt[ok])


def test_e4m3_golden_points():
    g = json.load(open(os.path.join(GOLDEN, "e4m3_points.json")))
    for code_hex, val in g["points"]:
        c = np.array([int(code_hex, 16)], dtype=np.uint8)
        v = e4m3_decode(c)[0]
        assert v == val and np.signbit(v) == np.signbit(val), code_hex
        assert e4m3_encode(np.array([val]))[0] == c[0], code_hex
    for code_hex in g["nan_codes"]:
        assert np.isnan(e4m3_decode(np.array([int(code_hex, 16)], dtype=np.uint8))[0])


def test_e4m3_encode_roundtrip_and_midpoints():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = e4m3_decode(codes)
    assert np.array_equal(e4m3_encode(vals), codes)
    # every midpoint between consecutive non-negative finite values: ties go to even mantissa
    pos = np.sort(e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8)))
    mids = (pos[:-1] + pos[1:]) / 2.0
    for m in (mids, -mids):
        assert np.array_equal(e4m3_encode(m), _lib_e4m3(m))
    enc = e4m3_encode(mids)
    assert np.all(enc % 2 == 0), "ties must round to an even mantissa"


def test_e4m3_encode_matches_library_on_random_float32():
    rng = np.random.default_rng(7)
    mant = rng.uniform(1.0, 2.0, 200_000)
    expo = rng.integers(-14, 9, 200_000)
    x = f32_round(np.ldexp(mant, expo) * rng.choice([-1.0, 1.0], 200_000))
    x = x[np.abs(x) < 464.0]                   # ml_dtypes turns larger values into NaN
    assert np.array_equal(e4m3_encode(x), _lib_e4m3(x))
    tx = torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(e4m3_encode(x), tx)


def test_e4m3_saturation_sign_and_nan():
    big = np.array([448.0, 463.99, 464.0, 500.0, 1e6, np.inf])
    assert np.all(e4m3_encode(big) == 0x7E)
    assert np.all(e4m3_encode(-big) == 0xFE)
    assert e4m3_encode(np.array([-0.0]))[0] == 0x80
    assert e4m3_encode(np.array([-1e-9]))[0] == 0x80     # negative underflow keeps the sign
    assert e4m3_encode(np.array([1e-9]))[0] == 0x00
    assert e4m3_encode(np.array([np.nan]))[0] == 0x7F
    # smallest subnormal and the rounding boundary around it
    assert e4m3_encode(np.array([2.0 ** -9]))[0] == 0x01
    assert e4m3_encode(np.array([2.0 ** -10]))[0] == 0x00          # tie -> even (0)
    assert e4m3_encode(np.array([1.5 * 2.0 ** -9]))[0] == 0x02     # tie -> even (2)


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(3)
    mant = rng.uniform(1.0, 2.0, 100_000)
    expo = rng.integers(-140, 128, 100_000)
    x = f32_round(np.ldexp(mant, expo) * rng.choice([-1.0, 1.0], 100_000))
    x = x[np.isfinite(x)]
    # exact ties between two bf16 neighbours
    b = bf16_bits_to_f64(rng.integers(0, 0x7F00, 20_000).astype(np.uint16))
    b2 = bf16_bits_to_f64(np.frombuffer(f64_to_bf16_bits(b).tobytes(), np.uint16) + 1)
    ties = f32_round((b + b2) / 2.0)
    for v in (x, ties, -ties):
        t = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
        assert np.array_equal(bf16_round(v), t)


def test_bf16_bits_roundtrip_and_overflow():
    bits = np.arange(0, 0x7F80, dtype=np.uint16)           # all finite non-negative bf16
    v = bf16_bits_to_f64(bits)
    assert np.array_equal(f64_to_bf16_bits(v), bits)
    assert bf16_round(np.array([3.5e38]))[0] == np.inf
    assert bf16_round(np.array([-3.5e38]))[0] == -np.inf
    assert bf16_round(np.array([3.389e38]))[0] == float.fromhex("0x1.fep127")
    assert bf16_round(np.array([3.38e38]))[0] == float.fromhex("0x1.fcp127")
