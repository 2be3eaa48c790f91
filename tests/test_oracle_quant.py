"""Pins for the oracle's INT4 weight quantisation, packing and FP8 activation
quantisation (CPU only)."""
import json
import os

import numpy as np
import pytest
import torch
from scipy import integrate, stats

from oracle import (bf16_bits_to_f64, bf16_round, dequantize_int4, e4m3_decode, e4m3_encode,
                    f32_round, pack_uint4b8, quant_act_fp8_per_token, rtn_quantize_int4,
                    unpack_uint4b8)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


# ---------------------------------------------------------------- packing

def test_pack_golden_words():
    g = json.load(open(os.path.join(GOLDEN, "pack_uint4b8.json")))
    q = np.array(g["q"], dtype=np.int8)[None, :]
    words = pack_uint4b8(q).view(np.uint32)[0]
    assert [hex(int(w)) for w in words] == g["words_hex"]


def test_pack_exhaustive_roundtrip_every_position():
    # value v at position p, all other positions a different value
    rows = []
    for v in range(-8, 8):
        for p in range(8):
            r = np.full(8, (v + 3) % 16 - 8, dtype=np.int8)
            r[p] = v
            rows.append(r)
    q = np.array(rows, dtype=np.int8)
    packed = pack_uint4b8(q)
    assert np.array_equal(unpack_uint4b8(packed), q)
    # independent unpack with Python integers
    for r, w in zip(q, packed.view(np.uint32)[:, 0]):
        w = int(w)
        assert [((w >> (4 * i)) & 0xF) - 8 for i in range(8)] == list(r)


def test_pack_rejects_out_of_range():
    with pytest.raises(ValueError):
        pack_uint4b8(np.full((1, 8), 8))


# ---------------------------------------------------------------- RTN

def test_rtn_brute_force_tiny():
    rng = np.random.default_rng(11)
    w = _bf16(rng.standard_normal((6, 256)) * 0.05)
    w[2, :128] = 0.0                                    # an all-zero group
    w[3, 5] = -0.0
    q, s = rtn_quantize_int4(w)
    for r in range(w.shape[0]):
        for g in range(2):
            grp = w[r, g * 128:(g + 1) * 128]
            amax = max(abs(float(v)) for v in grp)
            sg = float(bf16_round(np.array([float(np.float32(amax / 7.0))]))[0])
            assert s[r, g] == sg
            for i, v in enumerate(grp):
                if sg == 0.0:
                    want = 0
                else:
                    ratio = float(np.float32(v / sg))
                    # nearest integer in [-8, 7], ties to even, by brute force
                    cands = sorted(range(-8, 8), key=lambda c: (abs(ratio - c), c % 2))
                    want = cands[0]
                assert q[r, g * 128 + i] == want


def test_rtn_invariants():
    rng = np.random.default_rng(5)
    w = _bf16(rng.standard_normal((64, 1024)) * rng.uniform(1e-3, 10, (64, 1))
              * rng.uniform(0.5, 2.0, (1, 1024)))
    q, s = rtn_quantize_int4(w)
    deq = dequantize_int4(pack_uint4b8(q), s)
    sfull = np.repeat(s, 128, axis=1)
    assert np.all(np.abs(w - deq) <= sfull / 2 * (1 + 1e-6))
    qa = np.abs(q.astype(np.int64)).reshape(64, 8, 128).max(axis=2)
    assert np.all(qa == 7), "absmax / 7 scaling puts the group maximum at |q| = 7"
    assert q.min() >= -8 and q.max() <= 7
    assert np.all(_bf16(s) == s), "scales are bf16 values"


def test_scale_reading_fp32_then_bf16_equals_direct_rounding():
    """bf16(float32(a / 7)) == bf16(a / 7) for every finite positive bf16 a: the
    float32 division the kernels use cannot move the stored scale."""
    bits = np.arange(1, 0x7F80, dtype=np.uint16)
    a = bf16_bits_to_f64(bits)
    assert np.array_equal(bf16_round(f32_round(a / 7.0)), bf16_round(a / 7.0))


def test_int4_reading_fp32_division_equals_exact_rounding():
    """rint(float32(w / s)) == rint(w / s) for bf16 w, s in the RTN range: no
    quotient of two 8-bit significands lies within float32 rounding of a .5."""
    rng = np.random.default_rng(9)
    s = bf16_bits_to_f64(rng.integers(0x0080, 0x7E00, 400_000).astype(np.uint16))
    w = _bf16(s * rng.uniform(-7.05, 7.05, s.size))
    exact = np.rint(w / s)
    assert np.array_equal(np.rint(f32_round(w / s)), exact)


def _gaussian_rtn_rel_error(n=128):
    """Closed-form relative L2 error of RTN absmax/7 on i.i.d. Gaussian groups:
    the group maximum is reproduced exactly and the other n-1 errors are
    uniform on [-s/2, s/2] with s = M/7, so
    err^2 / w^2 = (n-1)/n * E[M^2] / (12 * 49) (sigma = 1)."""
    dens = lambda m: m * m * n * (2 * stats.norm.cdf(m) - 1) ** (n - 1) * 2 * stats.norm.pdf(m)
    em2, _ = integrate.quad(dens, 0, 20)
    return float(np.sqrt((n - 1) / n * em2 / (12 * 49)))


def test_rtn_reconstruction_error_matches_gaussian_closed_form():
    rng = np.random.default_rng(0)
    w = _bf16(rng.standard_normal((512, 4096)) * 0.02)
    q, s = rtn_quantize_int4(w)
    rec = dequantize_int4(pack_uint4b8(q), s)
    rel = np.linalg.norm(w - rec) / np.linalg.norm(w)
    pred = _gaussian_rtn_rel_error()
    assert abs(rel - pred) / pred < 0.01, (rel, pred)
    g = json.load(open(os.path.join(GOLDEN, "reconstruction_error.json")))
    # Gaussian weights have lighter tails than the real ones: below the pages' naive RTN
    assert rel < g["pages_real_weights"]["rtn_naive"]


# ---------------------------------------------------------------- activations

def test_act_quant_brute_force_tiny():
    rng = np.random.default_rng(2)
    x = _bf16(rng.standard_normal((5, 128)) * rng.uniform(0.01, 50, (5, 1)))
    x[1] = 0.0
    x[2, 7] = -0.0
    codes, scale = quant_act_fp8_per_token(x)
    all_codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    all_vals = e4m3_decode(all_codes)
    for t in range(5):
        amax = float(np.max(np.abs(x[t])))
        sc = float(np.float32(amax / 448.0))
        assert scale[t] == sc
        for i in range(128):
            if sc == 0.0:
                assert codes[t, i] == 0
                continue
            r = float(np.float32(x[t, i] / sc))
            r = max(-448.0, min(448.0, r))
            d = np.abs(all_vals - r)
            best = all_codes[d == d.min()]
            if len(best) > 1 and np.all(e4m3_decode(best) == 0.0):
                best = best[(best >> 7) == int(np.signbit(r))]   # zero keeps the sign of r
            elif len(best) > 1:
                best = best[(best & 1) == 0]                     # tie: even mantissa
            assert codes[t, i] == best[0], (t, i, r)


def test_act_quant_invariants():
    rng = np.random.default_rng(4)
    x = _bf16(rng.standard_normal((32, 6144)))
    x[:, rng.choice(6144, 61, replace=False)] *= 20.0
    codes, scale = quant_act_fp8_per_token(x)
    dec = e4m3_decode(codes)
    assert np.all(np.abs(dec).max(axis=1) == 448.0)
    # reconstruction within half an E4M3 spacing (relative 2^-4) or the subnormal half step
    err = np.abs(dec * scale[:, None] - x)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, scale[:, None] * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(err <= bound)
