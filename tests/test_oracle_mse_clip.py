"""Pins of the oracle's per-group MSE clip search (GLM-5.3-W4A8 model card,
"quantisation method": 11 shrink ratios 1.00 -> 0.70 per group of 128, the
MSE-optimal scale kept).

The candidate scales and codes are recomputed here through independent
routes (numpy float32 arithmetic, torch's bf16 conversion), and the errors
are compared exactly with rational arithmetic, so a mistake in the oracle's
candidate construction, error or arg-min fails these tests.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle


def _bf16_torch(x32: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(x32, np.float32)).to(torch.bfloat16).float().numpy()


def _exact_choice(group: np.ndarray):
    """(index of the best ratio, its scale, its codes) by exact arithmetic."""
    g32 = group.astype(np.float32)
    amax = np.float32(np.abs(g32).max())
    best = None
    for i in range(11):
        r = np.float32((100.0 - 3.0 * i) / 100.0)
        s = np.float32(_bf16_torch(np.float32(np.float32(amax * r) / np.float32(7.0))))
        if s == 0:
            q = np.zeros(128)
        else:
            q = np.clip(np.rint((g32 / s).astype(np.float32)), -8, 7)
        err = sum((Fraction(float(w)) - int(qq) * Fraction(float(s))) ** 2
                  for w, qq in zip(g32, q))
        if best is None or err < best[0]:
            best = (err, i, float(s), q.astype(np.int8))
    return best[1], best[2], best[3]


def test_ratio_table():
    r = oracle.CLIP_RATIOS
    assert r.dtype == np.float32 and len(r) == 11
    assert r[0] == 1.0 and abs(float(r[-1]) - 0.70) < 1e-7
    assert np.all(np.diff(r.astype(np.float64)) < 0)


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_choice_matches_exact_rational_search(seed):
    rng = np.random.default_rng(seed)
    rows = []
    rows.append(rng.normal(0, 0.02, 512))                       # Gaussian
    rows.append(rng.standard_t(3, 512) * 0.01)                  # heavy tails
    x = rng.normal(0, 0.01, 512); x[::128] *= 12.0; rows.append(x)  # one outlier per group
    rows.append(rng.uniform(-0.05, 0.05, 512))                  # flat
    w = oracle.bf16_round(np.stack(rows))
    q, s = oracle.mse_clip_quantize_int4(w)
    for r in range(w.shape[0]):
        for g in range(w.shape[1] // 128):
            _, s_exact, q_exact = _exact_choice(w[r, g * 128:(g + 1) * 128])
            assert s[r, g] == s_exact
            assert np.array_equal(q[r, g * 128:(g + 1) * 128], q_exact)


def test_ratio_one_is_plain_rtn_when_clipping_cannot_help():
    # equal magnitudes: RTN reproduces every weight from bf16-exact scales, any
    # shrink makes the clamped values worse, so the search keeps ratio 1.00
    rng = np.random.default_rng(7)
    c = oracle.bf16_round(np.array([0.0703125]))[0]   # 0.0703125 / 7 is not needed exactly
    w = np.where(rng.random((4, 256)) < 0.5, -c, c)
    q_r, s_r = oracle.rtn_quantize_int4(w)
    q_m, s_m = oracle.mse_clip_quantize_int4(w)
    assert np.array_equal(q_r, q_m) and np.array_equal(s_r, s_m)


def test_single_nonzero_group_keeps_the_full_scale():
    w = np.zeros((1, 128))
    w[0, 5] = oracle.bf16_round(np.array([0.0371]))[0]
    q_r, s_r = oracle.rtn_quantize_int4(w)
    q_m, s_m = oracle.mse_clip_quantize_int4(w)
    assert np.array_equal(s_r, s_m) and q_m[0, 5] == 7


def test_error_never_above_rtn_and_zero_groups():
    rng = np.random.default_rng(11)
    w = oracle.bf16_round(rng.normal(0, 0.02, (16, 1024)))
    w[3, :128] = 0.0
    q_r, s_r = oracle.rtn_quantize_int4(w)
    q_m, s_m = oracle.mse_clip_quantize_int4(w)
    d_r = (w - oracle.dequantize_int4(oracle.pack_uint4b8(q_r), s_r)).reshape(16, 8, 128)
    d_m = (w - oracle.dequantize_int4(oracle.pack_uint4b8(q_m), s_m)).reshape(16, 8, 128)
    assert np.all((d_m ** 2).sum(-1) <= (d_r ** 2).sum(-1) * (1 + 1e-12))
    assert s_m[3, 0] == 0 and np.all(q_m[3, :128] == 0)
    assert q_m.min() >= -8 and q_m.max() <= 7


def test_gaussian_reconstruction_error_drops_like_the_pages_report():
    # Context, not an exact pin: the pages measure 0.124 (naive RTN) -> 0.103
    # (with the clip search) on real weights, a 17 % drop; on N(0, 0.02)
    # weights RTN gives 0.1173 (closed form, test_oracle_quant) and the search
    # must land clearly below it.
    rng = np.random.default_rng(5)
    w = oracle.bf16_round(rng.normal(0, 0.02, (128, 4096)))
    q, s = oracle.mse_clip_quantize_int4(w)
    rel = np.linalg.norm(w - oracle.dequantize_int4(oracle.pack_uint4b8(q), s)) / np.linalg.norm(w)
    assert 0.095 < rel < 0.107, rel
