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


def _exact_errors(group: np.ndarray):
    """Exact squared error of each of the 11 candidates, built independently
    (numpy float32 scale route, torch bf16 conversion, rational sums)."""
    g32 = group.astype(np.float32)
    amax = np.float32(np.abs(g32).max())
    out = []
    for i in range(11):
        r = np.float32((100.0 - 3.0 * i) / 100.0)
        s = np.float32(_bf16_torch(np.float32(np.float32(amax * r) / np.float32(7.0))))
        q = np.zeros(128) if s == 0 else np.clip(np.rint((g32 / s).astype(np.float32)), -8, 7)
        out.append((float(s), sum((Fraction(float(w)) - int(qq) * Fraction(float(s))) ** 2
                                  for w, qq in zip(g32, q))))
    return out


def test_float_errors_within_the_stated_bound():
    # the float64 candidate errors stay within MSE_ERR_REL_BOUND of the exact
    # sums, on Gaussian, heavy-tailed, subnormal-heavy and outlier groups
    rng = np.random.default_rng(21)
    rows = [rng.normal(0, 0.02, 256), rng.standard_t(2, 256) * 0.01,
            rng.normal(0, 1e-39, 256), np.where(rng.random(256) < 0.02, 3.0, 1e-3)]
    w = oracle.bf16_round(np.stack(rows))
    q_all, s_all, e_all = oracle.mse_clip_candidates(w)
    for r in range(w.shape[0]):
        for g in range(2):
            exact = _exact_errors(w[r, g * 128:(g + 1) * 128])
            for i, (s, ex) in enumerate(exact):
                assert s_all[i, r, g] == s
                assert abs(Fraction(float(e_all[i, r, g])) - ex) <= \
                    Fraction(oracle.MSE_ERR_REL_BOUND) * ex


# Sparse groups in which two DISTINCT candidate scales give exactly the same
# squared error (found by a seeded search over groups of 1-3 nonzero bf16
# values): ((position, value) pairs, the tied candidate indices).  The rule
# keeps the first of the exact minima, i.e. the larger ratio.
EXACT_TIES = [
    ([(34, "-0x1.ea00000000000p-2"), (47, "-0x1.cc00000000000p-3")], (4, 5)),
    ([(127, "-0x1.3800000000000p-3"), (123, "-0x1.4200000000000p-3")], (0, 5)),
    ([(53, "-0x1.f000000000000p-2"), (79, "0x1.6a00000000000p-1")], (0, 1)),
    ([(79, "-0x1.0a00000000000p-5"), (15, "-0x1.f000000000000p-1"),
      (75, "0x1.0000000000000p+0")], (0, 1)),
    ([(123, "-0x1.9400000000000p-1"), (9, "-0x1.8400000000000p-1"),
      (89, "0x1.4e00000000000p-5")], (1, 5)),
]


@pytest.mark.parametrize("case", range(len(EXACT_TIES)))
def test_exact_ties_keep_the_larger_ratio(case):
    vals, (i, j) = EXACT_TIES[case]
    g = np.zeros(128)
    for pos, hx in vals:
        g[pos] = float.fromhex(hx)
    exact = _exact_errors(g)
    assert exact[i][0] != exact[j][0]                  # two different scales ...
    assert exact[i][1] == exact[j][1]                  # ... with the same exact error
    assert exact[i][1] == min(e for _, e in exact)     # and it is the least
    q, s = oracle.mse_clip_quantize_int4(g[None])
    assert s[0, 0] == exact[i][0]
