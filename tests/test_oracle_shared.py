"""Pins of the oracle's FP8 128 x 128-block shared expert (GLM-5.3-W4A8 model
card, intro and "quantisation method": the shared expert keeps FP8 E4M3
weights with one scale per 128 x 128 block).  CPU only.

* block quantiser: scales recomputed in numpy float32, codes against a
  brute-force nearest-code search over every finite E4M3 value, block
  independence, the block maximum at +-448;
* group activation quantiser: reduces to the per-token quantiser on each
  128-wide slice;
* the expert: an element loop with per-block promotion (a different
  association of the same sums) and the per-token quantiser for every slice;
* the layer: a zero shared expert changes nothing, zero routed experts leave
  the shared expert alone.
"""
import math

import numpy as np
import pytest

import workloads
from oracle import (ExpertStore, bf16_round, dequant_fp8_block, e4m3_decode, moe_forward,
                    quant_act_fp8_group, quant_act_fp8_per_token, quant_fp8_block,
                    shared_expert_forward)

FINITE = np.array([c for c in range(256) if (c & 0x7F) != 0x7F])
FINITE_VAL = e4m3_decode(FINITE)


def _nearest_code(v: float) -> int:
    """Nearest finite E4M3 value to v (saturating), ties to the even code."""
    v = max(-448.0, min(448.0, v))
    d = np.abs(FINITE_VAL - v)
    best = np.flatnonzero(d == d.min())
    cand = FINITE[best]
    if len(cand) > 1:   # a tie (or +0 / -0): keep the sign of v, then the even mantissa
        cand = [c for c in cand if (c >= 128) == (math.copysign(1.0, v) < 0)] or list(cand)
        even = [c for c in cand if c % 2 == 0]
        cand = even or cand
    return int(cand[0])


def _bf16(x):
    return bf16_round(x)


def test_block_quant_brute_force():
    rng = np.random.default_rng(1)
    R, K = 256, 256
    w = rng.normal(0, 0.02, (R, K)) * np.repeat(np.repeat(np.exp(rng.normal(0, 2, (2, 2))),
                                                         128, 0), 128, 1)
    w[128:, :128] = 0.0                         # one all-zero block
    w = _bf16(w)
    codes, s = quant_fp8_block(w)
    assert codes.dtype == np.uint8 and s.shape == (2, 2)
    for bi in range(2):
        for bj in range(2):
            blk = w[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128]
            amax = np.float32(np.abs(blk).max())
            sf = np.float32(amax / np.float32(448.0))
            assert s[bi, bj] == float(sf)
            cb = codes[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128]
            if sf == 0:
                assert np.all(cb == 0)
                continue
            # the block maximum lands on +-448
            i, j = np.unravel_index(np.argmax(np.abs(blk)), blk.shape)
            assert cb[i, j] in (0x7E, 0xFE)
            # every 7th element against the brute-force nearest code
            for (r, c) in zip(*np.nonzero(np.ones_like(blk, bool))):
                if (r * 128 + c) % 7:
                    continue
                v = float(np.float32(np.float32(blk[r, c]) / sf))
                assert cb[r, c] == _nearest_code(v), (bi, bj, r, c)


def test_block_quant_blocks_are_independent_and_roundtrip():
    rng = np.random.default_rng(2)
    w = _bf16(rng.normal(0, 0.05, (128, 384)))
    c1, s1 = quant_fp8_block(w)
    w2 = w.copy()
    w2[:, 128:256] *= 37.0
    c2, s2 = quant_fp8_block(w2)
    assert np.array_equal(c1[:, :128], c2[:, :128]) and np.array_equal(c1[:, 256:], c2[:, 256:])
    assert s1[0, 0] == s2[0, 0] and s1[0, 2] == s2[0, 2] and s2[0, 1] != s1[0, 1]
    # E4M3 keeps 3 mantissa bits: relative error per element <= 2^-4 above the
    # subnormal range of the block
    d = dequant_fp8_block(c1, s1)
    big = np.abs(w) > 2.0 ** -6 * np.repeat(s1, 128, axis=1)
    assert np.all(np.abs(d - w)[big] <= 2.0 ** -4 * np.abs(w)[big])


def test_group_activation_quant_is_per_token_quant_of_each_slice():
    rng = np.random.default_rng(3)
    x = rng.normal(0, 1, (5, 512)) * np.exp(rng.normal(0, 2, (5, 4))).repeat(128, axis=1)
    x[1, 128:256] = 0.0
    x = _bf16(x)
    codes, s = quant_act_fp8_group(x)
    assert s.shape == (5, 4)
    for g in range(4):
        c_ref, s_ref = quant_act_fp8_per_token(x[:, g * 128:(g + 1) * 128])
        assert np.array_equal(codes[:, g * 128:(g + 1) * 128], c_ref)
        assert np.array_equal(s[:, g], s_ref)
    assert s[1, 1] == 0 and np.all(codes[1, 128:256] == 0)


def _brute_force_expert(x, w13c, s13, w2c, s2):
    """Element loops: per 128-block partial dot products, promoted by the two
    scales, summed over the blocks; the per-token quantiser on every slice."""
    T, H = x.shape
    I = w13c.shape[0] // 2
    a_codes, a_s = np.zeros((T, H), np.uint8), np.zeros((T, H // 128))
    for g in range(H // 128):
        a_codes[:, g * 128:(g + 1) * 128], a_s[:, g] = quant_act_fp8_per_token(
            x[:, g * 128:(g + 1) * 128])
    ad, w1d, w2d = e4m3_decode(a_codes), e4m3_decode(w13c), e4m3_decode(w2c)
    y = np.zeros((T, H))
    for t in range(T):
        G = np.zeros(2 * I)
        for n in range(2 * I):
            for g in range(H // 128):
                part = sum(ad[t, kk] * w1d[n, kk] for kk in range(g * 128, (g + 1) * 128))
                G[n] += a_s[t, g] * s13[n // 128, g] * part
        h = np.array([G[n] / (1.0 + math.exp(-G[n])) * G[I + n] for n in range(I)])
        hc, hs = np.zeros(I, np.uint8), np.zeros(I // 128)
        for g in range(I // 128):
            c, s_ = quant_act_fp8_per_token(h[None, g * 128:(g + 1) * 128])
            hc[g * 128:(g + 1) * 128], hs[g] = c[0], s_[0]
        hd = e4m3_decode(hc)
        for n in range(H):
            for g in range(I // 128):
                part = sum(hd[kk] * w2d[n, kk] for kk in range(g * 128, (g + 1) * 128))
                y[t, n] += hs[g] * s2[n // 128, g] * part
    return y


def test_shared_expert_matches_block_promotion_loops():
    rng = np.random.default_rng(4)
    T, H, I = 2, 256, 128
    x = _bf16(rng.normal(0, 1, (T, H)))
    w13c, s13 = quant_fp8_block(_bf16(rng.normal(0, 0.05, (2 * I, H))))
    w2c, s2 = quant_fp8_block(_bf16(rng.normal(0, 0.05, (H, I))))
    res = shared_expert_forward(x, w13c, s13, w2c, s2)
    ref = _brute_force_expert(x, w13c, s13, w2c, s2)
    assert np.allclose(res["y"], ref, rtol=1e-12, atol=1e-14)


def _layer_inputs(cfg):
    hidden = workloads.gen_hidden(cfg).double().numpy()
    logits = workloads.gen_logits(cfg).numpy()
    ws = [workloads.gen_expert_weights(cfg, e) for e in range(cfg.E)]
    return hidden, logits, ws


def test_layer_with_zero_shared_expert_is_the_routed_layer():
    cfg = workloads.MoEConfig("sh0", T=4, H=256, I=128, E=3, k=2, seed=81)
    hidden, logits, ws = _layer_inputs(cfg)
    store = ExpertStore(cfg.E, lambda e: (ws[e][0].double().numpy(), ws[e][1].double().numpy()))
    zc13, zs13 = quant_fp8_block(np.zeros((2 * cfg.I, cfg.H)))
    zc2, zs2 = quant_fp8_block(np.zeros((cfg.H, cfg.I)))
    a = moe_forward(hidden, logits, store, cfg.k)
    b = moe_forward(hidden, logits, store, cfg.k, shared=(zc13, zs13, zc2, zs2))
    assert np.array_equal(a["out"], b["out"])


def test_layer_with_zero_routed_experts_is_the_shared_expert():
    cfg = workloads.MoEConfig("sh1", T=4, H=256, I=128, E=3, k=2, seed=82)
    hidden, logits, _ = _layer_inputs(cfg)
    zero = (np.zeros((2 * cfg.I, cfg.H)), np.zeros((cfg.H, cfg.I)))
    store = ExpertStore(cfg.E, lambda e: zero)
    rng = np.random.default_rng(5)
    sh = (*quant_fp8_block(_bf16(rng.normal(0, 0.05, (2 * cfg.I, cfg.H)))),
          *quant_fp8_block(_bf16(rng.normal(0, 0.05, (cfg.H, cfg.I)))))
    res = moe_forward(hidden, logits, store, cfg.k, shared=sh)
    alone = shared_expert_forward(hidden, *sh)
    assert np.array_equal(res["out"], bf16_round(alone["y"]))
    assert np.any(res["out"] != 0)
