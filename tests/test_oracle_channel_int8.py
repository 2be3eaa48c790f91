"""Pins of the oracle's per-channel INT4 weight / per-token INT8 activation
variant ("GLM-5.3-Channel-INT4-w4a8" model card, quantisation table: RTN,
static, per-channel INT4 routed experts; dynamic per-token INT8
activations).  CPU only.

* INT8 activation codes against a brute-force nearest-code search;
* per-channel INT4 against a brute-force nearest-code search per row;
* the whole layer against an element-loop brute force that never forms the
  permutation.
"""
import math

import numpy as np
import torch

import workloads
from oracle import (ExpertStore, bf16_round, f32_round, moe_forward, pack_uint4b8,
                    quant_act_int8_per_token, route_topk, rtn_quantize_int4_channel,
                    unpack_uint4b8)


def _nearest_even(v: float, lo: int, hi: int) -> int:
    """Nearest integer in [lo, hi] to v by search; ties to the even integer."""
    best = None
    for c in range(lo, hi + 1):
        d = abs(v - c)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return best[1]


def test_int8_activation_codes_brute_force():
    rng = np.random.default_rng(3)
    x = rng.normal(0, 1, (6, 96)) * np.exp(rng.normal(0, 2, (6, 1)))
    x[:, 7] *= 20.0
    x[2] = 0.0
    x[4, :4] = np.array([127.0, 0.5, 1.5, -2.5])        # exact ties at scale 1
    x = bf16_round(x)
    codes, scale = quant_act_int8_per_token(x)
    for t in range(x.shape[0]):
        amax = np.abs(x[t]).max()
        s = np.float32(np.float32(amax) / np.float32(127.0))
        assert scale[t] == s
        for h in range(x.shape[1]):
            if s == 0:
                assert codes[t, h] == 0
                continue
            v = float(np.float32(np.float32(x[t, h]) / s))
            assert codes[t, h] == _nearest_even(v, -127, 127), (t, h)
        if s != 0:
            assert np.abs(codes[t]).max() == 127
    assert list(codes[4, :4]) == [127, 0, 2, -2]


def test_channel_int4_brute_force():
    rng = np.random.default_rng(4)
    w = bf16_round(rng.normal(0, 0.02, (5, 256)) * np.exp(rng.normal(0, 1, (5, 1))))
    w[1] = 0.0
    q, s = rtn_quantize_int4_channel(w)
    assert s.shape == (5, 1)
    for r in range(w.shape[0]):
        amax = np.float32(np.abs(w[r]).max())
        sb = torch.tensor([amax / np.float32(7.0)], dtype=torch.float32).to(torch.bfloat16)
        assert s[r, 0] == float(sb.float())
        for k in range(w.shape[1]):
            if s[r, 0] == 0:
                assert q[r, k] == 0
                continue
            v = float(np.float32(np.float32(w[r, k]) / np.float32(s[r, 0])))
            assert q[r, k] == _nearest_even(v, -8, 7)


def _brute_force_layer_int8(hidden, logits, experts, k):
    T, H = hidden.shape
    ids, w = route_topk(logits, k)
    codes, a_s = quant_act_int8_per_token(hidden)
    out = np.zeros((T, H))
    for t in range(T):
        acc = np.zeros(H)
        for j in range(k):
            w13p, s13, w2p, s2 = experts[int(ids[t, j])]
            q1, q2 = unpack_uint4b8(w13p), unpack_uint4b8(w2p)
            I = q1.shape[0] // 2
            g = np.zeros(2 * I)
            for n in range(2 * I):
                isum = 0
                for kap in range(H):
                    isum += int(codes[t, kap]) * int(q1[n, kap])
                g[n] = a_s[t] * s13[n, 0] * isum
            h = np.array([g[n] / (1.0 + math.exp(-g[n])) * g[I + n] for n in range(I)])
            hc, hs = quant_act_int8_per_token(h[None, :])
            y = np.zeros(H)
            for n in range(H):
                isum = 0
                for kap in range(I):
                    isum += int(hc[0, kap]) * int(q2[n, kap])
                y[n] = hs[0] * s2[n, 0] * isum
            acc += float(w[t, j]) * y
        out[t] = bf16_round(acc)
    return out


def test_forward_int8_matches_brute_force():
    cfg = workloads.MoEConfig("bf8", T=4, H=128, I=128, E=3, k=2, seed=78)
    hidden = workloads.gen_hidden(cfg).float().double().numpy()
    logits = workloads.gen_logits(cfg).numpy()
    ws = [workloads.gen_expert_weights(cfg, e) for e in range(cfg.E)]
    store = ExpertStore(cfg.E, lambda e: (ws[e][0].double().numpy(), ws[e][1].double().numpy()),
                        quantize=rtn_quantize_int4_channel)
    res = moe_forward(hidden, logits, store, cfg.k, act_format="int8")
    ref = _brute_force_layer_int8(hidden, logits, store, cfg.k)
    # float64 sums in different orders: the bf16 outputs agree except at exact
    # bf16 ties, which the float64 rounding noise cannot reach here
    assert np.array_equal(res["out"], ref)
