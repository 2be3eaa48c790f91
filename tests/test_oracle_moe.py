"""Pins for the oracle's whole-layer forward (CPU only).

* brute force: a per-(token, slot) loop that never forms the permutation and
  computes every dot product element by element;
* exact integer case: inputs chosen so that every quantisation step is exact
  and the gate/up pre-activations are integers known in closed form;
* identical experts: the renormalised weights sum to one, so the output does
  not depend on the routing.
"""
import math

import numpy as np
import pytest
import torch

import workloads
from oracle import (ExpertStore, e4m3_decode, moe_forward, pack_uint4b8,
                    quant_act_fp8_per_token, route_topk, rtn_quantize_int4, unpack_uint4b8,
                    bf16_round)


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


def _store_from_arrays(w13s, w2s):
    return ExpertStore(len(w13s), lambda e: (w13s[e], w2s[e]))


def _brute_force_layer(hidden, logits, experts, k):
    """out[t] = bf16(sum_j w_j * FFN_{e_j}(x_t)) with explicit element loops."""
    T, H = hidden.shape
    ids, w = route_topk(logits, k)
    codes, a_s = quant_act_fp8_per_token(hidden)
    out = np.zeros((T, H))
    for t in range(T):
        acc = np.zeros(H)
        for j in range(k):
            w13p, s13, w2p, s2 = experts[int(ids[t, j])]
            q1, q2 = unpack_uint4b8(w13p), unpack_uint4b8(w2p)
            I = q1.shape[0] // 2
            x = [a_s[t] * v for v in e4m3_decode(codes[t])]
            g = np.zeros(2 * I)
            for n in range(2 * I):
                s = 0.0
                for kap in range(H):
                    s += x[kap] * (float(q1[n, kap]) * s13[n, kap // 128])
                g[n] = s
            h = np.array([g[n] / (1.0 + math.exp(-g[n])) * g[I + n] for n in range(I)])
            hc, hs = quant_act_fp8_per_token(h[None, :])
            hd = [hs[0] * v for v in e4m3_decode(hc[0])]
            y = np.zeros(H)
            for n in range(H):
                s = 0.0
                for kap in range(I):
                    s += hd[kap] * (float(q2[n, kap]) * s2[n, kap // 128])
                y[n] = s
            acc += float(w[t, j]) * y
        out[t] = bf16_round(acc)
    return out


def test_forward_matches_brute_force_multi_expert():
    cfg = workloads.MoEConfig("bf", T=5, H=128, I=128, E=3, k=2, seed=77)
    hidden = workloads.gen_hidden(cfg).float().double().numpy()
    logits = workloads.gen_logits(cfg).numpy()
    ws = [workloads.gen_expert_weights(cfg, e) for e in range(cfg.E)]
    store = _store_from_arrays([a.double().numpy() for a, _ in ws],
                               [b.double().numpy() for _, b in ws])
    res = moe_forward(hidden, logits, store, cfg.k)
    ref = _brute_force_layer(hidden, logits, store, cfg.k)
    # both are float64 up to summation order; the bf16 outputs agree except at
    # exact bf16 rounding ties, which float64 noise cannot reach here
    assert np.array_equal(res["out"], ref)
    # a token subset gives the same rows
    sub = moe_forward(hidden, logits, store, cfg.k, tokens=np.array([3, 0]))
    assert np.array_equal(sub["out"], res["out"][[3, 0]])


def test_forward_exact_integer_case():
    """T=1, H=I=128, E=1, k=1.  x in {-7..7} with absmax 7 gives the activation
    scale 7/448 = 2^-6 and codes 64*x, all exact; weights c*q with q in
    {-7..7} (each row holds a +-7) and c a power of two give scale c and the
    values q back.  So G = x . W^T is an exact integer multiple of c."""
    H = I = 128
    x = np.array([(kap % 15) - 7 for kap in range(H)], dtype=np.float64)[None, :]
    rng = np.random.default_rng(123)
    q1 = rng.integers(-7, 8, (2 * I, H))
    q1[:, 0] = 7
    q2 = rng.integers(-7, 8, (H, I))
    q2[:, 3] = -7
    c1, c2 = 2.0 ** -8, 2.0 ** -6
    w13, w2 = q1 * c1, q2 * c2
    codes, a_s = quant_act_fp8_per_token(x)
    assert a_s[0] == 2.0 ** -6 and np.array_equal(e4m3_decode(codes[0]) * a_s[0], x[0])
    qq, ss = rtn_quantize_int4(w13)
    assert np.all(ss == c1) and np.array_equal(qq, q1)
    G = (x[0].astype(np.int64) @ q1.T.astype(np.int64)) * c1        # integer closed form
    h = G[:I] / (1.0 + np.exp(-G[:I])) * G[I:]
    hc, hs = quant_act_fp8_per_token(h[None, :])
    Y = (hs[0] * e4m3_decode(hc[0])) @ (q2 * c2).T
    logits = np.zeros((1, 1), dtype=np.float32)
    res = moe_forward(x, logits, _store_from_arrays([w13], [w2]), 1)
    assert res["topk_w"][0, 0] == 1.0
    assert np.array_equal(res["inter_codes"][0], hc[0]) and res["inter_scales"][0] == hs[0]
    assert np.array_equal(res["out"][0], bf16_round(Y))
    # swapping gate and up changes the answer (the pin sees a transposed split)
    h_sw = G[I:] / (1.0 + np.exp(-G[I:])) * G[:I]
    assert not np.allclose(h, h_sw)


def test_forward_identical_experts_is_routing_invariant():
    cfg = workloads.MoEConfig("ident", T=6, H=256, I=128, E=4, k=2, seed=5)
    hidden = workloads.gen_hidden(cfg).float().double().numpy()
    w13, w2 = workloads.gen_expert_weights(cfg, 0)
    w13, w2 = w13.double().numpy(), w2.double().numpy()
    store = _store_from_arrays([w13] * 4, [w2] * 4)
    logits = workloads.gen_logits(cfg).numpy()
    res = moe_forward(hidden, logits, store, cfg.k)
    single = moe_forward(hidden, np.zeros((cfg.T, 1), np.float32),
                         _store_from_arrays([w13], [w2]), 1)
    # sum_j w_j = 1 up to float32 rounding of the weights: within one bf16 step
    d = np.abs(res["out"] - single["out"])
    assert np.all(d <= np.abs(single["out"]) * 2.0 ** -7 + 1e-30)
    assert np.mean(d == 0) > 0.95


def test_forward_tiny_workload_shapes():
    cfg = workloads.CONFIGS[0]
    hidden = workloads.gen_hidden(cfg).float().double().numpy()
    logits = workloads.gen_logits(cfg).numpy()
    ws = [workloads.gen_expert_weights(cfg, e) for e in range(cfg.E)]
    store = _store_from_arrays([a.double().numpy() for a, _ in ws],
                               [b.double().numpy() for _, b in ws])
    res = moe_forward(hidden, logits, store, cfg.k)
    assert res["out"].shape == (cfg.T, cfg.H)
    assert len(res["inter_codes"]) == cfg.T * cfg.k
    assert np.all(np.isfinite(res["out"]))
