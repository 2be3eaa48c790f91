"""GPU parity of w4a8_moe_forward against the oracle.

Bit-exact: packed weights and scales, input activation codes and scales,
routing ids, expert offsets, permutation.  Within tolerance (float): routing
weights (1e-6 relative), the SwiGLU output h and the down-projection rows
(relative Frobenius 1e-4: FP32 accumulation on both GEMMs), the intermediate
E4M3 codes (a code may move by one step where the FP32 and float64 values of h
straddle a rounding midpoint) and the final bf16 output (relative Frobenius
2e-3).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a8_quantized_moe_b200 as w4
from gpu_helpers import (assert_mse_clip_choice, aux_buffers, bf16_bits, codes_agree, f64,
                         rel_fro, repack_b200, small_case, unrepack_b200)

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3          # final bf16 output, relative Frobenius
MID_TOL = 1e-4          # h and Y rows (float32 GEMMs vs float64)
CODE_MATCH = 0.999      # fraction of intermediate E4M3 codes equal to the oracle's


def _store(w13, w2, mse_clip=False):
    return oracle.ExpertStore(w13.shape[0], lambda e: (f64(w13[e]), f64(w2[e])),
                              quantize=oracle.mse_clip_quantize_int4 if mse_clip else None)


def run_and_compare(cfg, hidden, logits, w13, w2, check_rows=None, mse_clip=False):
    E, k = cfg.E, cfg.k
    T, H, I = hidden.shape[0], cfg.H, cfg.I
    layer = w4.W4A8MoELayer.from_bf16(w13.cuda(), w2.cuda(), k, mse_clip=mse_clip)
    aux = aux_buffers(T, H, I, E, k)
    out = layer(hidden.cuda(), logits.cuda(), aux=aux)
    w4.w4a8_check_device_error()
    store = _store(w13, w2, mse_clip)
    res = oracle.moe_forward(f64(hidden), logits.numpy(), store, k)

    # packed weights (bit-exact; with the clip search, near ties within the
    # float64 summation bound may take either tied candidate)
    for e in range(E):
        p13, s13, p2, s2 = store[e]
        if mse_clip:
            for wq, packed, scales in ((w13[e], layer.w13_packed[e], layer.w13_scales[e]),
                                       (w2[e], layer.w2_packed[e], layer.w2_scales[e])):
                assert_mse_clip_choice(unrepack_b200(packed.cpu().numpy()),
                                       bf16_bits(scales.t()), f64(wq))
            continue
        assert np.array_equal(layer.w13_packed[e].cpu().numpy(), repack_b200(p13))
        assert np.array_equal(bf16_bits(layer.w13_scales[e].t()), oracle.f64_to_bf16_bits(s13))
        assert np.array_equal(layer.w2_packed[e].cpu().numpy(), repack_b200(p2))
        assert np.array_equal(bf16_bits(layer.w2_scales[e].t()), oracle.f64_to_bf16_bits(s2))
    # routing + permutation (bit-exact), weights (1e-6)
    assert np.array_equal(aux["topk_ids"].cpu().numpy(), res["topk_ids"])
    assert np.array_equal(aux["expert_offsets"].cpu().numpy(), res["expert_offsets"])
    assert np.array_equal(aux["sorted_token_ids"].cpu().numpy(), res["sorted_token_ids"])
    assert np.array_equal(aux["row_of"].cpu().numpy(), res["row_of"])
    assert np.allclose(aux["topk_w"].cpu().numpy(), res["topk_w"], rtol=1e-6, atol=1e-30)
    # activation codes (bit-exact)
    assert np.array_equal(aux["act_codes"].cpu().numpy(), res["act_codes"])
    assert np.array_equal(aux["act_scales"].cpu().numpy().astype(np.float64), res["act_scales"])
    # intermediate
    rows = sorted(res["inter_h"].keys())
    gh = aux["inter_h"].cpu().numpy()[rows]
    oh = np.stack([res["inter_h"][r] for r in rows])
    e_h = rel_fro(gh, oh)
    gc = aux["inter_codes"].cpu().numpy()[rows]
    oc = np.stack([res["inter_codes"][r] for r in rows])
    frac, dist = codes_agree(gc, oc)
    gy = aux["y_rows"].cpu().numpy()[rows]
    oy = np.stack([res["y_rows"][r] for r in rows])
    e_y = rel_fro(gy, oy)
    e_out = rel_fro(f64(out), res["out"])
    print(f"\n[{cfg.name}] h {e_h:.2e}  codes {frac:.6f} (max step {dist})  Y {e_y:.2e}  "
          f"out {e_out:.2e}")
    assert e_h <= MID_TOL, e_h
    assert frac >= CODE_MATCH and dist <= 1, (frac, dist)
    gs = aux["inter_scales"].cpu().numpy().astype(np.float64)[rows]
    os_ = np.array([res["inter_scales"][r] for r in rows])
    assert np.allclose(gs, os_, rtol=1e-5, atol=0)
    assert e_y <= MID_TOL * 10, e_y
    assert e_out <= OUT_TOL, e_out
    return out, res, aux


def test_forward_tiny_workload():
    cfg = workloads.CONFIGS[0]
    run_and_compare(cfg, *small_case(cfg))


@pytest.mark.parametrize("cfg", [
    workloads.MoEConfig("single_token_dense", T=1, H=128, I=128, E=1, k=1, seed=11),
    workloads.MoEConfig("k_equals_E", T=3, H=128, I=128, E=4, k=4, seed=12),
    workloads.MoEConfig("ragged", T=37, H=384, I=256, E=6, k=3, seed=13),
    workloads.MoEConfig("multi_block_segments", T=300, H=256, I=128, E=2, k=2, seed=14),
    workloads.MoEConfig("zipf_empty", T=200, H=256, I=256, E=16, k=4, seed=15, zipf_s=1.1,
                        forced_empty=5),
    workloads.MoEConfig("outliers_wide", T=24, H=1024, I=512, E=8, k=2, seed=16,
                        outlier_frac=0.01),
    # few tokens per expert on average (the narrow-tile shape) but skewed, so
    # the busiest experts span several 32-token tiles
    workloads.MoEConfig("decode_shape_multi_block", T=96, H=256, I=128, E=8, k=2, seed=17,
                        zipf_s=1.1),
], ids=lambda c: c.name)
def test_forward_edge_cases(cfg):
    run_and_compare(cfg, *small_case(cfg))


@pytest.mark.parametrize("cfg", [
    workloads.CONFIGS[0],
    workloads.MoEConfig("ragged_clip", T=37, H=384, I=256, E=6, k=3, seed=13),
    workloads.MoEConfig("multi_block_clip", T=300, H=256, I=128, E=2, k=2, seed=14),
], ids=lambda c: c.name)
def test_forward_with_mse_clip_weights(cfg):
    # experts quantised by the clip search (codes -8 occur) on both sides
    run_and_compare(cfg, *small_case(cfg), mse_clip=True)


def test_forward_zero_token_row_and_no_aux_path():
    cfg = workloads.MoEConfig("zero_row", T=8, H=256, I=128, E=4, k=2, seed=21)
    hidden, logits, w13, w2 = small_case(cfg)
    hidden[3] = 0.0
    out, res, _ = run_and_compare(cfg, hidden, logits, w13, w2)
    assert torch.all(out[3] == 0)
    # the same call without aux buffers gives the same bits
    layer = w4.W4A8MoELayer.from_bf16(w13.cuda(), w2.cuda(), cfg.k)
    out2 = layer(hidden.cuda(), logits.cuda())
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    # and it is deterministic run to run
    out3 = layer(hidden.cuda(), logits.cuda())
    assert torch.equal(out2.view(torch.int16), out3.view(torch.int16))


def test_forward_zero_tokens():
    cfg = workloads.MoEConfig("empty", T=0, H=256, I=128, E=4, k=2, seed=3)
    w13 = torch.zeros(4, 256, 256, dtype=torch.bfloat16, device="cuda")
    w2 = torch.zeros(4, 256, 128, dtype=torch.bfloat16, device="cuda")
    layer = w4.W4A8MoELayer.from_bf16(w13, w2, 2)
    out = layer(torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda"),
                torch.zeros(0, 4, device="cuda"))
    assert out.shape == (0, 256)


def test_pages_format_goes_through_prepare():
    # the experts as the pages store them (compressed-tensors pack-quantized
    # words and [E, rows, K/128] scales) reach the forward only through
    # w4a8_prepare_experts_b200: from_packed gives the layout from_bf16 gives,
    # and the forward refuses the pages' scale layout with a message naming it
    cfg = workloads.MoEConfig("pages_format", T=12, H=256, I=128, E=3, k=2, seed=31)
    hidden, logits, w13, w2 = small_case(cfg)
    p13, s13 = w4.w4a8_pack_int4(w13.cuda())
    p2, s2 = w4.w4a8_pack_int4(w2.cuda())
    ref = w4.W4A8MoELayer.from_bf16(w13.cuda(), w2.cuda(), cfg.k)
    lay = w4.W4A8MoELayer.from_packed(p13, s13, p2, s2, cfg.k)
    for a, b in ((lay.w13_packed, ref.w13_packed), (lay.w13_scales, ref.w13_scales),
                 (lay.w2_packed, ref.w2_packed), (lay.w2_scales, ref.w2_scales)):
        assert a.shape == b.shape and torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16
                                                  else a, b.view(torch.int16)
                                                  if b.dtype == torch.bfloat16 else b)
    assert torch.equal(p13, w4.w4a8_pack_int4(w13.cuda())[0])   # not in place by default
    out = lay(hidden.cuda(), logits.cuda())
    assert torch.equal(out.view(torch.int16), ref(hidden.cuda(), logits.cuda()).view(torch.int16))
    with pytest.raises(ValueError, match="w4a8_prepare_experts_b200"):
        w4.w4a8_moe_forward(hidden.cuda(), logits.cuda(), p13, s13, p2, s2, cfg.k)


def test_forward_replayed_from_a_cuda_graph():
    # the forward on fixed buffers, captured once and replayed: bit-identical to
    # the eager call, and a replay after new inputs are copied in computes them
    cfg = workloads.MoEConfig("graph", T=48, H=256, I=128, E=8, k=2, seed=41, zipf_s=1.1)
    hidden, logits, w13, w2 = small_case(cfg)
    layer = w4.W4A8MoELayer.from_bf16(w13.cuda(), w2.cuda(), cfg.k)
    h_dev, l_dev = hidden.cuda(), logits.cuda()
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    eager = layer(h_dev, l_dev).clone()
    graph = w4.capture_graph(lambda: layer(h_dev, l_dev, out=out))
    out.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
    cfg2 = cfg.with_(seed=42)
    h2, l2 = workloads.gen_hidden(cfg2), workloads.gen_logits(cfg2)
    h_dev.copy_(h2)
    l_dev.copy_(l2)
    graph.replay()
    w4.w4a8_check_device_error()
    ref2 = layer(h2.cuda(), l2.cuda())
    assert torch.equal(out.view(torch.int16), ref2.view(torch.int16))
