"""GPU parity of the expert-parallel entry points on one GPU.

Expert parallelism splits the experts over ranks; here every rank's share is
computed on the one GPU in turn (no rank waits on another), from the same
gathered tokens: w4a8_moe_forward_experts over each rank's expert range, the
float32 partial sums added, and one bf16 rounding (w4a8_cast_f32_bf16).  The
result must match w4a8_moe_forward on the whole layer (up to float32
summation order) and the oracle (relative Frobenius 2e-3).  Also: the
top-k-only routing call is bit-exact against the oracle, and an expert id
outside [-1, E) is skipped and reported by the device latch.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a8_quantized_moe_b200 as w4
from gpu_helpers import aux_buffers, f64, rel_fro, small_case
from w4a8_quantized_moe_b200.ep import expert_partition

pytestmark = pytest.mark.gpu


def _share(layer, g, G):
    b, n = expert_partition(layer.E, G)[g]
    return b, n, (layer.w13_packed[b:b + n], layer.w13_scales[b:b + n],
                  layer.w2_packed[b:b + n], layer.w2_scales[b:b + n])


def _agreement(a: torch.Tensor, b: torch.Tensor):
    """(fraction of bit-equal bf16 values, relative Frobenius distance)."""
    same = float((a.view(torch.int16) == b.view(torch.int16)).float().mean())
    return same, rel_fro(f64(a), f64(b))


def _emulated_ep(layer, codes, scales, ids, w, G):
    total = torch.zeros(codes.shape[0], layer.H, dtype=torch.float32, device="cuda")
    for g in range(G):
        b, n, wl = _share(layer, g, G)
        if n == 0:
            continue
        total += w4.w4a8_moe_forward_experts(codes, scales, ids, w, layer.E, b, *wl)
    w4.w4a8_check_device_error()
    return w4.w4a8_cast_f32_bf16(total)


@pytest.mark.parametrize("cfg,G", [
    (workloads.CONFIGS[0], 2),
    (workloads.MoEConfig("ep_ragged", T=37, H=384, I=256, E=6, k=3, seed=13), 4),
    (workloads.MoEConfig("ep_multi_block", T=300, H=256, I=128, E=4, k=2, seed=14), 3),
    (workloads.MoEConfig("ep_zipf_empty", T=200, H=256, I=256, E=16, k=4, seed=15, zipf_s=1.1,
                         forced_empty=5), 8),
], ids=lambda x: getattr(x, "name", str(x)))
def test_expert_shares_sum_to_the_layer(cfg, G):
    hidden, logits, w13, w2 = small_case(cfg)
    layer = w4.W4A8MoELayer.from_bf16(w13.cuda(), w2.cuda(), cfg.k)
    aux = aux_buffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    ref = layer(hidden.cuda(), logits.cuda(), aux=aux)
    ids, w = w4.w4a8_moe_route_topk(logits.cuda(), cfg.k)
    assert torch.equal(ids, aux["topk_ids"]) and torch.equal(w, aux["topk_w"])
    out = _emulated_ep(layer, aux["act_codes"], aux["act_scales"], ids, w, G)
    store = oracle.ExpertStore(cfg.E, lambda e: (f64(w13[e]), f64(w2[e])))
    res = oracle.moe_forward(f64(hidden), logits.numpy(), store, cfg.k)
    # the shares' float32 sums are added in another order than the layer's slot
    # sum: a value can round to the neighbouring bf16 value where the sum sits at a
    # midpoint, or move further where the slots nearly cancel
    same, dist = _agreement(out, ref)
    e_oracle = rel_fro(f64(out), res["out"])
    print(f"\n[{cfg.name}, {G} shares] vs layer: {same:.5f} bit-equal, rel-Frobenius "
          f"{dist:.2e}; vs oracle {e_oracle:.2e}")
    assert same >= 0.999 and dist <= 1e-4
    assert e_oracle <= 2e-3


def test_route_topk_bit_exact():
    cfg = workloads.MoEConfig("topk", T=1000, H=128, I=128, E=256, k=8, seed=5, zipf_s=1.1,
                              forced_empty=16)
    logits = workloads.gen_logits(cfg)
    ids, w = w4.w4a8_moe_route_topk(logits.cuda(), cfg.k)
    rid, rw = oracle.route_topk(logits.numpy(), cfg.k)
    assert np.array_equal(ids.cpu().numpy(), rid)
    assert np.allclose(w.cpu().numpy(), rw, rtol=1e-6, atol=1e-30)


def test_padding_slots_and_bad_ids():
    cfg = workloads.MoEConfig("ep_pad", T=24, H=256, I=128, E=4, k=2, seed=21)
    hidden, logits, w13, w2 = small_case(cfg)
    layer = w4.W4A8MoELayer.from_bf16(w13.cuda(), w2.cuda(), cfg.k)
    codes, scales = w4.w4a8_quant_act_fp8_per_token(hidden.cuda())
    ids, w = w4.w4a8_moe_route_topk(logits.cuda(), cfg.k)
    b, n, wl = _share(layer, 0, 1)
    base = w4.w4a8_moe_forward_experts(codes, scales, ids, w, cfg.E, b, *wl)
    # slot 1 of tokens 3 and 5 emptied (-1): their contribution disappears
    ids_pad = ids.clone()
    ids_pad[3, 1] = -1
    ids_pad[5, 1] = -1
    got = w4.w4a8_moe_forward_experts(codes, scales, ids_pad, w, cfg.E, b, *wl)
    w4.w4a8_check_device_error()
    keep = [t for t in range(cfg.T) if t not in (3, 5)]
    assert rel_fro(got[keep].cpu().numpy(), base[keep].cpu().numpy()) <= 1e-6
    print(f"\n[padding] other tokens bit-equal: {torch.equal(got[keep], base[keep])}")
    w_pad = w.clone()
    w_pad[3, 1] = 0.0
    w_pad[5, 1] = 0.0
    again = w4.w4a8_moe_forward_experts(codes, scales, ids, w_pad, cfg.E, b, *wl)
    assert rel_fro(got[[3, 5]].cpu().numpy(), again[[3, 5]].cpu().numpy()) <= 1e-6
    # an id outside [-1, E) is skipped on the device and reported
    ids_bad = ids_pad.clone()
    ids_bad[3, 1] = cfg.E + 3
    ids_bad[5, 1] = -7
    bad = w4.w4a8_moe_forward_experts(codes, scales, ids_bad, w, cfg.E, b, *wl)
    with pytest.raises(w4.W4A8Error, match="DEVICE_INDEX"):
        w4.w4a8_check_device_error()
    assert torch.equal(bad, got)
    w4.w4a8_check_device_error()            # the latch was cleared


def test_decode_workload_split_over_eight_shares():
    # the decode workload's experts split over 8 shares, 8 x 64 gathered tokens
    cfg = workloads.CONFIGS[1].with_(T=512, name="decode_ep8")
    dev = torch.device("cuda")
    E, H, I = cfg.E, cfg.H, cfg.I
    p13 = torch.empty(E, 2 * I, H // 8, dtype=torch.int32, device=dev)
    s13 = torch.empty(E, 2 * I, H // 128, dtype=torch.bfloat16, device=dev)
    p2 = torch.empty(E, H, I // 8, dtype=torch.int32, device=dev)
    s2 = torch.empty(E, H, I // 128, dtype=torch.bfloat16, device=dev)
    for e in range(E):
        a, b_ = workloads.gen_expert_weights(cfg, e, device=dev)
        w4.w4a8_pack_int4(a, packed=p13[e], scales=s13[e])
        w4.w4a8_pack_int4(b_, packed=p2[e], scales=s2[e])
    p13, s13 = w4.w4a8_prepare_experts_b200(p13, s13, packed_out=p13)
    p2, s2 = w4.w4a8_prepare_experts_b200(p2, s2, packed_out=p2)
    layer = w4.W4A8MoELayer(p13, s13, p2, s2, cfg.k)
    hidden = workloads.gen_hidden(cfg, device=dev)
    logits = workloads.gen_logits(cfg, device=dev)
    aux = dict(act_codes=torch.empty(cfg.T, H, dtype=torch.uint8, device=dev),
               act_scales=torch.empty(cfg.T, dtype=torch.float32, device=dev),
               topk_ids=torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=dev),
               topk_w=torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=dev))
    ref = layer(hidden, logits, aux=aux)
    out = _emulated_ep(layer, aux["act_codes"], aux["act_scales"], aux["topk_ids"],
                       aux["topk_w"], 8)
    same, dist = _agreement(out, ref)
    print(f"\n[decode, 8 shares of 32 experts, 512 tokens] vs layer: {same:.5f} bit-equal, "
          f"rel-Frobenius {dist:.2e}")
    assert same >= 0.999 and dist <= 1e-4
