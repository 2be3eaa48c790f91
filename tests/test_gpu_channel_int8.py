"""GPU parity of the per-channel INT4 / per-token INT8 variant against the
oracle ("GLM-5.3-Channel-INT4-w4a8" model card quantisation table).

Bit-exact: per-channel packed words and bf16 scales, the prepared words and
nibble sums, routing, permutation, the input INT8 codes and scales.  Within
tolerance: the intermediate INT8 codes (a code may move by one step where the
float32 and float64 values of h straddle a rounding midpoint), h and the Y
rows (relative Frobenius 1e-4; the dot products are exact integers on both
sides) and the bf16 output (relative Frobenius 2e-3).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a8_quantized_moe_b200 as w4
from gpu_helpers import aux_buffers, bf16_bits, f64, rel_fro, repack_b200, small_case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("R,K", [(1, 128), (9, 384), (64, 6144), (300, 2048)])
def test_pack_channel_bit_exact(R, K):
    g = torch.Generator().manual_seed(R + K)
    w = (torch.randn(R, K, generator=g) * 0.02 * torch.exp(torch.randn(R, 1, generator=g)))
    w = w.to(torch.bfloat16)
    w[0, :] = 0.0 if R > 1 else w[0, :]
    packed, scales = w4.w4a8_pack_int4_channel(w.cuda())
    q, s = oracle.rtn_quantize_int4_channel(f64(w))
    assert np.array_equal(packed.cpu().numpy(), oracle.pack_uint4b8(q))
    assert np.array_equal(bf16_bits(scales), oracle.f64_to_bf16_bits(s[:, 0]))


def test_prepare_channel_words_and_sums():
    g = torch.Generator().manual_seed(3)
    words = torch.randint(-2**31, 2**31, (3, 40, 64), generator=g, dtype=torch.int64).to(torch.int32)
    src = words.cuda()
    out, sums = w4.w4a8_prepare_experts_channel_b200(src)
    assert np.array_equal(out.cpu().numpy(), repack_b200(words.numpy()))
    u = words.numpy().view(np.uint32).astype(np.int64)
    ref = sum(((u >> (4 * j)) & 0xF) for j in range(8)).sum(axis=-1)
    assert np.array_equal(sums.cpu().numpy(), ref)


def _compare(cfg, hidden, logits, w13, w2):
    E, k, T, H, I = cfg.E, cfg.k, hidden.shape[0], cfg.H, cfg.I
    layer = w4.W4A8ChannelInt8Layer.from_bf16(w13.cuda(), w2.cuda(), k)
    aux = aux_buffers(T, H, I, E, k)
    out = layer(hidden.cuda(), logits.cuda(), aux=aux)
    w4.w4a8_check_device_error()
    store = oracle.ExpertStore(E, lambda e: (f64(w13[e]), f64(w2[e])),
                               quantize=oracle.rtn_quantize_int4_channel)
    res = oracle.moe_forward(f64(hidden), logits.numpy(), store, k, act_format="int8")

    assert np.array_equal(aux["topk_ids"].cpu().numpy(), res["topk_ids"])
    assert np.array_equal(aux["sorted_token_ids"].cpu().numpy(), res["sorted_token_ids"])
    assert np.array_equal(aux["row_of"].cpu().numpy(), res["row_of"])
    codes = aux["act_codes"].cpu().numpy().astype(np.int64) - 128      # stored offset-binary
    assert np.array_equal(codes, res["act_codes"].astype(np.int64))
    assert np.array_equal(aux["act_scales"].cpu().numpy().astype(np.float64), res["act_scales"])
    rows = sorted(res["inter_h"].keys())
    e_h = rel_fro(aux["inter_h"].cpu().numpy()[rows], np.stack([res["inter_h"][r] for r in rows]))
    gc = aux["inter_codes"].cpu().numpy()[rows].astype(np.int64) - 128
    oc = np.stack([res["inter_codes"][r] for r in rows]).astype(np.int64)
    frac, dist = float(np.mean(gc == oc)), int(np.abs(gc - oc).max(initial=0))
    e_y = rel_fro(aux["y_rows"].cpu().numpy()[rows], np.stack([res["y_rows"][r] for r in rows]))
    e_out = rel_fro(f64(out), res["out"])
    print(f"\n[{cfg.name} int8] h {e_h:.2e}  codes {frac:.6f} (max step {dist})  Y {e_y:.2e}  "
          f"out {e_out:.2e}")
    assert e_h <= 1e-4 and frac >= 0.999 and dist <= 1
    assert e_y <= 1e-3 and e_out <= 2e-3


@pytest.mark.parametrize("cfg", [
    workloads.CONFIGS[0],
    workloads.MoEConfig("single_token_dense", T=1, H=128, I=128, E=1, k=1, seed=11),
    workloads.MoEConfig("ragged", T=37, H=384, I=256, E=6, k=3, seed=13),
    workloads.MoEConfig("multi_block_segments", T=300, H=256, I=128, E=2, k=2, seed=14),
    workloads.MoEConfig("zipf_empty", T=200, H=256, I=256, E=16, k=4, seed=15, zipf_s=1.1,
                        forced_empty=5),
    workloads.MoEConfig("decode_shape_multi_block", T=96, H=256, I=128, E=8, k=2, seed=17,
                        zipf_s=1.1),
], ids=lambda c: c.name)
def test_forward_channel_int8(cfg):
    _compare(cfg, *small_case(cfg))


@pytest.mark.parametrize("ci", [1, 3], ids=lambda i: workloads.CONFIGS[i].name)
def test_forward_channel_int8_full_size_sampled(ci):
    """Full-size decode and prefill workloads in the launch configuration the
    bench times: routing and input codes checked for all tokens, the output
    for a seeded sample of tokens."""
    import bench
    cfg = workloads.CONFIGS[ci]
    dev = torch.device("cuda")
    layer = bench.build_layer(cfg, dev, w4, "channel-int8")
    hidden = workloads.gen_hidden(cfg, device=dev)
    logits = workloads.gen_logits(cfg, device=dev)
    T, k, E = cfg.T, cfg.k, cfg.E
    aux = dict(topk_ids=torch.empty(T, k, dtype=torch.int32, device=dev),
               act_codes=torch.empty(T, cfg.H, dtype=torch.uint8, device=dev),
               act_scales=torch.empty(T, dtype=torch.float32, device=dev))
    out = layer(hidden, logits, aux=aux)
    w4.w4a8_check_device_error()
    rng = np.random.default_rng(ci)
    toks = np.unique(np.concatenate([[0, T - 1], rng.choice(T, 3, replace=False)]))
    h_host = hidden[torch.as_tensor(toks, device=dev)].cpu()

    def weights(e):
        a, b = workloads.gen_expert_weights(cfg, e, device=dev)
        return f64(a), f64(b)

    store = oracle.ExpertStore(E, weights, quantize=oracle.rtn_quantize_int4_channel)
    res = oracle.moe_forward(None, logits.cpu().numpy(), store, k, tokens=toks,
                             hidden_of_tokens=f64(h_host), act_format="int8")
    assert np.array_equal(aux["topk_ids"].cpu().numpy(), res["topk_ids"])
    for t0 in range(0, T, 4096):
        rc, rs = oracle.quant_act_int8_per_token(f64(hidden[t0:t0 + 4096]))
        got = aux["act_codes"][t0:t0 + 4096].cpu().numpy().astype(np.int64) - 128
        assert np.array_equal(got, rc.astype(np.int64))
    e_out = rel_fro(f64(out[torch.as_tensor(toks, device=dev)]), res["out"])
    print(f"\n[{cfg.name} int8] sampled tokens {toks.tolist()} out rel-Frobenius {e_out:.2e}")
    assert e_out <= 2e-3
