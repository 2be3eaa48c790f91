"""GPU parity of the FP8 128 x 128-block shared expert against the oracle
(GLM-5.3-W4A8 model card, intro and "quantisation method": the shared expert
keeps E4M3 weights with one scale per 128 x 128 block).

Bit-exact: block codes and scales, the input's group codes and scales.
Within tolerance: h (relative Frobenius 1e-4: float32 accumulation), the
intermediate codes (>= 99.9 % equal, the rest one step: float32 and float64 h
may straddle a rounding midpoint), the expert output y (1e-3) and the layer
output with the routed experts (2e-3).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a8_quantized_moe_b200 as w4
from gpu_helpers import aux_buffers, codes_agree, f64, rel_fro, small_case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("R,K", [(128, 128), (256, 384), (512, 6144), (6144, 256)])
def test_quant_fp8_block_bit_exact(R, K):
    g = torch.Generator().manual_seed(R * 7 + K)
    w = torch.randn(R, K, generator=g) * 0.02
    w *= torch.exp(torch.randn(R // 128, 1, K // 128, 1, generator=g) * 2).expand(
        R // 128, 128, K // 128, 128).reshape(R, K)
    w[:128, :128] = 0.0                                     # an all-zero block
    w = w.to(torch.bfloat16)
    codes, scales = w4.w4a8_quant_fp8_block(w.cuda())
    rc, rs = oracle.quant_fp8_block(f64(w))
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales.cpu().numpy().astype(np.float64), rs)


@pytest.mark.parametrize("T,H", [(1, 128), (5, 384), (300, 6144), (4097, 256)])
def test_quant_act_fp8_group_bit_exact(T, H):
    g = torch.Generator().manual_seed(T + H)
    x = torch.randn(T, H, generator=g) * torch.exp(torch.randn(T, 1, generator=g) * 2)
    x[0, :128] = 0.0
    if H > 128:
        x[:, 130] *= 40.0
    x = x.to(torch.bfloat16)
    codes, scales = w4.w4a8_quant_act_fp8_group(x.cuda())
    rc, rs = oracle.quant_act_fp8_group(f64(x))
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales.cpu().numpy().astype(np.float64), rs)


def _shared_weights(cfg, device="cpu"):
    ws13, ws2 = workloads.gen_shared_weights(cfg, device=device)
    return ws13, ws2


@pytest.mark.parametrize("T,H,I", [(1, 128, 128), (37, 384, 256), (300, 256, 128),
                                   (130, 1024, 512)])
def test_shared_expert_forward(T, H, I):
    cfg = workloads.MoEConfig("shared", T=T, H=H, I=I, E=1, k=1, seed=T + H + I)
    hidden = workloads.gen_hidden(cfg)
    ws13, ws2 = _shared_weights(cfg)
    sh = w4.SharedExpertFP8.from_bf16(ws13.cuda(), ws2.cuda())
    dev = torch.device("cuda")
    aux = dict(act_codes=torch.empty(T, H, dtype=torch.uint8, device=dev),
               act_scales=torch.empty(T, H // 128, dtype=torch.float32, device=dev),
               h=torch.empty(T, I, dtype=torch.float32, device=dev),
               h_codes=torch.empty(T, I, dtype=torch.uint8, device=dev),
               h_scales=torch.empty(T, I // 128, dtype=torch.float32, device=dev))
    y = sh(hidden.cuda(), aux=aux)
    w4.w4a8_check_device_error()
    w13c, s13 = oracle.quant_fp8_block(f64(ws13))
    w2c, s2 = oracle.quant_fp8_block(f64(ws2))
    assert np.array_equal(sh.weights[0].cpu().numpy(), w13c)
    assert np.array_equal(sh.weights[3].cpu().numpy().astype(np.float64), s2)
    res = oracle.shared_expert_forward(f64(hidden), w13c, s13, w2c, s2)
    assert np.array_equal(aux["act_codes"].cpu().numpy(), res["act_codes"])
    assert np.array_equal(aux["act_scales"].cpu().numpy().astype(np.float64), res["act_scales"])
    e_h = rel_fro(aux["h"].cpu().numpy(), res["h"])
    frac, dist = codes_agree(aux["h_codes"].cpu().numpy(), res["h_codes"])
    e_y = rel_fro(y.cpu().numpy(), res["y"])
    print(f"\n[shared T={T} H={H} I={I}] h {e_h:.2e}  codes {frac:.6f} (max step {dist})  "
          f"y {e_y:.2e}")
    assert e_h <= 1e-4 and frac >= 0.999 and dist <= 1 and e_y <= 1e-3


@pytest.mark.parametrize("cfg", [
    workloads.CONFIGS[0],
    workloads.MoEConfig("ragged", T=37, H=384, I=256, E=6, k=3, seed=13),
    workloads.MoEConfig("multi_block_segments", T=300, H=256, I=128, E=2, k=2, seed=14),
    workloads.MoEConfig("zipf_empty", T=200, H=256, I=256, E=16, k=4, seed=15, zipf_s=1.1,
                        forced_empty=5),
], ids=lambda c: c.name)
def test_layer_with_shared_expert(cfg):
    hidden, logits, w13, w2 = small_case(cfg)
    ws13, ws2 = _shared_weights(cfg)
    layer = w4.W4A8MoELayerShared.from_bf16_with_shared(w13.cuda(), w2.cuda(), cfg.k,
                                                        ws13.cuda(), ws2.cuda())
    out = layer(hidden.cuda(), logits.cuda())
    w4.w4a8_check_device_error()
    store = oracle.ExpertStore(cfg.E, lambda e: (f64(w13[e]), f64(w2[e])))
    sh = (*oracle.quant_fp8_block(f64(ws13)), *oracle.quant_fp8_block(f64(ws2)))
    res = oracle.moe_forward(f64(hidden), logits.numpy(), store, cfg.k, shared=sh)
    e_out = rel_fro(f64(out), res["out"])
    # the shared expert really contributes: without it the output differs
    plain = w4.W4A8MoELayer(layer.w13_packed, layer.w13_scales, layer.w2_packed,
                            layer.w2_scales, cfg.k)(hidden.cuda(), logits.cuda())
    e_plain = rel_fro(f64(plain), res["out"])
    print(f"\n[{cfg.name} + shared] out {e_out:.2e} (routed only: {e_plain:.2e})")
    assert e_out <= 2e-3 and e_plain > 0.05


def _shared_aux(T, H, I):
    dev = "cuda"
    return dict(act_codes=torch.empty(T, H, dtype=torch.uint8, device=dev),
                act_scales=torch.empty(T, H // 128, dtype=torch.float32, device=dev),
                h=torch.empty(T, I, dtype=torch.float32, device=dev),
                h_codes=torch.empty(T, I, dtype=torch.uint8, device=dev),
                h_scales=torch.empty(T, I // 128, dtype=torch.float32, device=dev))


@pytest.mark.parametrize("cfg", [
    workloads.CONFIGS[0],
    workloads.MoEConfig("fused_even_groups", T=48, H=512, I=256, E=16, k=2, seed=41),
    # gate/up K = 384 (three groups: the unpaired decode shape), two shared token blocks
    workloads.MoEConfig("fused_odd_groups", T=100, H=384, I=256, E=32, k=2, seed=42),
    workloads.MoEConfig("fused_one_token", T=1, H=256, I=128, E=8, k=2, seed=43),
], ids=lambda c: c.name)
def test_shared_gemms_inside_the_routed_launches(cfg):
    """Decode-sized, unsplit batches: the shared expert's two GEMMs run as the
    second phase of the routed GEMM launches (64-token tiles).  Its h and y
    must be those of the shared expert's own launches (128-token tiles: the
    same float32 arithmetic per element), and the layer must match the oracle."""
    assert cfg.T * cfg.k <= 32 * cfg.E and cfg.T * cfg.k < 8 * cfg.E   # decode, no split
    hidden, logits, w13, w2 = small_case(cfg)
    ws13, ws2 = _shared_weights(cfg)
    layer = w4.W4A8MoELayerShared.from_bf16_with_shared(w13.cuda(), w2.cuda(), cfg.k,
                                                        ws13.cuda(), ws2.cuda())
    Is = ws2.shape[1]
    fused = _shared_aux(cfg.T, cfg.H, Is)
    aux = aux_buffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    out = layer(hidden.cuda(), logits.cuda(), aux=aux, shared_aux=fused)
    alone = _shared_aux(cfg.T, cfg.H, Is)
    y_alone = layer.shared(hidden.cuda(), aux=alone)
    w4.w4a8_check_device_error()
    assert torch.equal(fused["act_codes"], alone["act_codes"])
    assert torch.equal(fused["act_scales"], alone["act_scales"])
    same_h = float((fused["h"] == alone["h"]).float().mean())
    e_h = rel_fro(fused["h"].cpu().numpy(), alone["h"].cpu().numpy())
    assert e_h <= 1e-6, e_h
    frac, dist = codes_agree(fused["h_codes"].cpu().numpy(), alone["h_codes"].cpu().numpy())
    assert frac >= 0.999 and dist <= 1, (frac, dist)
    # the shared y of the fused down launch: the output is the routed sum from
    # the same call's Y rows plus the shared expert's own y, rounded once to bf16
    Y = aux["y_rows"].double().cpu().numpy()
    w = aux["topk_w"].double().cpu().numpy()
    rows = aux["row_of"].cpu().numpy()
    ys = y_alone.double().cpu().numpy()
    ref = np.einsum("tj,tjh->th", w, Y[rows]) + ys
    # one bf16 rounding (half a unit, 2^-9 relative), float32 summation order
    mag = np.einsum("tj,tjh->th", np.abs(w), np.abs(Y[rows])) + np.abs(ys)
    dev_ = np.abs(f64(out) - ref)
    assert np.all(dev_ <= 2.0 ** -8 * np.abs(ref) + 1e-6 * mag + 1e-30), \
        float((dev_ / (np.abs(ref) + 1e-30)).max())
    store = oracle.ExpertStore(cfg.E, lambda e: (f64(w13[e]), f64(w2[e])))
    sh = (*oracle.quant_fp8_block(f64(ws13)), *oracle.quant_fp8_block(f64(ws2)))
    res = oracle.moe_forward(f64(hidden), logits.numpy(), store, cfg.k, shared=sh)
    e_out = rel_fro(f64(out), res["out"])
    print(f"\n[{cfg.name}] shared h bit-equal {same_h:.5f} (rel {e_h:.1e}) against its own "
          f"launches; layer out {e_out:.2e}")
    assert e_out <= 2e-3


def test_shared_gemms_in_launches_of_their_own():
    """The same decode cases with W4A8_SHARED_FUSED=0 (the shared expert's GEMMs
    in launches of their own), in a child process."""
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    env = dict(os.environ, W4A8_SHARED_FUSED="0")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p",
                        "no:cacheprovider", os.path.join(here, "test_gpu_shared.py"), "-k",
                        "test_layer_with_shared_expert and not full_size"],
                       env=env, capture_output=True, text=True, timeout=600)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-15:])
    assert r.returncode == 0, tail
    assert " passed" in r.stdout, tail


@pytest.mark.parametrize("ci", [1, 3], ids=lambda i: workloads.CONFIGS[i].name)
def test_layer_with_shared_expert_full_size_sampled(ci):
    """Full-size decode and prefill workloads with the shared expert: the output
    for a seeded sample of tokens."""
    import bench
    cfg = workloads.CONFIGS[ci]
    dev = torch.device("cuda")
    layer = bench.build_layer(cfg, dev, w4, "w4a8+shared")
    hidden = workloads.gen_hidden(cfg, device=dev)
    logits = workloads.gen_logits(cfg, device=dev)
    out = layer(hidden, logits)
    w4.w4a8_check_device_error()
    T = cfg.T
    rng = np.random.default_rng(ci + 100)
    toks = np.unique(np.concatenate([[0, T - 1], rng.choice(T, 3, replace=False)]))
    h_host = hidden[torch.as_tensor(toks, device=dev)].cpu()

    def weights(e):
        a, b = workloads.gen_expert_weights(cfg, e, device=dev)
        return f64(a), f64(b)

    ws13, ws2 = workloads.gen_shared_weights(cfg, device=dev)
    sh = (*oracle.quant_fp8_block(f64(ws13)), *oracle.quant_fp8_block(f64(ws2)))
    store = oracle.ExpertStore(cfg.E, weights)
    res = oracle.moe_forward(None, logits.cpu().numpy(), store, cfg.k, tokens=toks,
                             hidden_of_tokens=f64(h_host), shared=sh)
    e_out = rel_fro(f64(out[torch.as_tensor(toks, device=dev)]), res["out"])
    print(f"\n[{cfg.name} + shared] sampled tokens {toks.tolist()} out rel-Frobenius {e_out:.2e}")
    assert e_out <= 2e-3


def test_shared_expert_zero_tokens_and_bad_shapes():
    dev = torch.device("cuda")
    w13 = torch.zeros(256, 256, dtype=torch.bfloat16, device=dev)
    w2 = torch.zeros(256, 128, dtype=torch.bfloat16, device=dev)
    sh = w4.SharedExpertFP8.from_bf16(w13, w2)
    y = sh(torch.zeros(0, 256, dtype=torch.bfloat16, device=dev))
    assert y.shape == (0, 256)
    # all-zero weights: every block scale is 0 and the output is exactly 0
    y = sh(torch.randn(5, 256, device=dev).to(torch.bfloat16))
    w4.w4a8_check_device_error()
    assert torch.count_nonzero(y) == 0
    with pytest.raises(w4.W4A8Error, match="UNSUPPORTED_SHAPE"):
        w4.w4a8_quant_fp8_block(torch.zeros(100, 128, dtype=torch.bfloat16, device=dev))
