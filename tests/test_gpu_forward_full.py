"""GPU parity at the full workload sizes, in the launch configuration bench.py
times (all experts packed on the device, one w4a8_moe_forward per batch).

Routing, the permutation and the input activation codes are compared
bit-exact for all tokens; the packed weights of every expert the sample
touches are compared bit-exact; the oracle computes the layer for a seeded
sample of tokens (it finishes those one by one), whose output rows must be
within relative Frobenius 2e-3 of the GPU rows.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a8_quantized_moe_b200 as w4
from gpu_helpers import bf16_bits, codes_agree, f64, rel_fro, repack_b200

pytestmark = pytest.mark.gpu

SAMPLE_TOKENS = 3


def _pack_all(cfg, device):
    E, H, I = cfg.E, cfg.H, cfg.I
    p13 = torch.empty(E, 2 * I, H // 8, dtype=torch.int32, device=device)
    s13 = torch.empty(E, 2 * I, H // 128, dtype=torch.bfloat16, device=device)
    p2 = torch.empty(E, H, I // 8, dtype=torch.int32, device=device)
    s2 = torch.empty(E, H, I // 128, dtype=torch.bfloat16, device=device)
    for e in range(E):
        w13, w2 = workloads.gen_expert_weights(cfg, e, device=device)
        w4.w4a8_pack_int4(w13, packed=p13[e], scales=s13[e])
        w4.w4a8_pack_int4(w2, packed=p2[e], scales=s2[e])
    p13, s13 = w4.w4a8_prepare_experts_b200(p13, s13, packed_out=p13)
    p2, s2 = w4.w4a8_prepare_experts_b200(p2, s2, packed_out=p2)
    return w4.W4A8MoELayer(p13, s13, p2, s2, cfg.k)


@pytest.mark.parametrize("ci", [1, 2, 3, 4], ids=lambda i: workloads.CONFIGS[i].name)
def test_forward_full_size_sampled(ci):
    cfg = workloads.CONFIGS[ci]
    dev = torch.device("cuda")
    layer = _pack_all(cfg, dev)
    hidden = workloads.gen_hidden(cfg, device=dev)
    logits = workloads.gen_logits(cfg, device=dev)
    T, k, E = cfg.T, cfg.k, cfg.E
    aux = dict(topk_ids=torch.empty(T, k, dtype=torch.int32, device=dev),
               topk_w=torch.empty(T, k, dtype=torch.float32, device=dev),
               expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
               sorted_token_ids=torch.empty(T * k, dtype=torch.int32, device=dev),
               row_of=torch.empty(T, k, dtype=torch.int32, device=dev),
               act_codes=torch.empty(T, cfg.H, dtype=torch.uint8, device=dev),
               act_scales=torch.empty(T, dtype=torch.float32, device=dev))
    out = layer(hidden, logits, aux=aux)
    w4.w4a8_check_device_error()

    rng = np.random.default_rng(ci)
    toks = np.unique(np.concatenate([[0, T - 1], rng.choice(T, SAMPLE_TOKENS, replace=False)]))
    l_host = logits.cpu().numpy()
    h_host = hidden[torch.as_tensor(toks, device=dev)].cpu()

    def weights(e):
        a, b = workloads.gen_expert_weights(cfg, e, device=dev)
        return f64(a), f64(b)

    store = oracle.ExpertStore(E, weights)
    # the oracle sees the sampled tokens' hidden rows; routing covers all T
    res = oracle.moe_forward(None, l_host, store, k, tokens=toks, hidden_of_tokens=f64(h_host))

    assert np.array_equal(aux["topk_ids"].cpu().numpy(), res["topk_ids"])
    assert np.array_equal(aux["expert_offsets"].cpu().numpy(), res["expert_offsets"])
    assert np.array_equal(aux["sorted_token_ids"].cpu().numpy(), res["sorted_token_ids"])
    assert np.array_equal(aux["row_of"].cpu().numpy(), res["row_of"])
    assert np.allclose(aux["topk_w"].cpu().numpy(), res["topk_w"], rtol=1e-6, atol=1e-30)
    # activation codes of every token (bit-exact) against the oracle quantiser
    for t0 in range(0, T, 4096):
        rc, rs = oracle.quant_act_fp8_per_token(f64(hidden[t0:t0 + 4096]))
        assert np.array_equal(aux["act_codes"][t0:t0 + 4096].cpu().numpy(), rc)
        assert np.array_equal(aux["act_scales"][t0:t0 + 4096].cpu().numpy().astype(np.float64), rs)
    # packed weights of the touched experts (bit-exact)
    for e in sorted(set(res["topk_ids"][toks].reshape(-1).tolist())):
        p13, s13, p2, s2 = store[e]
        assert np.array_equal(layer.w13_packed[e].cpu().numpy(), repack_b200(p13))
        assert np.array_equal(bf16_bits(layer.w13_scales[e].t()), oracle.f64_to_bf16_bits(s13))
        assert np.array_equal(layer.w2_packed[e].cpu().numpy(), repack_b200(p2))
        assert np.array_equal(bf16_bits(layer.w2_scales[e].t()), oracle.f64_to_bf16_bits(s2))
    e_out = rel_fro(f64(out[torch.as_tensor(toks, device=dev)]), res["out"])
    counts = np.diff(res["expert_offsets"].astype(np.int64))
    print(f"\n[{cfg.name}] sampled tokens {toks.tolist()} out rel-Frobenius {e_out:.2e}; "
          f"active experts {np.count_nonzero(counts)}, max segment {counts.max()}")
    assert e_out <= 2e-3, e_out
    if cfg.forced_empty:
        fe = workloads.forced_empty_experts(cfg).numpy()
        assert np.all(counts[fe] == 0)
