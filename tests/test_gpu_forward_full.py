"""GPU parity at the full workload sizes, in the launch configuration bench.py
times (all experts packed on the device, one w4a8_moe_forward per batch).

For every token: routing, the permutation and the input activation codes are
compared bit-exact.  For a sample of tokens the oracle computes the layer
(one expert at a time, in a pool of worker processes), and the library's
intermediate values of those tokens' segment rows are compared element by
element through the forward's aux buffers: the SwiGLU output h, the
intermediate E4M3 codes and scales, and the down-projection rows Y; then the
output rows.  The sample is the first and last token, 32 random tokens, and
the tokens of the rows that sit on tile boundaries of the three largest
expert segments, for both tile widths of the grouped GEMM (32 and 128 rows):
the first and last row of the first tile, of a middle tile, of the last full
tile and of the partial last tile.  The packed words and scales of every
expert the sample touches are compared bit-exact (by digest).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a8_quantized_moe_b200 as w4
from gpu_helpers import bf16_bits, boundary_rows, codes_agree, f64, rel_fro
from oracle_pool import OraclePool, digest, unrepack_b200

pytestmark = pytest.mark.gpu

RANDOM_TOKENS = 32
OUT_TOL = 2e-3              # final bf16 output, relative Frobenius
H_TOL = 1e-4                # h per row (float32 GEMM vs float64), relative
Y_TOL = 1e-3                # Y rows together, relative Frobenius
CODE_MATCH = 0.999          # fraction of intermediate E4M3 codes equal to the oracle's


@pytest.fixture(scope="module")
def pool():
    p = OraclePool()
    yield p
    p.close()


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
def test_forward_full_size_sampled(ci, pool):
    cfg = workloads.CONFIGS[ci]
    dev = torch.device("cuda")
    layer = _pack_all(cfg, dev)
    hidden = workloads.gen_hidden(cfg, device=dev)
    logits = workloads.gen_logits(cfg, device=dev)
    T, H, I, k, E = cfg.T, cfg.H, cfg.I, cfg.k, cfg.E
    A = T * k
    aux = dict(topk_ids=torch.empty(T, k, dtype=torch.int32, device=dev),
               topk_w=torch.empty(T, k, dtype=torch.float32, device=dev),
               expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
               sorted_token_ids=torch.empty(A, dtype=torch.int32, device=dev),
               row_of=torch.empty(T, k, dtype=torch.int32, device=dev),
               act_codes=torch.empty(T, H, dtype=torch.uint8, device=dev),
               act_scales=torch.empty(T, dtype=torch.float32, device=dev),
               inter_h=torch.empty(A, I, dtype=torch.float32, device=dev),
               inter_codes=torch.empty(A, I, dtype=torch.uint8, device=dev),
               inter_scales=torch.empty(A, dtype=torch.float32, device=dev),
               y_rows=torch.empty(A, H, dtype=torch.float32, device=dev))
    out = layer(hidden, logits, aux=aux)
    w4.w4a8_check_device_error()

    # routing and permutation of all T tokens (bit-exact), by the oracle
    l_host = logits.cpu().numpy()
    ids, wts = oracle.route_topk(l_host, k)
    offsets, sorted_tok, row_of = oracle.permute_by_expert(ids, E)
    assert np.array_equal(aux["topk_ids"].cpu().numpy(), ids)
    assert np.array_equal(aux["expert_offsets"].cpu().numpy(), offsets)
    assert np.array_equal(aux["sorted_token_ids"].cpu().numpy(), sorted_tok)
    assert np.array_equal(aux["row_of"].cpu().numpy(), row_of)
    assert np.allclose(aux["topk_w"].cpu().numpy(), wts, rtol=1e-6, atol=1e-30)
    # activation codes of every token (bit-exact) against the oracle quantiser
    for t0 in range(0, T, 4096):
        rc, rs = oracle.quant_act_fp8_per_token(f64(hidden[t0:t0 + 4096]))
        assert np.array_equal(aux["act_codes"][t0:t0 + 4096].cpu().numpy(), rc)
        assert np.array_equal(aux["act_scales"][t0:t0 + 4096].cpu().numpy().astype(np.float64), rs)

    # the sample: boundary rows of the largest segments, random tokens, ends
    rng = np.random.default_rng(ci)
    b_rows = boundary_rows(offsets)
    toks = np.unique(np.concatenate([[0, T - 1], rng.choice(T, RANDOM_TOKENS, replace=False),
                                     sorted_tok[b_rows]])).astype(np.int64)
    h_host = hidden[torch.as_tensor(toks, device=dev)].cpu()

    def weight_bits(e):
        a, b = workloads.gen_expert_weights(cfg, e, device=dev)
        return bf16_bits(a), bf16_bits(b)

    res = oracle.moe_forward(None, l_host, None, k, tokens=toks, hidden_of_tokens=f64(h_host),
                             expert_map=pool.expert_map(weight_bits))

    # packed words and scales of every touched expert (bit-exact, by digest)
    touched = sorted(set(ids[toks].reshape(-1).tolist()))
    for e in touched:
        got = digest(unrepack_b200(layer.w13_packed[e].cpu().numpy()),
                     bf16_bits(layer.w13_scales[e].t()),
                     unrepack_b200(layer.w2_packed[e].cpu().numpy()),
                     bf16_bits(layer.w2_scales[e].t()))
        assert got == pool.digests[e], f"expert {e}: packed weights differ from the oracle's"

    # every segment row of the sampled tokens, element by element
    rows = np.array(sorted(res["inter_h"].keys()), dtype=np.int64)
    assert set(b_rows.tolist()) <= set(rows.tolist())
    ridx = torch.as_tensor(rows, device=dev)
    gh = aux["inter_h"][ridx].cpu().numpy().astype(np.float64)
    oh = np.stack([res["inter_h"][r] for r in rows])
    gc = aux["inter_codes"][ridx].cpu().numpy()
    oc = np.stack([res["inter_codes"][r] for r in rows])
    gs = aux["inter_scales"][ridx].cpu().numpy().astype(np.float64)
    os_ = np.array([res["inter_scales"][r] for r in rows])
    gy = aux["y_rows"][ridx].cpu().numpy().astype(np.float64)
    oy = np.stack([res["y_rows"][r] for r in rows])
    e_h = np.array([rel_fro(a, b) for a, b in zip(gh, oh)])
    e_y = np.array([rel_fro(a, b) for a, b in zip(gy, oy)])
    frac, dist = codes_agree(gc, oc)
    o_rows = f64(out[torch.as_tensor(toks, device=dev)])
    e_out = rel_fro(o_rows, res["out"])
    e_tok = np.array([rel_fro(a, b) for a, b in zip(o_rows, res["out"])])
    counts = np.diff(offsets.astype(np.int64))
    print(f"\n[{cfg.name}] {len(toks)} tokens, {len(rows)} segment rows "
          f"({len(b_rows)} on tile boundaries), {len(touched)} experts: max row error h "
          f"{e_h.max():.2e}, Y {e_y.max():.2e} (all rows {rel_fro(gy, oy):.2e}); codes "
          f"{frac:.6f} equal (max step {dist}); "
          f"out {e_out:.2e} (worst token {e_tok.max():.2e}); active experts "
          f"{np.count_nonzero(counts)}, max segment {counts.max()}")
    assert e_h.max() <= H_TOL, e_h.max()
    assert frac >= CODE_MATCH and dist <= 1, (frac, dist)
    assert np.allclose(gs, os_, rtol=1e-5, atol=0)
    # a one-step code difference moves its row's Y by up to a few 1e-3, so rows
    # are held to the float32 accumulation bound only where every code agrees
    exact_rows = np.all(gc == oc, axis=1)
    assert e_y[exact_rows].max(initial=0.0) <= H_TOL, e_y[exact_rows].max(initial=0.0)
    assert rel_fro(gy, oy) <= Y_TOL, rel_fro(gy, oy)
    assert e_out <= OUT_TOL, e_out
    # per token, where every code of the token's rows agrees (a one-step code
    # difference, a float32-vs-float64 midpoint, moves a token by up to ~3e-3)
    row_ok = dict(zip(rows.tolist(), exact_rows.tolist()))
    tok_ok = np.array([all(row_ok[int(r)] for r in row_of[t]) for t in toks])
    assert e_tok[tok_ok].max(initial=0.0) <= OUT_TOL, e_tok[tok_ok].max(initial=0.0)
    if cfg.forced_empty:
        fe = workloads.forced_empty_experts(cfg).numpy()
        assert np.all(counts[fe] == 0)

