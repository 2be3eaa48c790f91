"""GPU parity of the expert-parallel entry points on one GPU.

Expert parallelism splits the experts over ranks; here every rank's share is
computed on the one GPU in turn (no rank waits on another), from the same
gathered tokens: w4a8_moe_forward_experts over each rank's expert range, the
float32 partial sums added, and one bf16 rounding (w4a8_cast_f32_bf16).  The
result must match w4a8_moe_forward on the whole layer (up to float32
summation order) and the oracle (relative Frobenius 2e-3).  Also: the
top-k-only routing call is bit-exact against the oracle, and an expert id
outside [-1, E) is skipped and reported by the device latch.  The
all-to-all(v) form: the dispatch plan, row gather and combine are bit-exact
against their definition, and whole emulated steps of several ranks (the
collectives as slices on the one GPU) match the layer on each rank's tokens.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a8_quantized_moe_b200 as w4
from ep_reference import combine_reference, plan_reference
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


# ------------------------------------------------ all-to-all(v) dispatch
@pytest.mark.parametrize("T,k,E,n,pad", [
    (0, 2, 6, 3, 0.0), (1, 1, 4, 1, 0.0), (37, 3, 6, 4, 0.1), (3000, 8, 256, 8, 0.05),
    (500, 4, 7, 3, 0.0), (200, 2, 3, 5, 0.0), (1100, 8, 256, 64, 0.0), (64, 8, 256, 1, 0.0),
], ids=lambda v: str(v))
def test_dispatch_plan_bit_exact(T, k, E, n, pad):
    g = np.random.default_rng(T * 31 + E)
    ids = g.integers(0, E, size=(T, k)).astype(np.int32)
    ids[g.random((T, k)) < pad] = -1                  # empty slots go nowhere
    counts, rows, pos = w4.w4a8_ep_dispatch_plan(torch.from_numpy(ids).cuda(), E, n)
    rc, rr, rp = plan_reference(ids, E, n)
    m = int(rc.sum())
    assert torch.equal(counts.cpu(), rc)
    assert torch.equal(rows.cpu()[:m], rr[:m])
    assert torch.equal(pos.cpu(), rp)


def test_gather_and_combine_rows_bit_exact():
    g = np.random.default_rng(3)
    T, H, k, n = 333, 384, 4, 5
    codes = torch.from_numpy(g.integers(0, 256, size=(T, H), dtype=np.uint8)).cuda()
    scales = torch.from_numpy(g.random(T, dtype=np.float32)).cuda()
    ids = torch.from_numpy(g.integers(-1, 20, size=(T, k)).astype(np.int32)).cuda()
    w = torch.from_numpy(g.random((T, k), dtype=np.float32)).cuda()
    counts, rows, pos = w4.w4a8_ep_dispatch_plan(ids, 20, n)
    m = int(counts.sum())
    c, s, i, ww = w4.w4a8_ep_gather_rows(codes, scales, ids, w, rows, m)
    r = rows[:m].long()
    assert torch.equal(c, codes[r]) and torch.equal(s, scales[r])
    assert torch.equal(i, ids[r]) and torch.equal(ww, w[r])
    back = torch.from_numpy(g.standard_normal((m, H)).astype(np.float32) * 3).cuda()
    out = w4.w4a8_ep_combine_rows(back, pos)
    ref = combine_reference(back.cpu().numpy(), pos.cpu().numpy())
    bits = oracle.f64_to_bf16_bits(ref.astype(np.float64))
    assert np.array_equal(out.cpu().view(torch.int16).numpy().view(np.uint16), bits)
    none = (pos.cpu() < 0).all(dim=1)                 # tokens that went nowhere: zeros
    assert not out.cpu()[none].any()


@pytest.mark.parametrize("cfg,G,tokens", [
    (workloads.MoEConfig("a2a_ragged", T=0, H=384, I=256, E=6, k=3, seed=31), 4, [37, 0, 5, 64]),
    (workloads.MoEConfig("a2a_zipf", T=0, H=256, I=256, E=16, k=4, seed=32, zipf_s=1.1,
                         forced_empty=5), 8, [50, 20, 1, 0, 33, 16, 64, 9]),
    (workloads.MoEConfig("a2a_wide", T=0, H=256, I=128, E=4, k=2, seed=33), 3, [300, 129, 70]),
], ids=lambda x: getattr(x, "name", str(x)))
def test_all_to_all_step_emulated(cfg, G, tokens):
    """G ranks' all-to-all(v) steps on one GPU: the collectives are slices of
    the send buffers in source-rank order; each rank's output must match the
    layer on its own tokens."""
    ws = [workloads.gen_expert_weights(cfg, e) for e in range(cfg.E)]
    w13 = torch.stack([a for a, _ in ws]).cuda()
    w2 = torch.stack([b for _, b in ws]).cuda()
    layer = w4.W4A8MoELayer.from_bf16(w13, w2, cfg.k)
    batches = []
    for s, T in enumerate(tokens):
        c = cfg.with_(T=T, seed=cfg.seed + 7 * s)
        hidden, logits = workloads.gen_hidden(c).cuda(), workloads.gen_logits(c).cuda()
        codes, scales = w4.w4a8_quant_act_fp8_per_token(hidden)
        ids, w = w4.w4a8_moe_route_topk(logits, cfg.k)
        counts, rows, pos = w4.w4a8_ep_dispatch_plan(ids, cfg.E, G)
        send = w4.w4a8_ep_gather_rows(codes, scales, ids, w, rows, int(counts.sum()))
        batches.append((hidden, logits, counts.tolist(), send, pos))
    offs = [np.concatenate([[0], np.cumsum(b[2])]) for b in batches]
    parts = {}
    for r in range(G):                                 # rank r: rows from every source
        recv = [torch.cat([b[3][f][offs[s][r]:offs[s][r + 1]] for s, b in enumerate(batches)])
                for f in range(4)]
        b_, n_ = expert_partition(cfg.E, G)[r]
        partial = torch.zeros(recv[0].shape[0], cfg.H, dtype=torch.float32, device="cuda")
        if n_ and recv[0].shape[0]:
            wl = (layer.w13_packed[b_:b_ + n_], layer.w13_scales[b_:b_ + n_],
                  layer.w2_packed[b_:b_ + n_], layer.w2_scales[b_:b_ + n_])
            partial = w4.w4a8_moe_forward_experts(*recv, cfg.E, b_, *wl)
        o = 0
        for s, b in enumerate(batches):                # split back by source
            m = b[2][r]
            parts[(s, r)] = partial[o:o + m]
            o += m
    w4.w4a8_check_device_error()
    for s, (hidden, logits, counts, _, pos) in enumerate(batches):
        back = torch.cat([parts[(s, r)] for r in range(G)])
        out = w4.w4a8_ep_combine_rows(back, pos)
        if hidden.shape[0] == 0:
            assert out.shape == (0, cfg.H)
            continue
        ref = layer(hidden, logits)
        same, dist = _agreement(out, ref)
        print(f"\n[{cfg.name}, rank {s} of {G}, {hidden.shape[0]} tokens] vs layer: "
              f"{same:.5f} bit-equal, rel-Frobenius {dist:.2e}")
        assert same >= 0.999 and dist <= 1e-4


def test_bad_send_rows_are_reported_by_the_debug_build():
    """Only on the bounds-checking build (W4A8_LIBRARY=debug): a send-row
    index outside [0, T) and a send-list index outside [0, n_rows) are skipped
    and raise the device latch.  The release build does not check them, so the
    test does not run there."""
    if not w4.w4a8_build_flags() & 1:
        pytest.skip("release build: indices are not checked")
    T, H, k = 8, 128, 2
    codes = torch.zeros(T, H, dtype=torch.uint8, device="cuda")
    scales = torch.ones(T, dtype=torch.float32, device="cuda")
    ids = torch.zeros(T, k, dtype=torch.int32, device="cuda")
    w = torch.ones(T, k, dtype=torch.float32, device="cuda")
    rows = torch.tensor([0, 3, T + 5, 1], dtype=torch.int32, device="cuda")
    c, s, i, ww = w4.w4a8_ep_gather_rows(codes, scales, ids, w, rows, 4)
    with pytest.raises(w4.W4A8Error, match="DEVICE_INDEX"):
        w4.w4a8_check_device_error()
    back = torch.ones(4, H, dtype=torch.float32, device="cuda")
    pos = torch.full((T, 2), -1, dtype=torch.int32, device="cuda")
    pos[0, 0], pos[1, 1], pos[2, 0] = 0, 9, 3          # 9 is past the 4 rows
    out = w4.w4a8_ep_combine_rows(back, pos)
    with pytest.raises(w4.W4A8Error, match="DEVICE_INDEX"):
        w4.w4a8_check_device_error()
    assert out[0].float().eq(1).all() and out[1].float().eq(0).all()
    w4.w4a8_check_device_error()                       # the latch was cleared
