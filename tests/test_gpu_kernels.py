"""GPU parity of the standalone entry points against the oracle: INT4 packing,
FP8 activation codes, routing and the permutation are bit-exact."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a8_quantized_moe_b200 as w4
from gpu_helpers import assert_mse_clip_choice, bf16_bits, f64, repack_b200

pytestmark = pytest.mark.gpu


def _weights(R, K, seed):
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(R, K, generator=g) * 0.02 * torch.exp(torch.randn(R, 1, generator=g))
    wb = w.to(torch.bfloat16)
    wb[0, :128] = 0.0                                # all-zero group
    if R > 1:
        wb[1, 5] = -0.0
    if R > 2:                                        # exact .5 ties: amax 7 -> scale 1
        wb[2, :128] = 0.0
        wb[2, :8] = torch.tensor([7.0, 0.5, 1.5, 2.5, -0.5, -2.5, 3.5, -6.5])
    if R > 3:                                        # bf16 subnormals
        wb[3, :128] = (torch.randn(128, generator=g) * 1e-39).to(torch.bfloat16)
    return wb


@pytest.mark.parametrize("R,K", [(1, 128), (7, 256), (64, 6144), (300, 2048), (4096, 512)])
def test_pack_int4_bit_exact(R, K):
    wb = _weights(R, K, R * 131 + K)
    packed, scales = w4.w4a8_pack_int4(wb.cuda())
    q, s = oracle.rtn_quantize_int4(f64(wb))
    assert np.array_equal(packed.cpu().numpy(), oracle.pack_uint4b8(q))
    assert np.array_equal(bf16_bits(scales), oracle.f64_to_bf16_bits(s))


@pytest.mark.parametrize("R,K", [(1, 128), (7, 256), (64, 6144), (300, 2048)])
def test_pack_int4_mse_clip_bit_exact(R, K):
    wb = _weights(R, K, R * 977 + K)
    packed, scales = w4.w4a8_pack_int4(wb.cuda(), mse_clip=True)
    # the kernel sums each candidate's squared error in its own float64 order;
    # it must hold the oracle's exact choice except at near ties within the
    # summation bound, where either tied candidate is correct
    n_ties = assert_mse_clip_choice(packed.cpu().numpy(), bf16_bits(scales), f64(wb))
    print(f"\n[{R}x{K}] groups resolved differently at a near tie: {n_ties}")


def test_pack_int4_3d_and_empty():
    wb = _weights(2 * 64, 256, 5).reshape(2, 64, 256)
    packed, scales = w4.w4a8_pack_int4(wb.cuda())
    assert packed.shape == (2, 64, 32) and scales.shape == (2, 64, 2)
    q, s = oracle.rtn_quantize_int4(f64(wb.reshape(128, 256)))
    assert np.array_equal(packed.reshape(128, 32).cpu().numpy(), oracle.pack_uint4b8(q))
    p0, s0 = w4.w4a8_pack_int4(torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda"))
    assert p0.shape == (0, 32)


@pytest.mark.parametrize("E,rows,K", [(1, 1, 128), (3, 5, 384), (4, 256, 2048), (2, 4096, 6144)])
def test_prepare_experts_bit_exact(E, rows, K):
    g = torch.Generator().manual_seed(E * 7 + rows + K)
    words = torch.randint(-2**31, 2**31, (E, rows, K // 8), generator=g, dtype=torch.int64)
    src = words.to(torch.int32).cuda()
    sc = torch.randn(E, rows, K // 128, generator=g).to(torch.bfloat16).cuda()
    p_out, s_out = w4.w4a8_prepare_experts_b200(src, sc)
    assert np.array_equal(p_out.cpu().numpy(), repack_b200(src.cpu().numpy()))
    assert np.array_equal(bf16_bits(s_out), bf16_bits(sc.transpose(1, 2)))
    expect = p_out.cpu().numpy()
    w4.w4a8_prepare_experts_b200(src, sc, packed_out=src)   # in place gives the same words
    assert np.array_equal(src.cpu().numpy(), expect)


def test_prepare_experts_empty_and_overlap_rejected():
    w4.w4a8_prepare_experts_b200(torch.zeros(0, 4, 16, dtype=torch.int32, device="cuda"),
                                 torch.zeros(0, 4, 1, dtype=torch.bfloat16, device="cuda"))
    buf = torch.zeros(2, 4, 32, dtype=torch.int32, device="cuda")
    sc = torch.zeros(1, 4, 2, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(w4.W4A8Error):   # words partly overlapping
        w4.w4a8_prepare_experts_b200(buf[0:1], sc, packed_out=buf.view(-1)[8:136].view(1, 4, 32))
    scales_buf = torch.zeros(8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(w4.W4A8Error):   # scales_out on top of scales
        w4.w4a8_prepare_experts_b200(buf[0:1], scales_buf.view(1, 4, 2),
                                     scales_out=scales_buf.view(1, 2, 4))


def _acts(T, H, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, H, generator=g) * torch.exp(2 * torch.randn(T, 1, generator=g))
    if H >= 64:
        x[:, torch.randperm(H, generator=g)[: max(1, H // 100)]] *= 20.0
    xb = x.to(torch.bfloat16)
    if T > 1:
        xb[1] = 0.0                                   # zero row -> scale 0, codes 0
    if T > 2:
        xb[2, 0] = -0.0
        xb[2, 1] = -1e-30                             # underflows to a signed zero code
    if T > 3:
        xb[3] = -xb[3].abs()                          # all-negative row
    return xb


@pytest.mark.parametrize("T,H", [(1, 128), (3, 16), (17, 512), (64, 6144), (5, 16384), (300, 2048)])
def test_act_quant_bit_exact(T, H):
    xb = _acts(T, H, T * 7 + H)
    codes, scales = w4.w4a8_quant_act_fp8_per_token(xb.cuda())
    rc, rs = oracle.quant_act_fp8_per_token(f64(xb))
    assert np.array_equal(scales.cpu().numpy().astype(np.float64), rs)
    assert np.array_equal(codes.cpu().numpy(), rc)


def test_act_quant_empty():
    c, s = w4.w4a8_quant_act_fp8_per_token(torch.zeros(0, 128, dtype=torch.bfloat16, device="cuda"))
    assert c.shape == (0, 128) and s.shape == (0,)


def _logits(T, E, kind, seed):
    cfg = workloads.MoEConfig("route", T=T, H=128, I=128, E=E, k=1, seed=seed,
                              zipf_s=1.1 if "zipf" in kind else 0.0,
                              forced_empty=(E // 16 if "empty" in kind else 0))
    l = workloads.gen_logits(cfg)
    if kind == "ties":
        l = torch.round(l * 2) / 2                    # many exact ties
    return l


@pytest.mark.parametrize("T,E,k,kind", [
    (16, 8, 2, "n"), (64, 256, 8, "n"), (256, 256, 8, "zipf"), (1000, 256, 8, "empty"),
    (37, 5, 3, "n"), (5, 1, 1, "n"), (300, 1024, 32, "n"), (2048, 64, 6, "ties"),
    (257, 33, 33, "n"), (65536, 256, 8, "zipf_empty"), (1, 256, 8, "n")])
def test_route_permute_bit_exact(T, E, k, kind):
    if k > E or k > 32:
        pytest.skip("outside the supported k range")
    l = _logits(T, E, kind, T + E + k)
    r = w4.w4a8_moe_route_permute(l.cuda(), k)
    ids, wts = oracle.route_topk(l.numpy(), k)
    off, st, ro = oracle.permute_by_expert(ids, E)
    assert np.array_equal(r["topk_ids"].cpu().numpy(), ids)
    assert np.array_equal(r["expert_offsets"].cpu().numpy(), off)
    assert np.array_equal(r["sorted_token_ids"].cpu().numpy(), st)
    assert np.array_equal(r["row_of"].cpu().numpy(), ro)
    gw = r["topk_w"].cpu().numpy().astype(np.float64)
    assert np.allclose(gw, wts.astype(np.float64), rtol=1e-6, atol=1e-30)


def test_route_k_out_of_range_is_rejected():
    with pytest.raises(w4.W4A8Error, match="UNSUPPORTED_SHAPE"):
        w4.w4a8_moe_route_permute(torch.zeros(4, 8, device="cuda"), 9)


def test_route_empty_tokens():
    r = w4.w4a8_moe_route_permute(torch.zeros(0, 8, device="cuda"), 2)
    assert r["expert_offsets"].cpu().tolist() == [0] * 9
