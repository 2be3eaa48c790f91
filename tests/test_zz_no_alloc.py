"""w4a8_moe_route_permute_noalloc, the routing entry point for callers that
cannot allocate device memory when they route (plugin interfaces that pass
only planned buffers, fixed device memory budgets).  It keeps
its scratch in a static device array instead of a caller workspace; its
outputs must equal those of w4a8_moe_route_permute, on consecutive calls that
reuse the same scratch.

This file is collected last on purpose, so that a run stopping at the first
failure has run every other test first; it also passes on its own in a fresh
process.
"""
import ctypes

import pytest
import torch

import workloads
import w4a8_quantized_moe_b200 as w4

pytestmark = pytest.mark.gpu

FIELDS = ["topk_ids", "topk_w", "expert_offsets", "sorted_token_ids", "row_of"]


def _logits(T, E, seed, zipf=0.0):
    cfg = workloads.MoEConfig("noalloc", T=T, H=128, I=128, E=E, k=1, seed=seed, zipf_s=zipf)
    return workloads.gen_logits(cfg).cuda()


def _noalloc_through_c_abi(logits, k):
    """Call the C entry point directly with caller-allocated outputs."""
    T, E = logits.shape
    dev = logits.device
    out = dict(topk_ids=torch.full((T, k), -1, dtype=torch.int32, device=dev),
               topk_w=torch.full((T, k), -1.0, dtype=torch.float32, device=dev),
               expert_offsets=torch.full((E + 1,), -1, dtype=torch.int32, device=dev),
               sorted_token_ids=torch.full((T * k,), -1, dtype=torch.int32, device=dev),
               row_of=torch.full((T, k), -1, dtype=torch.int32, device=dev))
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    L = w4.lib()
    st = L.w4a8_moe_route_permute_noalloc(
        p(logits), T, E, k, p(out["topk_ids"]), p(out["topk_w"]), p(out["expert_offsets"]),
        p(out["sorted_token_ids"]), p(out["row_of"]),
        ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
    assert st == 0, L.w4a8_last_error().decode()
    return out


def _assert_same(got, ref):
    torch.cuda.synchronize()
    for name in ["topk_ids", "expert_offsets", "sorted_token_ids", "row_of"]:
        assert torch.equal(got[name], ref[name]), name
    # same kernels, same arithmetic: the weights agree far inside the 1e-6 tolerance
    assert torch.allclose(got["topk_w"], ref["topk_w"], rtol=1e-6, atol=0.0)


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    cases = [(300, 256, 8, 1, 0.0), (1000, 64, 6, 2, 1.1), (300, 256, 8, 1, 0.0), (37, 5, 3, 4, 0.0)]
    for T, E, k, seed, zipf in cases:       # back to back: the static scratch is reused
        logits = _logits(T, E, seed, zipf)
        got = _noalloc_through_c_abi(logits, k)
        ref = w4.w4a8_moe_route_permute(logits, k)
        _assert_same(got, ref)


def test_noalloc_rejects_sizes_beyond_the_static_scratch():
    T, E, k = 256 * 65, 1024, 8          # ceil(T / 256) * E = 66560 > 65536
    logits = torch.zeros(T, E, device="cuda")
    with pytest.raises(w4.W4A8Error, match="static scratch"):
        w4.w4a8_moe_route_permute_noalloc(logits, k)
    # the largest accepted size at E = 256 still works and matches
    logits = _logits(65536, 256, 9, 1.1)
    _assert_same(_noalloc_through_c_abi(logits, 8), w4.w4a8_moe_route_permute(logits, 8))
