"""Helpers shared by the GPU parity tests (not a test module)."""
import numpy as np
import torch

import oracle
import workloads
from oracle_pool import repack_b200, unrepack_b200  # noqa: F401 (re-exported)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f64(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> float64 numpy values."""
    return oracle.bf16_bits_to_f64(bf16_bits(t))


def rel_fro(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def e4m3_ordinal(codes: np.ndarray) -> np.ndarray:
    """Position of each E4M3 code on the number line (+0 and -0 both 0)."""
    c = codes.astype(np.int64)
    mag = c & 0x7F
    return np.where(c & 0x80, -mag, mag)


def codes_agree(gpu: np.ndarray, ref: np.ndarray):
    """(fraction exactly equal, max ordinal distance) of two E4M3 code arrays."""
    eq = (gpu == ref) | ((gpu & 0x7F) == 0) & ((ref & 0x7F) == 0)
    dist = np.abs(e4m3_ordinal(gpu) - e4m3_ordinal(ref))
    return float(np.mean(eq)), int(dist.max(initial=0))


def small_case(cfg: workloads.MoEConfig):
    """CPU-generated inputs of a small workload: hidden, logits, w13 [E,2I,H], w2 [E,H,I]."""
    hidden = workloads.gen_hidden(cfg)
    logits = workloads.gen_logits(cfg)
    ws = [workloads.gen_expert_weights(cfg, e) for e in range(cfg.E)]
    w13 = torch.stack([a for a, _ in ws])
    w2 = torch.stack([b for _, b in ws])
    return hidden, logits, w13, w2


def aux_buffers(T, H, I, E, k, device="cuda"):
    A = T * k
    return dict(
        topk_ids=torch.empty(T, k, dtype=torch.int32, device=device),
        topk_w=torch.empty(T, k, dtype=torch.float32, device=device),
        expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=device),
        sorted_token_ids=torch.empty(A, dtype=torch.int32, device=device),
        row_of=torch.empty(T, k, dtype=torch.int32, device=device),
        act_codes=torch.empty(T, H, dtype=torch.uint8, device=device),
        act_scales=torch.empty(T, dtype=torch.float32, device=device),
        inter_h=torch.empty(A, I, dtype=torch.float32, device=device),
        inter_codes=torch.empty(A, I, dtype=torch.uint8, device=device),
        inter_scales=torch.empty(A, dtype=torch.float32, device=device),
        y_rows=torch.empty(A, H, dtype=torch.float32, device=device),
    )


def assert_mse_clip_choice(packed: np.ndarray, scale_bits: np.ndarray, w: np.ndarray) -> int:
    """Check a clip-search quantisation (the pages' word layout [R, K/8] and bf16
    scale bits [R, K/128]) against the oracle's candidates for the float64
    weights ``w`` [R, K].  Every group must hold one of its 11 candidates (codes
    and scale); where that candidate is not the oracle's exact choice it must
    be within the float64 summation bound of the least error (a near tie that
    a different, equally valid, summation order may resolve the other way).
    Returns the number of such groups."""
    B = oracle.MSE_ERR_REL_BOUND
    R, K = w.shape
    G = K // 128
    q_all, s_all, e_all = oracle.mse_clip_candidates(w)
    q_o, s_o = oracle.mse_clip_quantize_int4(w)
    q_g = oracle.unpack_uint4b8(packed).reshape(R, G, 128)
    s_g = oracle.bf16_bits_to_f64(scale_bits).reshape(R, G)
    same = (s_g == s_o) & np.all(q_g == q_o.reshape(R, G, 128), axis=2)
    e_best = np.take_along_axis(e_all, np.argmin(e_all, axis=0)[None], axis=0)[0]
    n_ties = 0
    for r, g in zip(*np.nonzero(~same)):
        match = [i for i in range(11) if s_all[i, r, g] == s_g[r, g]
                 and np.array_equal(q_all[i, r].reshape(G, 128)[g], q_g[r, g])]
        assert match, f"group ({r}, {g}) holds none of the 11 candidates"
        i = match[0]
        assert e_all[i, r, g] * (1 - B) <= e_best[r, g] * (1 + B), \
            f"group ({r}, {g}): candidate {i} is not within the error bound of the minimum"
        n_ties += 1
    return n_ties



TILE_WIDTHS = (32, 128)     # token rows per grouped-GEMM tile: decode and prefill shapes


def boundary_rows(offsets: np.ndarray, n_segments: int = 3) -> np.ndarray:
    """Segment rows on tile boundaries of the largest segments (the first and last row of
    the first tile, a middle tile, the last full tile and the partial last tile,
    for each tile width)."""
    counts = np.diff(offsets.astype(np.int64))
    rows = set()
    for e in np.argsort(-counts, kind="stable")[:n_segments]:
        lo, n = int(offsets[e]), int(counts[e])
        if n == 0:
            continue
        for width in TILE_WIDTHS:
            tiles = -(-n // width)
            full = n // width
            for t in {0, tiles // 2, max(full - 1, 0), tiles - 1}:
                first = lo + t * width
                last = min(lo + (t + 1) * width, lo + n) - 1
                rows.update((first, last))
    return np.array(sorted(rows), dtype=np.int64)
