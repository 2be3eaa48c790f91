"""Helpers shared by the GPU parity tests (not a test module)."""
import numpy as np
import torch

import oracle
import workloads


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


def repack_b200(packed: np.ndarray) -> np.ndarray:
    """Expected word layout of w4a8_prepare_experts_b200, from the header's definition:
    nibble j of each word moves to nibble 2j (j < 4) or 2(j - 4) + 1 (j >= 4)."""
    w = np.asarray(packed).view(np.uint32).astype(np.uint64)
    r = np.zeros_like(w)
    for j in range(8):
        dst = 2 * j if j < 4 else 2 * (j - 4) + 1
        r |= ((w >> np.uint64(4 * j)) & np.uint64(0xF)) << np.uint64(4 * dst)
    return r.astype(np.uint32).view(np.int32).reshape(np.shape(packed))


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
