"""The FP8 128 x 128-block shared expert (oracle; test infrastructure only).

GLM-5.3-W4A8 model card, intro and "quantisation method" (item on the
non-expert layers): only the routed experts are INT4; attention, the shared
expert and the dense MLP keep the official FP8 block format unchanged, E4M3
weights with one float32 scale per 128 x 128 block of the weight matrix
(stored as ``weight_scale``).  The model card's storage-format paragraph calls
these layers compressed-tensors ``float-quantized`` FP8 128 x 128 block.

Readings taken where the pages are silent:
* block scale: s = float32(absmax of the block / 448) and
  code = E4M3(float32(w / s)); a block whose absmax is 0 has s = 0 and
  all-zero codes (the official checkpoint ships these scales; synthetic
  weights are quantised with this rule);
* activations of an FP8-block layer: dynamic, one float32 scale per token and
  per 128-wide group of channels, s = float32(absmax / 448), code =
  E4M3(float32(x / s)) (the group-wise form of the routed path's per-token
  rule; the pages name no other granularity for these layers);
* the shared expert has the routed experts' shape: one SwiGLU FFN with gate
  rows [0, I) and up rows [I, 2I) of a [2I, H] weight and a [H, I] down
  weight; h = silu(gate) * up is requantised per token and 128-group with the
  activation rule;
* the layer output adds the shared expert to the routed combine before the
  single bf16 rounding: out[t] = bf16(sum_j w[t, j] Y[row_of[t, j]] + Y_s[t]).

All products and sums are float64.
"""
from __future__ import annotations

import numpy as np

from .numerics import e4m3_decode, e4m3_encode, f32_round, E4M3_MAX

BLOCK = 128


def quant_fp8_block(w, block: int = BLOCK):
    """E4M3 codes with one float32 scale per ``block`` x ``block`` tile.

    ``w``: float64 [R, K] (bf16 values), R and K multiples of ``block``.
    Returns ``(codes uint8 [R, K], scales float64 [R / block, K / block]
    holding float32 values)``.
    """
    w = np.asarray(w, dtype=np.float64)
    R, K = w.shape
    if R % block or K % block:
        raise ValueError("both dimensions must be multiples of the block size")
    tiles = w.reshape(R // block, block, K // block, block)
    amax = np.abs(tiles).max(axis=(1, 3))                          # [R/b, K/b]
    s = f32_round(amax / E4M3_MAX)
    safe = np.where(s > 0, s, 1.0)
    ratio = f32_round(tiles / safe[:, None, :, None])
    codes = e4m3_encode(ratio)
    codes[np.broadcast_to((s == 0)[:, None, :, None], codes.shape)] = 0
    return codes.reshape(R, K), s


def dequant_fp8_block(codes, scales, block: int = BLOCK):
    """float64 [R, K] weights decoded from block codes and scales."""
    c = e4m3_decode(codes)
    R, K = c.shape
    s = np.repeat(np.repeat(np.asarray(scales, dtype=np.float64), block, axis=0), block, axis=1)
    return c * s[:R, :K]


def quant_act_fp8_group(x, group: int = BLOCK):
    """Dynamic E4M3 quantisation per row and ``group``-wide channel group.

    ``x``: float64 [T, H], H a multiple of ``group``.  Returns ``(codes uint8
    [T, H], scales float64 [T, H / group] holding float32 values)``.
    """
    x = np.asarray(x, dtype=np.float64)
    T, H = x.shape
    if H % group:
        raise ValueError("H must be a multiple of the group size")
    g = x.reshape(T, H // group, group)
    amax = np.abs(g).max(axis=2) if T else np.zeros((0, H // group))
    s = f32_round(amax / E4M3_MAX)
    safe = np.where(s > 0, s, 1.0)
    codes = e4m3_encode(f32_round(g / safe[..., None]))
    codes[np.broadcast_to((s == 0)[..., None], codes.shape)] = 0
    return codes.reshape(T, H), s


def dequant_act_fp8_group(codes, scales, group: int = BLOCK):
    """float64 [T, H] activations decoded from group codes and scales."""
    c = e4m3_decode(codes)
    return c * np.repeat(np.asarray(scales, dtype=np.float64), group, axis=1)


def shared_expert_forward(x, w13_codes, w13_scales, w2_codes, w2_scales):
    """The FP8-block SwiGLU expert for the rows of ``x`` (float64 [T, H]).

    Returns a dict: ``act_codes`` / ``act_scales`` (the quantised input),
    ``h`` (float64 [T, I]), ``h_codes`` / ``h_scales`` and ``y`` (float64
    [T, H]).
    """
    ac, asc = quant_act_fp8_group(x)
    xd = dequant_act_fp8_group(ac, asc)
    I = w13_codes.shape[0] // 2
    G = xd @ dequant_fp8_block(w13_codes, w13_scales).T            # [T, 2I]
    h = G[:, :I] / (1.0 + np.exp(-G[:, :I])) * G[:, I:]
    hc, hs = quant_act_fp8_group(h)
    y = dequant_act_fp8_group(hc, hs) @ dequant_fp8_block(w2_codes, w2_scales).T
    return dict(act_codes=ac, act_scales=asc, h=h, h_codes=hc, h_scales=hs, y=y)
