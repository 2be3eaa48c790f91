"""Weight and activation quantisation of the W4A8 layer (oracle; test
infrastructure only).

Weights (GLM-5.3-W4A8 model card, section "quantisation method"; intro and
table "differences from the other 4-bit releases"): symmetric INT4, one scale
per group of 128 consecutive weights along K, stored in compressed-tensors
``pack-quantized`` form: each 4-bit value q in [-8, 7] is stored as the
unsigned nibble q + 8 ("uint4b8"), 8 nibbles per int32 word ("8 four-bit
weights per int32 slot", the note on the ~370B parameter display).  The pages
describe round-to-nearest with a per-group MSE search over 11 shrink ratios of
the scale (model card, "quantisation method": ratios 1.00 down to 0.70, the
MSE-optimal scale kept).  ``rtn_quantize_int4`` is the plain round-to-nearest
step with scale = absmax / 7 (the ratio-1.00 member of that search);
``mse_clip_quantize_int4`` is the search.

Readings taken where the pages are silent:
* scale: s = bf16(absmax / 7), rounded to bf16 (the stored scale dtype) before
  it is used, so the quantiser divides by exactly the scale the GEMM
  multiplies by;
* q = clamp(round_half_even(float32(w / s)), -8, 7); a group whose absmax is 0
  has s = 0 and q = 0;
* nibble order: element kappa of a row goes to word kappa // 8, bits
  4*(kappa % 8) .. 4*(kappa % 8) + 3 (little-endian nibbles along K); the
  packed tensor is row-major [rows, K / 8].

Activations (model card, "quantisation method" last item and the table above:
FP8 per-token dynamic activations): one float32 scale per token,
scale = float32(absmax / 448) (448 = largest finite E4M3 value), and
code = E4M3(float32(x / scale)); a token whose absmax is 0 gets scale 0 and
all-zero codes.
"""
from __future__ import annotations

import numpy as np

from .numerics import bf16_round, f32_round, e4m3_encode, E4M3_MAX

GROUP = 128


def rtn_quantize_int4(w, group: int = GROUP):
    """Symmetric INT4 RTN per group of ``group`` along the last axis.

    ``w``: float64 [R, K] holding bf16 values.  Returns ``(q, s)`` with q int8
    [R, K] in [-8, 7] and s float64 [R, K // group] holding bf16 values.
    """
    w = np.asarray(w, dtype=np.float64)
    R, K = w.shape
    if K % group:
        raise ValueError("K must be a multiple of the group size")
    wg = w.reshape(R, K // group, group)
    amax = np.abs(wg).max(axis=2)
    # float decides the stored scale: take it in float32 division, then bf16
    s = bf16_round(f32_round(amax / 7.0))
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = f32_round(wg / s[..., None])
    q = np.clip(np.rint(ratio), -8, 7)
    q = np.where(s[..., None] == 0.0, 0.0, q)
    return q.astype(np.int8).reshape(R, K), s


# The 11 shrink ratios 1.00, 0.97, ..., 0.70 (evenly spaced; the plainest reading
# of "11 ratios from 1.00 to 0.70"), as float32 values (100 - 3 i) / 100.
CLIP_RATIOS = np.array([np.float32((100.0 - 3.0 * i) / 100.0) for i in range(11)],
                       dtype=np.float32)


def _squared_error_fixed_order(d):
    """Sum of d**2 over the last axis (128 = 32 x 4) in float64, in one fixed
    order: each run of 4 consecutive values summed in sequence, then the 32
    partial sums combined by five pairwise (xor 16, 8, 4, 2, 1) exchanges.
    The pages do not say how the MSE is accumulated; fixing the order makes the
    arg-min below a deterministic function of the inputs, which the kernel
    reproduces operation for operation."""
    sq = d * d
    p = sq[..., 0::4] + sq[..., 1::4]
    p = p + sq[..., 2::4]
    p = p + sq[..., 3::4]
    lanes = np.arange(32)
    for off in (16, 8, 4, 2, 1):
        p = p + p[..., lanes ^ off]
    return p[..., 0]


def mse_clip_quantize_int4(w, group: int = GROUP):
    """Symmetric INT4 with the per-group MSE clip search (model card,
    "quantisation method": for each group of 128, 11 shrink ratios of the
    scale from 1.00 to 0.70 are tried and the MSE-optimal scale is kept).

    For each ratio r (float32 ``CLIP_RATIOS``, tried from 1.00 down):
      s_r = bf16(float32(float32(absmax * r) / 7));
      q_r = clamp(round_half_even(float32(w / s_r)), -8, 7), 0 where s_r = 0;
      e_r = sum over the group of (w - q_r * s_r)**2 in float64 (fixed order,
            ``_squared_error_fixed_order``).
    The first ratio with the smallest e_r is kept (ties keep the larger
    scale).  r = 1.00 is exactly ``rtn_quantize_int4``.  With r < 1 the code
    -8 becomes reachable.  Returns ``(q, s)`` as ``rtn_quantize_int4`` does.
    """
    w = np.asarray(w, dtype=np.float64)
    R, K = w.shape
    if K % group or group != 128:
        raise ValueError("group must be 128 and divide K")
    wg = w.reshape(R, K // group, group)
    amax = np.abs(wg).max(axis=2)
    best_e = np.full(amax.shape, np.inf)
    best_q = np.zeros(wg.shape)
    best_s = np.zeros(amax.shape)
    for r in CLIP_RATIOS:
        s = bf16_round(f32_round(f32_round(amax * np.float64(r)) / 7.0))
        with np.errstate(divide="ignore", invalid="ignore"):
            q = np.clip(np.rint(f32_round(wg / s[..., None])), -8, 7)
        q = np.where(s[..., None] == 0.0, 0.0, q)
        e = _squared_error_fixed_order(wg - q * s[..., None])
        take = e < best_e
        best_e = np.where(take, e, best_e)
        best_s = np.where(take, s, best_s)
        best_q = np.where(take[..., None], q, best_q)
    return best_q.astype(np.int8).reshape(R, K), best_s


def rtn_quantize_int4_channel(w):
    """Per-channel symmetric INT4 RTN ("GLM-5.3-Channel-INT4-w4a8" model card,
    quantisation table: RTN, static, per-channel INT4 routed experts): one bf16
    scale per output row, i.e. the group rule with the group spanning all of
    K.  Returns ``(q int8 [R, K], s float64 [R, 1])``."""
    w = np.asarray(w, dtype=np.float64)
    return rtn_quantize_int4(w, group=w.shape[1])


def pack_uint4b8(q):
    """Pack int [R, K] values in [-8, 7] into int32 [R, K // 8] uint4b8 words."""
    q = np.asarray(q).astype(np.int64)
    R, K = q.shape
    if K % 8:
        raise ValueError("K must be a multiple of 8")
    if q.min(initial=0) < -8 or q.max(initial=0) > 7:
        raise ValueError("values out of INT4 range")
    u = (q + 8).reshape(R, K // 8, 8).astype(np.uint64)
    word = np.zeros((R, K // 8), dtype=np.uint64)
    for i in range(8):
        word |= u[..., i] << np.uint64(4 * i)
    return word.astype(np.uint32).view(np.int32)


def unpack_uint4b8(packed):
    """Inverse of ``pack_uint4b8``: int32 [R, K/8] -> int8 [R, K]."""
    p = np.asarray(packed).view(np.uint32).astype(np.uint64)
    R, W = p.shape
    out = np.empty((R, W, 8), dtype=np.int8)
    for i in range(8):
        out[..., i] = ((p >> np.uint64(4 * i)) & np.uint64(0xF)).astype(np.int8) - 8
    return out.reshape(R, W * 8)


def dequantize_int4(packed, scales, group: int = GROUP):
    """float64 [R, K] = q * s with the group scale broadcast along K (exact)."""
    q = unpack_uint4b8(packed).astype(np.float64)
    R, K = q.shape
    s = np.asarray(scales, dtype=np.float64)
    return (q.reshape(R, K // group, group) * s[..., None]).reshape(R, K)


def quant_act_int8_per_token(x):
    """Per-row dynamic symmetric INT8 quantisation ("GLM-5.3-Channel-INT4-w4a8"
    model card, quantisation table: activations dynamic, per-token INT8).

    ``x``: float64 [T, H].  scale = float32(absmax / 127);
    code = clamp(round_half_even(float32(x / scale)), -127, 127); a row whose
    absmax is 0 gets scale 0 and codes 0.  Returns ``(codes int8 [T, H],
    scale float64 [T] holding float32 values)``.
    """
    x = np.asarray(x, dtype=np.float64)
    amax = np.abs(x).max(axis=1) if x.shape[1] else np.zeros(x.shape[0])
    scale = f32_round(amax / 127.0)
    safe = np.where(scale > 0, scale, 1.0)
    codes = np.clip(np.rint(f32_round(x / safe[:, None])), -127, 127)
    codes[scale == 0] = 0
    return codes.astype(np.int8), scale


def quant_act_fp8_per_token(x):
    """Per-row dynamic FP8 quantisation.

    ``x``: float64 [T, H].  Returns ``(codes uint8 [T, H], scale float64 [T]
    holding float32 values)``.
    """
    x = np.asarray(x, dtype=np.float64)
    amax = np.abs(x).max(axis=1) if x.shape[1] else np.zeros(x.shape[0])
    scale = f32_round(amax / E4M3_MAX)
    safe = np.where(scale > 0, scale, 1.0)
    ratio = f32_round(x / safe[:, None])
    codes = e4m3_encode(ratio)
    codes[scale == 0] = 0
    return codes, scale
