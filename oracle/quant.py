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

from fractions import Fraction

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

# Relative bound on |e_float - e_exact| for one candidate's squared error over a
# group of 128, e_float computed below in float64 in any summation order.  Each
# term fl(fl(w - q s)^2) is within (1 + u)^3 - 1 < 3.0001 u of the exact square
# (q s is exact: a 4-bit integer times a bf16 scale; one rounding for the
# difference, one for the square; u = 2^-53); summing 128 nonnegative terms in
# any order adds at most (1 + u)^127 - 1 < 127.001 u.  2^-45 = 256 u covers both.
MSE_ERR_REL_BOUND = 2.0 ** -45


def _exact_group_error(wrow, qrow, s) -> Fraction:
    """Sum over the group of (w - q s)^2 in exact rational arithmetic."""
    sf = Fraction(float(s))
    return sum(((Fraction(float(w)) - int(q) * sf) ** 2 for w, q in zip(wrow, qrow)),
               Fraction(0))


def mse_clip_candidates(w, group: int = GROUP):
    """The 11 candidates of the per-group MSE clip search and their errors.

    For each ratio r_i (float32 ``CLIP_RATIOS``, i = 0 .. 10):
      s_i = bf16(float32(float32(absmax * r_i) / 7));
      q_i = clamp(round_half_even(float32(w / s_i)), -8, 7), 0 where s_i = 0;
      e_i = sum over the group of (w - q_i * s_i)^2, computed in float64; it is
            within ``MSE_ERR_REL_BOUND * e_i`` of the exact value.
    Returns ``(q [11, R, K] int8, s [11, R, K // group] float64 holding bf16
    values, e [11, R, K // group] float64)``.
    """
    w = np.asarray(w, dtype=np.float64)
    R, K = w.shape
    if K % group or group != 128:
        raise ValueError("group must be 128 and divide K")
    wg = w.reshape(R, K // group, group)
    amax = np.abs(wg).max(axis=2)
    qs, ss, es = [], [], []
    for r in CLIP_RATIOS:
        s = bf16_round(f32_round(f32_round(amax * np.float64(r)) / 7.0))
        with np.errstate(divide="ignore", invalid="ignore"):
            q = np.clip(np.rint(f32_round(wg / s[..., None])), -8, 7)
        q = np.where(s[..., None] == 0.0, 0.0, q)
        d = wg - q * s[..., None]
        es.append(np.sum(d * d, axis=2))
        qs.append(q.astype(np.int8).reshape(R, K))
        ss.append(s)
    return np.stack(qs), np.stack(ss), np.stack(es)


def mse_clip_quantize_int4(w, group: int = GROUP):
    """Symmetric INT4 with the per-group MSE clip search (model card,
    "quantisation method": for each group of 128, 11 shrink ratios of the
    scale from 1.00 to 0.70 are tried and the MSE-optimal scale is kept).

    The candidates are those of ``mse_clip_candidates``.  The kept candidate
    is the one with the least EXACT squared error; among exact ties the first
    (largest) ratio.  The float64 errors decide wherever they are further
    apart than their error bound; candidates that stay within the bound of the
    least error are compared in rational arithmetic.  r = 1.00 is exactly
    ``rtn_quantize_int4``; with r < 1 the code -8 becomes reachable.  Returns
    ``(q, s)`` as ``rtn_quantize_int4`` does.
    """
    w = np.asarray(w, dtype=np.float64)
    R, K = w.shape
    q_all, s_all, e_all = mse_clip_candidates(w, group)
    G = K // group
    B = MSE_ERR_REL_BOUND
    # a candidate whose scale equals an earlier candidate's is the same candidate
    dup = np.zeros(e_all.shape, dtype=bool)
    for i in range(1, 11):
        dup[i] = np.any(s_all[:i] == s_all[i][None], axis=0)
    e_cmp = np.where(dup, np.inf, e_all)
    lo = e_cmp * (1.0 - B)                       # exact error is within [lo, hi]
    hi = e_cmp * (1.0 + B)
    best_hi = hi.min(axis=0)
    contenders = lo <= best_hi[None]             # [11, R, G]: could be the minimum
    choice = np.argmin(e_cmp, axis=0)            # decided where one contender remains
    wg = w.reshape(R, G, group)
    qg = q_all.reshape(11, R, G, group)
    for r, g in zip(*np.nonzero(contenders.sum(axis=0) > 1)):
        cands = np.nonzero(contenders[:, r, g])[0]
        exact = [_exact_group_error(wg[r, g], qg[i, r, g], s_all[i, r, g]) for i in cands]
        first_min = min(range(len(cands)), key=lambda j: exact[j])   # first of the exact minima
        choice[r, g] = cands[first_min]
    q = np.take_along_axis(qg, choice[None, ..., None], axis=0)[0].reshape(R, K)
    s = np.take_along_axis(s_all, choice[None], axis=0)[0]
    return q.astype(np.int8), s


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
