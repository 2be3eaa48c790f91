"""Routing, permutation and the W4A8 expert layer (oracle; test
infrastructure only).

The pages fix the expert numerics (INT4 group-128 weights, FP8 per-token
activations, INT4 converted to FP8 for the tensor-core product, GLM-5.3-W4A8
model card, intro and "quantisation method") and the layer shape (256 routed
experts per layer, three projections per expert: gate, up and down, "From
755GB to 395GB" blog, "what was quantised" and "the hard part is the memory
limit").  They do not print the gating function, the activation function or
the combine.  Readings taken here:

* routing: for each token take the k largest raw logits (ties go to the lower
  expert id); the k weights are the softmax of the selected logits
  (renormalised top-k), stored as float32;
* permutation: a stable counting sort of the (token, slot) assignments by
  expert: segment e holds the tokens routed to expert e in ascending token
  order; ``row_of[t, j]`` is the segment row of assignment (t, j);
* gate/up: rows [0, I) of the [2I, H] weight are the gate projection, rows
  [I, 2I) the up projection; intermediate h = silu(gate) * up with
  silu(x) = x / (1 + exp(-x)); no clamp;
* the intermediate is requantised to FP8 per segment row with the same rule
  as the input activations (scale = float32(absmax / 448));
* down: Y = (h-scale * h-codes) @ (q2 * s2)^T;
* combine: out[t] = bf16(sum_j w[t, j] * Y[row_of[t, j]]), summed in slot
  order; no extra routed scaling factor.  With a shared expert (the FP8-block
  expert of ``shared.py``), its output is added to that sum before the bf16
  rounding.

All products and sums are float64; the only roundings are the quantisation
points of the method (bf16 scales, INT4 values, FP8 codes, float32 scales and
routing weights, the bf16 output).
"""
from __future__ import annotations

from typing import Callable, Dict, Optional, Sequence

import numpy as np

from .numerics import bf16_round, e4m3_decode, f32_round
from .quant import (dequantize_int4, pack_uint4b8, quant_act_fp8_per_token,
                    quant_act_int8_per_token, rtn_quantize_int4)
from .shared import shared_expert_forward


def route_topk(logits, k: int):
    """Top-k routing: ids int32 [T, k] (best first), weights float32 [T, k].

    Order key per token: (-logit, expert id).  Weights: softmax over the k
    selected logits, computed in float64 and rounded to float32.
    """
    l = np.asarray(logits, dtype=np.float64)
    T, E = l.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    ids_key = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((ids_key, -l), axis=-1)
    ids = order[:, :k].astype(np.int32)
    sel = np.take_along_axis(l, ids.astype(np.int64), axis=1)
    ex = np.exp(sel - sel[:, :1])
    w = f32_round(ex / ex.sum(axis=1, keepdims=True))
    return ids, w.astype(np.float32)


def permute_by_expert(ids, E: int):
    """Stable counting sort of assignments by expert.

    Returns ``expert_offsets`` int32 [E+1], ``sorted_token_ids`` int32 [T*k]
    (token of each segment row) and ``row_of`` int32 [T, k].
    """
    ids = np.asarray(ids, dtype=np.int64)
    T, k = ids.shape
    flat = ids.reshape(-1)
    counts = np.bincount(flat, minlength=E)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    order = np.argsort(flat, kind="stable")       # by expert, then by t*k + j
    sorted_tok = (order // k).astype(np.int32)
    row_of = np.empty(T * k, dtype=np.int64)
    row_of[order] = np.arange(T * k)
    return offsets.astype(np.int32), sorted_tok, row_of.reshape(T, k).astype(np.int32)


class ExpertStore:
    """The oracle's own quantised experts, built lazily from bf16 weights.

    ``get_weights(e)`` returns float64 arrays ``(w13 [2I, H], w2 [H, I])``
    holding bf16 values; ``quantize`` is ``rtn_quantize_int4`` (default) or
    ``mse_clip_quantize_int4``.  Indexing returns
    ``(w13_packed int32 [2I, H/8], s13 [2I, H/128], w2_packed int32 [H, I/8],
    s2 [H, I/128])``.
    """

    def __init__(self, E: int, get_weights: Callable[[int], tuple], quantize=None):
        self.E = E
        self._get = get_weights
        self._quantize = quantize or rtn_quantize_int4
        self._cache: Dict[int, tuple] = {}

    def __getitem__(self, e: int):
        if e not in self._cache:
            w13, w2 = self._get(e)
            q13, s13 = self._quantize(w13)
            q2, s2 = self._quantize(w2)
            self._cache[e] = (pack_uint4b8(q13), s13, pack_uint4b8(q2), s2)
        return self._cache[e]

    def __len__(self):
        return self.E


def _silu(x):
    return x / (1.0 + np.exp(-x))


def expert_forward(x_deq, expert, act_format: str = "fp8"):
    """One expert on the dequantised activation rows ``x_deq`` (float64 [n, H]):
    gate/up GEMM, SwiGLU, requantisation of h per row, down GEMM.

    ``expert`` = ``(w13_packed, s13, w2_packed, s2)``.  Returns ``(h [n, I],
    h codes [n, I], h scales [n], Y [n, H])``.
    """
    quant, decode = _act_codec(act_format)
    w13p, s13, w2p, s2 = expert
    I = w13p.shape[0] // 2
    H_ = w13p.shape[1] * 8
    G = x_deq @ dequantize_int4(w13p, s13, group=H_ // s13.shape[1]).T   # [n, 2I]
    h = _silu(G[:, :I]) * G[:, I:]
    hc, hs = quant(h)
    hd = hs[:, None] * decode(hc)
    Ye = hd @ dequantize_int4(w2p, s2, group=I // s2.shape[1]).T        # [n, H]
    return h, hc, hs, Ye


def _act_codec(act_format: str):
    if act_format == "fp8":
        return quant_act_fp8_per_token, e4m3_decode
    if act_format == "int8":
        return quant_act_int8_per_token, lambda c: np.asarray(c, dtype=np.float64)
    raise ValueError(f"unknown act_format {act_format!r}")


def moe_forward(hidden, logits, experts: Sequence, k: int,
                tokens: Optional[np.ndarray] = None, hidden_of_tokens=None,
                act_format: str = "fp8", shared=None, expert_map=None):
    """The whole layer for all tokens, or for the token subset ``tokens``.

    ``hidden``: float64 [T, H] (bf16 values); ``logits``: float32 [T, E];
    ``experts[e]`` = ``(w13_packed, s13, w2_packed, s2)``.  Routing and the
    permutation always cover all T tokens (they are cheap); the expert GEMMs
    and the combine run only for the assignments of ``tokens`` (all tokens by
    default).  ``hidden`` may be None when ``hidden_of_tokens`` (float64
    [len(tokens), H], the rows of ``tokens``) is given instead.

    ``act_format``: "fp8" (E4M3 per-token activations, the W4A8 layer) or
    "int8" (symmetric INT8 per-token activations, the per-channel variant; the
    experts' scales then have one column per row).

    ``shared``: optional FP8-block shared expert ``(w13_codes, w13_scales,
    w2_codes, w2_scales)``; its ``shared_expert_forward`` result for the rows
    of ``tokens`` is returned under ``shared`` and its ``y`` is added to the
    routed sum before the bf16 rounding.

    ``expert_map``: optional ``f(tasks, act_format) -> results`` that evaluates
    ``expert_forward`` for each ``(e, x_deq rows)`` task in order (e.g. in
    worker processes); by default each task runs here on ``experts[e]``.

    Returns a dict with ``topk_ids``, ``topk_w``, ``expert_offsets``,
    ``sorted_token_ids``, ``row_of``, ``act_codes`` / ``act_scales`` (rows of
    ``tokens``), ``inter_h`` / ``inter_codes`` / ``inter_scales`` / ``y_rows``
    (keyed by segment row, for the rows computed), ``out`` float64
    [len(tokens), H] bf16 values and ``tokens``.
    """
    T, E = logits.shape
    if hidden_of_tokens is None:
        hidden = np.asarray(hidden, dtype=np.float64)

    ids, w = route_topk(logits, k)
    offsets, sorted_tok, row_of = permute_by_expert(ids, E)
    tokens = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    pos = {int(t): i for i, t in enumerate(tokens)}
    x_rows = hidden[tokens] if hidden_of_tokens is None else np.asarray(hidden_of_tokens,
                                                                         dtype=np.float64)
    H = x_rows.shape[1]

    quant, decode = _act_codec(act_format)
    codes, a_scale = quant(x_rows)
    x_deq = a_scale[:, None] * decode(codes)               # exact: 24-bit x <= 8-bit significands

    need_rows = np.sort(row_of[tokens].reshape(-1))
    Y: Dict[int, np.ndarray] = {}
    inter_h: Dict[int, np.ndarray] = {}
    inter_codes: Dict[int, np.ndarray] = {}
    inter_scales: Dict[int, float] = {}
    tasks = []
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        rows = need_rows[(need_rows >= lo) & (need_rows < hi)]
        if rows.size:
            tasks.append((e, rows, x_deq[[pos[int(sorted_tok[r])] for r in rows]]))
    if expert_map is None:
        results = [expert_forward(X, experts[e], act_format) for e, _, X in tasks]
    else:
        results = expert_map([(e, X) for e, _, X in tasks], act_format)
    for (e, rows, _), (h, hc, hs, Ye) in zip(tasks, results):
        for i, r in enumerate(rows):
            Y[int(r)] = Ye[i]
            inter_h[int(r)] = h[i]
            inter_codes[int(r)] = hc[i]
            inter_scales[int(r)] = float(hs[i])

    sh = shared_expert_forward(x_rows, *shared) if shared is not None else None
    out = np.zeros((len(tokens), H), dtype=np.float64)
    for i, t in enumerate(tokens):
        acc = np.zeros(H, dtype=np.float64)
        for j in range(k):
            acc = acc + float(w[t, j]) * Y[int(row_of[t, j])]
        if sh is not None:
            acc = acc + sh["y"][i]
        out[i] = bf16_round(acc)

    return dict(topk_ids=ids, topk_w=w, expert_offsets=offsets, sorted_token_ids=sorted_tok,
                row_of=row_of, act_codes=codes, act_scales=a_scale, inter_h=inter_h,
                inter_codes=inter_codes, inter_scales=inter_scales, y_rows=Y, out=out,
                tokens=tokens, shared=sh)
