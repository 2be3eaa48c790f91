"""Expert parallelism for the W4A8 MoE layer: one process per GPU, each
holding a contiguous range of the experts.

The pages deploy the W4A8 checkpoint only with expert parallelism
(GLM-5.3-W4A8 model card, "deployment": the W4A8 build must enable expert
parallelism; "performance" table: TP8+EP and 2 x (TP4+EP) on 8 GPUs).  Here
rank g of G owns the experts ``expert_partition(E, G)[g]``.  One step, for
each rank's own batch of tokens:

1. quantise the rank's tokens to E4M3 with per-token scales and route them
   (top-k ids and weights) -- the routing is computed where the tokens live;
2. dispatch: all-gather the codes, scales, ids and weights of every rank's
   tokens (padded to the largest batch; a padding token has ids -1);
3. each rank runs its own experts on all gathered tokens
   (``w4a8_moe_forward_experts``), giving float32 partial sums per token;
4. combine: reduce-scatter (sum) of the partial sums, so each rank receives
   the complete sums of its own tokens, which it rounds once to bf16.

With ``dispatch="all_to_all"`` (large batches) steps 2-4 send each token
only to the ranks that own one of its k experts: a dispatch plan (counts per
rank, the rank-major token list), an all-to-all of the counts, all-to-all(v)
of the token rows, the experts on the rows received, all-to-all(v) of the
partial sums back, and a combine that sums each token's returned rows in
rank order and rounds once to bf16.  The counts cross to the host once per
step (the all-to-all(v) split sizes).

Every compute step is a call into ``libw4a8.so``; the collectives are
``torch.distributed`` (NCCL between GPUs).  The compute steps are behind a
small interface (``ops``) so that the bookkeeping and the collectives can be
checked on CPU ranks (gloo) against the oracle by the tests.
"""
from __future__ import annotations

import datetime
from dataclasses import dataclass
from typing import Callable, List, Optional, Tuple

import torch

__all__ = ["expert_partition", "ExpertParallelMoE", "LibraryOps", "PaddedBatch"]


def expert_partition(E: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous expert ranges ``(begin, count)`` of ``world`` ranks: counts
    differ by at most one, the first ``E % world`` ranks hold one more.  A rank
    may hold none when ``world > E`` (count 0)."""
    if E < 1 or world < 1:
        raise ValueError("need E >= 1 and world >= 1")
    base, extra = divmod(E, world)
    out, b = [], 0
    for g in range(world):
        n = base + (1 if g < extra else 0)
        out.append((b, n))
        b += n
    return out


@dataclass
class PaddedBatch:
    """One rank's routed batch padded to the step's largest batch."""
    codes: torch.Tensor    # [T_max, H] uint8
    scales: torch.Tensor   # [T_max] float32
    ids: torch.Tensor      # [T_max, k] int32 (-1 in padding rows)
    weights: torch.Tensor  # [T_max, k] float32 (0 in padding rows)


class LibraryOps:
    """The compute steps of one expert-parallel step, on the CUDA library."""

    def __init__(self):
        from . import (w4a8_cast_f32_bf16, w4a8_moe_forward_experts, w4a8_moe_route_topk,
                       w4a8_quant_act_fp8_per_token)
        self._quant = w4a8_quant_act_fp8_per_token
        self._route = w4a8_moe_route_topk
        self._experts = w4a8_moe_forward_experts
        self._cast = w4a8_cast_f32_bf16
        self._ws = None

    def quant_route(self, hidden, logits, k, batch: PaddedBatch):
        T = hidden.shape[0]
        if T:
            self._quant(hidden, codes=batch.codes[:T], scales=batch.scales[:T])
            self._route(logits, k, topk_ids=batch.ids[:T], topk_w=batch.weights[:T])

    def experts(self, codes, scales, ids, weights, E, e_begin, weights_local, out):
        from . import w4a8_moe_experts_workspace_size
        T, H = codes.shape
        e_count, I = weights_local[0].shape[0], weights_local[2].shape[2] * 8
        need = max(w4a8_moe_experts_workspace_size(T, H, I, e_count, ids.shape[1]), 1)
        if self._ws is None or self._ws.numel() < need or self._ws.device != codes.device:
            self._ws = torch.empty(need, dtype=torch.uint8, device=codes.device)
        return self._experts(codes, scales, ids, weights, E, e_begin, *weights_local, out=out,
                             workspace=self._ws)

    def cast(self, x, out):
        return self._cast(x, out=out)

    def plan(self, ids, E, n_ranks):
        from . import w4a8_ep_dispatch_plan
        return w4a8_ep_dispatch_plan(ids, E, n_ranks)

    def gather(self, batch: PaddedBatch, T, rows, n_rows) -> PaddedBatch:
        from . import w4a8_ep_gather_rows
        c, s, i, w = w4a8_ep_gather_rows(batch.codes[:T], batch.scales[:T], batch.ids[:T],
                                         batch.weights[:T], rows, n_rows)
        return PaddedBatch(codes=c, scales=s, ids=i, weights=w)

    def combine(self, back, pos, out):
        from . import w4a8_ep_combine_rows
        return w4a8_ep_combine_rows(back, pos, out=out)


class ExpertParallelMoE:
    """This rank's share of an expert-parallel W4A8 layer.

    ``weights_local`` = ``(w13_packed, w13_scales, w2_packed, w2_scales)`` of
    the experts ``e_begin .. e_begin + e_count - 1`` only, in the layout of
    ``w4a8_prepare_experts_b200`` (whatever ``ops.experts`` takes); ``e_count``
    may be 0 (a rank with no experts; ``weights_local`` is then unused).
    ``group`` is the process group (default: the world).
    ``tokens_per_rank``: if every rank always calls with this many tokens,
    the step skips the collective that agrees on the padded batch size.
    ``dispatch``: ``"all_gather"`` (every token to every rank; decode) or
    ``"all_to_all"`` (each token to the ranks of its experts; prefill).  Every
    rank of the group must use the same.
    """

    def __init__(self, weights_local, E: int, k: int, e_begin: int, e_count: int, H: int,
                 I: int, group=None, ops=None, tokens_per_rank: Optional[int] = None,
                 dispatch: str = "all_gather"):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.E, self.k, self.H, self.I = E, k, H, I
        if e_begin < 0 or e_count < 0 or e_begin + e_count > E:
            raise ValueError(f"expert range [{e_begin}, {e_begin + e_count}) not inside [0, {E})")
        self.e_begin, self.e_count = e_begin, e_count
        self.weights_local = weights_local
        self.ops = ops if ops is not None else LibraryOps()
        self.tokens_per_rank = tokens_per_rank
        if dispatch not in ("all_gather", "all_to_all"):
            raise ValueError(f"dispatch must be 'all_gather' or 'all_to_all', not {dispatch!r}")
        self.dispatch = dispatch
        if dispatch == "all_to_all" and e_count:
            # the rank's range must be the one the dispatch plan assigns it
            if (e_begin, e_count) != expert_partition(E, self.world)[self.rank]:
                raise ValueError("all_to_all dispatch needs the contiguous expert_partition "
                                 "ranges")
        self._bufs = {}

    @classmethod
    def partitioned(cls, all_weights_fn: Callable[[int, int], tuple], E: int, k: int, H: int,
                    I: int, group=None, **kw) -> "ExpertParallelMoE":
        """Builds this rank's share; ``all_weights_fn(begin, count)`` returns the
        prepared weights of experts ``begin .. begin + count - 1`` (or None)."""
        import torch.distributed as dist
        g, G = dist.get_rank(group), dist.get_world_size(group)
        b, n = expert_partition(E, G)[g]
        return cls(all_weights_fn(b, n) if n else None, E, k, b, n, H, I, group=group, **kw)

    def _buffers(self, T_max: int, device, dtype_out=torch.bfloat16):
        key = (T_max, str(device))
        if key not in self._bufs:
            H, k, G = self.H, self.k, self.world
            pad = PaddedBatch(codes=torch.zeros(T_max, H, dtype=torch.uint8, device=device),
                              scales=torch.zeros(T_max, dtype=torch.float32, device=device),
                              ids=torch.full((T_max, k), -1, dtype=torch.int32, device=device),
                              weights=torch.zeros(T_max, k, dtype=torch.float32, device=device))
            gat = PaddedBatch(codes=torch.empty(G * T_max, H, dtype=torch.uint8, device=device),
                              scales=torch.empty(G * T_max, dtype=torch.float32, device=device),
                              ids=torch.empty(G * T_max, k, dtype=torch.int32, device=device),
                              weights=torch.empty(G * T_max, k, dtype=torch.float32,
                                                  device=device))
            partial = torch.zeros(G * T_max, H, dtype=torch.float32, device=device)
            summed = torch.empty(T_max, H, dtype=torch.float32, device=device)
            self._bufs = {key: (pad, gat, partial, summed)}   # keep one size at a time
        return self._bufs[key]

    def padded_tokens(self, T_local: int, device) -> int:
        """The step's batch size every rank pads to (the largest batch)."""
        if self.tokens_per_rank is not None:
            if T_local != self.tokens_per_rank:
                raise ValueError(f"{T_local} tokens on a layer built for {self.tokens_per_rank}")
            return T_local
        t = torch.tensor([T_local], dtype=torch.int64, device=device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX, group=self.group)
        return int(t.item())

    def __call__(self, hidden: torch.Tensor, logits: torch.Tensor,
                 out: Optional[torch.Tensor] = None) -> torch.Tensor:
        if self.dispatch == "all_to_all":
            return self._all_to_all_step(hidden, logits, out)
        dist, group = self.dist, self.group
        T = hidden.shape[0]
        dev = hidden.device
        T_max = self.padded_tokens(T, dev)
        pad, gat, partial, summed = self._buffers(T_max, dev)
        if T < T_max:   # rows T .. T_max - 1 are padding: no expert, weight 0
            pad.ids[T:].fill_(-1)
            pad.weights[T:].zero_()
        self.ops.quant_route(hidden, logits, self.k, pad)
        # dispatch: every rank's tokens to every rank
        dist.all_gather_into_tensor(gat.codes, pad.codes, group=group)
        dist.all_gather_into_tensor(gat.scales, pad.scales, group=group)
        dist.all_gather_into_tensor(gat.ids, pad.ids, group=group)
        dist.all_gather_into_tensor(gat.weights, pad.weights, group=group)
        if self.e_count:
            self.ops.experts(gat.codes, gat.scales, gat.ids, gat.weights, self.E, self.e_begin,
                             self.weights_local, partial)
        else:
            partial.zero_()
        # combine: each rank receives the sums of its own tokens
        dist.reduce_scatter_tensor(summed, partial, op=dist.ReduceOp.SUM, group=group)
        if out is None:
            out = torch.empty(T, self.H, dtype=torch.bfloat16, device=dev)
        if T:
            self.ops.cast(summed[:T], out)
        return out


    def _all_to_all_step(self, hidden, logits, out):
        dist, group, G = self.dist, self.group, self.world
        H, k = self.H, self.k
        T = hidden.shape[0]
        dev = hidden.device
        loc = PaddedBatch(codes=torch.empty(T, H, dtype=torch.uint8, device=dev),
                          scales=torch.empty(T, dtype=torch.float32, device=dev),
                          ids=torch.empty(T, k, dtype=torch.int32, device=dev),
                          weights=torch.empty(T, k, dtype=torch.float32, device=dev))
        self.ops.quant_route(hidden, logits, k, loc)
        counts, rows, pos = self.ops.plan(loc.ids, self.E, G)
        send = counts.to(torch.int64)
        recv = torch.empty_like(send)
        dist.all_to_all_single(recv, send, group=group)
        send_l, recv_l = send.tolist(), recv.tolist()
        n_send, n_recv = sum(send_l), sum(recv_l)
        sb = self.ops.gather(loc, T, rows, n_send)
        rb = PaddedBatch(codes=torch.empty(n_recv, H, dtype=torch.uint8, device=dev),
                         scales=torch.empty(n_recv, dtype=torch.float32, device=dev),
                         ids=torch.empty(n_recv, k, dtype=torch.int32, device=dev),
                         weights=torch.empty(n_recv, k, dtype=torch.float32, device=dev))
        for got, sent in ((rb.codes, sb.codes), (rb.scales, sb.scales), (rb.ids, sb.ids),
                          (rb.weights, sb.weights)):
            dist.all_to_all_single(got, sent, output_split_sizes=recv_l,
                                   input_split_sizes=send_l, group=group)
        partial = torch.zeros(n_recv, H, dtype=torch.float32, device=dev)
        if self.e_count and n_recv:
            self.ops.experts(rb.codes, rb.scales, rb.ids, rb.weights, self.E, self.e_begin,
                             self.weights_local, partial)
        back = torch.empty(n_send, H, dtype=torch.float32, device=dev)
        dist.all_to_all_single(back, partial, output_split_sizes=send_l,
                               input_split_sizes=recv_l, group=group)
        if out is None:
            out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        if T:
            self.ops.combine(back, pos, out)
        return out


def init_process_group_with_timeout(backend: str, seconds: float = 60.0, **kw):
    """``torch.distributed.init_process_group`` with a short timeout, so that
    ranks waiting on a rank that has gone end with an error instead of
    hanging."""
    import torch.distributed as dist
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=seconds), **kw)
