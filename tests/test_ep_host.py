"""Expert parallelism on CPU ranks (gloo): the bookkeeping and collectives of
``w4a8_quantized_moe_b200.ep`` with the oracle standing in for the library's
compute steps.

Each rank owns a contiguous expert range, quantises and routes its own
tokens, all-gathers them, computes its experts' float32 partial sums and
reduce-scatters them back; or, with the all-to-all(v) dispatch, sends each
token only to the ranks of its experts and adds the partial sums that come
back.  Every rank's output must match the single-process
oracle's ``moe_forward`` on that rank's tokens.  Cases: 2 and 4 ranks, equal
and uneven batches (a rank with no tokens), a rank whose experts no token
chooses, a rank that holds no experts (more ranks than experts), and a rank
that leaves between steps, which the others must notice as an error within
the process group's timeout instead of hanging.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import workloads
from ep_reference import combine_reference, plan_reference
from w4a8_quantized_moe_b200.ep import ExpertParallelMoE, PaddedBatch, expert_partition


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _f64(t: torch.Tensor) -> np.ndarray:
    return oracle.bf16_bits_to_f64(t.contiguous().view(torch.int16).numpy().view(np.uint16))


class OracleOps:
    """The compute steps of one expert-parallel step, by the oracle on CPU tensors."""

    def quant_route(self, hidden, logits, k, batch: PaddedBatch):
        T = hidden.shape[0]
        if T == 0:
            return
        codes, scales = oracle.quant_act_fp8_per_token(_f64(hidden))
        ids, w = oracle.route_topk(logits.numpy(), k)
        batch.codes[:T] = torch.from_numpy(codes)
        batch.scales[:T] = torch.from_numpy(scales.astype(np.float32))
        batch.ids[:T] = torch.from_numpy(ids)
        batch.weights[:T] = torch.from_numpy(w)

    def experts(self, codes, scales, ids, weights, E, e_begin, weights_local, out):
        x = scales.numpy().astype(np.float64)[:, None] * oracle.e4m3_decode(codes.numpy())
        ids_, w_ = ids.numpy(), weights.numpy().astype(np.float64)
        T, k = ids_.shape
        Y = {}
        for le, expert in enumerate(weights_local):
            rows = np.argwhere(ids_ == e_begin + le)        # (t, j), t ascending
            if len(rows):
                _, _, _, y = oracle.expert_forward(x[rows[:, 0]], expert)
                for (t, j), yy in zip(rows, y):
                    Y[(int(t), int(j))] = yy
        acc = np.zeros((T, codes.shape[1]))
        for t in range(T):
            for j in range(k):                               # slot order
                if (t, j) in Y:
                    acc[t] = acc[t] + w_[t, j] * Y[(t, j)]
        out.copy_(torch.from_numpy(acc.astype(np.float32)))
        return out

    def cast(self, x, out):
        bits = oracle.f64_to_bf16_bits(x.numpy().astype(np.float64))
        out.copy_(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16))
        return out

    # the all-to-all(v) dispatch, from its definition: token t goes to rank r
    # once when one of its ids lies in r's expert range; rank-major, tokens
    # ascending; the combine sums a token's returned rows in rank order
    def plan(self, ids, E, n):
        return plan_reference(ids.numpy(), E, n)

    def gather(self, batch, T, rows, n_rows):
        r = rows[:n_rows].long()
        return PaddedBatch(codes=batch.codes[:T][r], scales=batch.scales[:T][r],
                           ids=batch.ids[:T][r], weights=batch.weights[:T][r])

    def combine(self, back, pos, out):
        return self.cast(torch.from_numpy(combine_reference(back.numpy(), pos.numpy())), out)


def _cfg(E, forced_empty=0):
    return workloads.MoEConfig("ep", T=0, H=256, I=128, E=E, k=2, seed=77,
                               forced_empty=forced_empty)


def _experts(cfg, begin, count):
    store = oracle.ExpertStore(cfg.E, lambda e: tuple(_f64(w) for w in
                                                      workloads.gen_expert_weights(cfg, e)))
    return [store[e] for e in range(begin, begin + count)]


def _batch(cfg, rank, T):
    c = cfg.with_(T=T, seed=cfg.seed + 101 * rank)
    hidden = workloads.gen_hidden(c)
    logits = workloads.gen_logits(c)
    if cfg.forced_empty:   # the LAST experts (another rank's) are never chosen
        logits[:, cfg.E - cfg.forced_empty:] = -float("inf")
    return hidden, logits


def _init(rank, world, port, timeout_s):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=timeout_s))


def _ep_worker(rank, world, port, E, tokens, forced_empty, steps, q, dispatch):
    _init(rank, world, port, 60)
    try:
        cfg = _cfg(E, forced_empty)
        begin, count = expert_partition(E, world)[rank]
        layer = ExpertParallelMoE(_experts(cfg, begin, count) if count else None, E, cfg.k,
                                  begin, count, cfg.H, cfg.I, ops=OracleOps(), dispatch=dispatch)
        hidden, logits = _batch(cfg, rank, tokens[rank])
        outs = [layer(hidden, logits) for _ in range(steps)]
        # the single-process oracle on this rank's tokens, all experts
        store = oracle.ExpertStore(E, lambda e: tuple(_f64(w) for w in
                                                      workloads.gen_expert_weights(cfg, e)))
        if tokens[rank]:
            ref = oracle.moe_forward(_f64(hidden), logits.numpy(), store, cfg.k)["out"]
        else:
            ref = np.zeros((0, cfg.H))
        q.put((rank, [_f64(o) for o in outs], ref, count))
    except Exception as e:  # report, never hang the parent
        q.put((rank, repr(e), None, None))
    finally:
        dist.destroy_process_group()


def _run(world, E, tokens, forced_empty=0, steps=1, dispatch="all_gather"):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_ep_worker,
                         args=(r, world, port, E, tokens, forced_empty, steps, q, dispatch))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


def _check(res, tokens):
    for rank, outs, ref, _ in res:
        assert not isinstance(outs, str), f"rank {rank}: {outs}"
        for out in outs:
            assert out.shape == (tokens[rank], 256)
            if tokens[rank] == 0:
                continue
            err = np.linalg.norm(out - ref) / np.linalg.norm(ref)
            same = np.mean(out == ref)
            # float32 partial sums reduced across ranks, then one bf16 rounding:
            # equal to the float64 oracle except where a sum sits at a bf16 midpoint
            assert err <= 2e-3 and same >= 0.99, (rank, err, same)


def test_partition_covers_every_expert_once():
    for E in (1, 5, 8, 256):
        for G in (1, 2, 3, 4, 8):
            parts = expert_partition(E, G)
            assert len(parts) == G
            assert sum(n for _, n in parts) == E
            assert [b for b, _ in parts] == list(np.cumsum([0] + [n for _, n in parts[:-1]]))
            assert max(n for _, n in parts) - min(n for _, n in parts) <= 1
    with pytest.raises(ValueError):
        expert_partition(0, 2)


def test_two_ranks_equal_batches_two_steps():
    tokens = [16, 16]
    _check(_run(2, 8, tokens, steps=2), tokens)


def test_four_ranks_uneven_batches_and_an_unchosen_rank():
    # E = 6 over 4 ranks: 2, 2, 1, 1 experts; expert 5 (rank 3's only expert)
    # is forced to -inf, so rank 3's experts receive no token; rank 2 has no tokens
    tokens = [5, 16, 0, 3]
    res = _run(4, 6, tokens, forced_empty=1)
    _check(res, tokens)
    assert [c for *_, c in res] == [2, 2, 1, 1]


def test_more_ranks_than_experts():
    tokens = [4, 7, 2]
    res = _run(3, 2, tokens)
    _check(res, tokens)
    assert [c for *_, c in res] == [1, 1, 0]


def test_plan_reference_is_the_definition():
    # 3 ranks over E = 7 experts: 3, 2, 2 (ranges [0,3), [3,5), [5,7))
    ids = np.array([[0, 4], [6, 5], [-1, -1], [1, 2], [3, 6], [4, 4]], dtype=np.int32)
    counts, rows, pos = plan_reference(ids, 7, 3)
    assert counts.tolist() == [2, 3, 2]
    assert rows[:7].tolist() == [0, 3, 0, 4, 5, 1, 4]
    assert pos.tolist() == [[0, 2, -1], [-1, -1, 5], [-1, -1, -1], [1, -1, -1], [-1, 3, 6],
                            [-1, 4, -1]]
    back = np.arange(7 * 2, dtype=np.float32).reshape(7, 2)
    out = combine_reference(back, pos.numpy())
    assert out.tolist() == [[4, 6], [10, 11], [0, 0], [2, 3], [18, 20], [8, 9]]


def test_all_to_all_two_ranks_two_steps():
    tokens = [16, 16]
    _check(_run(2, 8, tokens, steps=2, dispatch="all_to_all"), tokens)


def test_all_to_all_four_ranks_uneven_batches_and_an_unchosen_rank():
    tokens = [5, 16, 0, 3]
    res = _run(4, 6, tokens, forced_empty=1, dispatch="all_to_all")
    _check(res, tokens)
    assert [c for *_, c in res] == [2, 2, 1, 1]


def test_all_to_all_more_ranks_than_experts():
    tokens = [4, 7, 2]
    res = _run(3, 2, tokens, dispatch="all_to_all")
    _check(res, tokens)


def _range_worker(port, q):
    _init(0, 1, port, 30)
    try:
        ExpertParallelMoE(None, 4, 2, 1, 3, 256, 128, ops=OracleOps(), dispatch="all_to_all")
        q.put("accepted")
    except ValueError:
        q.put("ValueError")
    finally:
        dist.destroy_process_group()


def test_all_to_all_needs_the_partition_ranges():
    # one rank must own all 4 experts under the partition; [1, 4) is refused
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_range_worker, args=(_free_port(), q))
    p.start()
    assert q.get(timeout=120) == "ValueError"
    p.join(timeout=60)


def _leaving_worker(rank, world, port, q):
    _init(rank, world, port, 5)
    cfg = _cfg(4)
    begin, count = expert_partition(4, world)[rank]
    layer = ExpertParallelMoE(_experts(cfg, begin, count), 4, cfg.k, begin, count, cfg.H,
                              cfg.I, ops=OracleOps(), tokens_per_rank=4)
    hidden, logits = _batch(cfg, rank, 4)
    layer(hidden, logits)                     # step 1 on both ranks
    if rank == 1:
        os._exit(0)                           # leaves between steps, nothing in flight
    try:
        layer(hidden, logits)                 # step 2: the peer is gone
        q.put("returned")
    except Exception as e:
        q.put(type(e).__name__)


def test_rank_leaving_between_steps_fails_the_next_step_not_hangs():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_leaving_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    outcome = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
    assert outcome != "returned"
