"""Pins for the oracle's top-k routing and expert permutation (CPU only)."""
import math

import numpy as np
import pytest
import torch

from oracle import permute_by_expert, route_topk


def test_topk_matches_torch_without_ties():
    rng = np.random.default_rng(1)
    for T, E, k in [(64, 256, 8), (17, 8, 2), (5, 1, 1), (33, 1024, 32)]:
        l = rng.standard_normal((T, E)).astype(np.float32)
        ids, w = route_topk(l, k)
        tv, ti = torch.topk(torch.from_numpy(l), k, dim=1, sorted=True)
        assert np.array_equal(ids, ti.numpy().astype(np.int32))
        # weights: softmax of the selected logits (library routine on the same values)
        ref = torch.softmax(tv.double(), dim=1).float().numpy()
        assert np.allclose(w, ref, rtol=1e-6, atol=0)
        assert np.all(np.abs(w.astype(np.float64).sum(axis=1) - 1.0) <= k * 2.0 ** -24)


def test_topk_ties_prefer_lower_expert_id():
    l = np.zeros((3, 8), dtype=np.float32)
    l[1, [5, 2, 7]] = 1.0
    l[2] = [0.5, 2.0, 0.5, 2.0, -1.0, 0.5, 2.0, 0.5]
    ids, w = route_topk(l, 3)
    assert ids[0].tolist() == [0, 1, 2]
    assert np.all(w[0] == np.float32(1.0 / 3.0))
    assert ids[1].tolist() == [2, 5, 7]
    assert ids[2].tolist() == [1, 3, 6]


def test_topk_closed_forms_and_neg_inf():
    l = np.array([[0.0, 1.5, -math.inf, 0.25],
                  [-math.inf, -math.inf, 3.0, -math.inf]], dtype=np.float32)
    ids, w = route_topk(l, 1)
    assert ids[:, 0].tolist() == [1, 2] and np.all(w == 1.0)
    ids, w = route_topk(l[:1], 2)
    assert ids[0].tolist() == [1, 3]
    assert w[0, 0] == np.float32(1.0 / (1.0 + math.exp(0.25 - 1.5)))
    ids, w = route_topk(l[:1], 3)
    assert 2 not in ids[0]                               # -inf never chosen while finite ones remain


def _brute_permute(ids, E):
    T, k = ids.shape
    offsets = [0]
    sorted_tok, row_of = [], np.full((T, k), -1)
    for e in range(E):
        for t in range(T):
            for j in range(k):
                if ids[t, j] == e:
                    row_of[t, j] = len(sorted_tok)
                    sorted_tok.append(t)
        offsets.append(len(sorted_tok))
    return np.array(offsets), np.array(sorted_tok), row_of


@pytest.mark.parametrize("T,E,k", [(16, 8, 2), (37, 5, 3), (1, 4, 4), (64, 256, 8)])
def test_permutation_brute_force_and_invariants(T, E, k):
    rng = np.random.default_rng(T * 1000 + E)
    l = rng.standard_normal((T, E)).astype(np.float32)
    l[:, rng.choice(E, max(0, E // 4), replace=False)] -= 4.0     # skew: some experts rare/empty
    ids, _ = route_topk(l, k)
    off, st, ro = permute_by_expert(ids, E)
    boff, bst, bro = _brute_permute(ids, E)
    assert np.array_equal(off, boff) and np.array_equal(st, bst) and np.array_equal(ro, bro)
    assert off[0] == 0 and off[-1] == T * k and np.all(np.diff(off) >= 0)
    for t in range(T):
        for j in range(k):
            r = ro[t, j]
            assert st[r] == t and off[ids[t, j]] <= r < off[ids[t, j] + 1]
    for e in range(E):
        seg = st[off[e]:off[e + 1]]
        assert np.all(np.diff(seg) > 0), "segments are in ascending token order"
