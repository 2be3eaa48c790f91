"""The all-to-all(v) dispatch and combine of expert parallelism, written from
their definition for the tests (host bookkeeping; no arithmetic of the layer).

Rank r of n owns the contiguous expert range of ``expert_partition(E, n)``.
Token t goes to rank r once when one of its ids lies in r's range (ids
outside [0, E) go nowhere); the send list is rank-major with tokens ascending
inside each rank.  The combine adds a token's returned rows in rank order in
float32.
"""
import numpy as np
import torch

from w4a8_quantized_moe_b200.ep import expert_partition


def plan_reference(ids: np.ndarray, E: int, n: int):
    """(counts int32 [n], rows int32 [max(T * min(k, n), 1)], pos int32 [T, n])."""
    T, k = ids.shape
    owner = np.full(E, -1)
    for r, (b, c) in enumerate(expert_partition(E, n)):
        owner[b:b + c] = r
    pos = np.full((T, n), -1, dtype=np.int32)
    rows, counts = [], []
    for r in range(n):
        mine = [t for t in range(T) if any(0 <= e < E and owner[e] == r for e in ids[t])]
        for t in mine:
            pos[t, r] = len(rows)
            rows.append(t)
        counts.append(len(mine))
    rows_out = np.zeros(max(T * min(k, n), 1), dtype=np.int32)
    rows_out[:len(rows)] = rows
    return (torch.tensor(counts, dtype=torch.int32), torch.from_numpy(rows_out),
            torch.from_numpy(pos))


def combine_reference(back: np.ndarray, pos: np.ndarray) -> np.ndarray:
    """float32 [T, H]: each token's rows back[pos[t, r]] added in rank order."""
    T, n = pos.shape
    acc = np.zeros((T, back.shape[1]), dtype=np.float32)
    for r in range(n):
        m = pos[:, r] >= 0
        acc[m] = acc[m] + back[pos[m, r]]
    return acc
