"""Sharding a ragged batch over several GPUs (one process per GPU).

Every (sequence, query) row of the indexer is independent: a query only reads its own
sequence's keys ("Lightning Indexer 详解" §2: one query scores its own cached history).  A
batch therefore splits across ranks by whole sequences, each rank runs the whole path on
its share, and nothing crosses between GPUs on the data path.  These helpers choose the
split (balanced by scored pairs) and put per-rank results back in batch order.
"""

from __future__ import annotations

import heapq

import numpy as np


def pairs_of(seq_len: int, q_len: int) -> int:
    """Causal (query, key) pairs of one sequence: queries at positions seq_len-q_len .. seq_len-1."""
    first = seq_len - q_len
    return q_len * (first + 1) + q_len * (q_len - 1) // 2


def shard_sequences(seq_lens, q_lens, world: int) -> list[list[int]]:
    """Split sequence ids over `world` ranks, longest-processing-time first on scored pairs.

    Every sequence goes to exactly one rank; each rank's list is in increasing id order.
    """
    if world < 1:
        raise ValueError("world must be >= 1")
    q_lens = list(seq_lens) if q_lens is None else list(q_lens)
    cost = [pairs_of(int(L), int(n)) for L, n in zip(seq_lens, q_lens)]
    order = sorted(range(len(cost)), key=lambda b: (-cost[b], b))
    heap = [(0, r) for r in range(world)]
    out = [[] for _ in range(world)]
    for b in order:
        load, r = heapq.heappop(heap)
        out[r].append(b)
        heapq.heappush(heap, (load + cost[b], r))
    return [sorted(x) for x in out]


def query_rows(q_lens, ids) -> np.ndarray:
    """Packed query rows (in the whole batch) of the given sequences, in the order of ids."""
    q_lens = np.asarray(q_lens, dtype=np.int64)
    off = np.concatenate([[0], np.cumsum(q_lens)[:-1]])
    return np.concatenate([off[b] + np.arange(q_lens[b]) for b in ids]) if len(ids) else np.zeros(0, np.int64)


def unshard_rows(total_rows: int, parts) -> np.ndarray:
    """Reassemble per-rank row blocks: parts = [(rows, values[len(rows), ...]), ...]."""
    parts = [(np.asarray(r), np.asarray(v)) for r, v in parts]
    shape = next((v.shape[1:] for _, v in parts if v.size), ())
    dtype = next((v.dtype for _, v in parts if v.size), np.float64)
    out = np.zeros((total_rows,) + tuple(shape), dtype=dtype)
    seen = np.zeros(total_rows, dtype=bool)
    for rows, vals in parts:
        if np.any(seen[rows]):
            raise ValueError("a row came from two ranks")
        out[rows] = vals
        seen[rows] = True
    if not seen.all():
        raise ValueError("some rows came from no rank")
    return out
