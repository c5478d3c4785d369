"""The multi-GPU path on CPU: world-size-2 gloo process groups.

Ranks split a ragged batch by sequence (sharding.shard_sequences), each runs the indexer
(here the oracle, on CPU) on its share only, results are all-gathered and reassembled, and
must equal one process running the whole batch.  The bench's job aggregation (max time over
ranks, pairs of all ranks) is checked on the same process group.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from sparse_attention_token_02_b200 import sharding
from sparse_attention_token_02_b200 import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _batch():
    return W.scaled(W.prefill(), seq_lens=(120, 300, 45, 260, 90, 7), q_lens=(120, 40, 45, 1, 90, 7), top_k=32)


def _oracle_rows(wl, inp, ids):
    rows = sharding.query_rows(wl.q_lens, ids)
    ks = [oracle.bf16_bits_to_f64(inp["k_bits"][b]) for b in ids]
    q = oracle.bf16_bits_to_f64(inp["q_bits"][rows])
    w = inp["w"][rows].astype(np.float64)
    res = oracle.prefill_oracle(q, ks, w, [wl.seq_lens[b] for b in ids], [wl.q_lens[b] for b in ids], wl.top_k)
    return rows, res["idx"], res["score"]


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = _batch()
        inp = W.make_inputs(wl)
        mine = sharding.shard_sequences(wl.seq_lens, wl.q_lens, world)[rank]
        rows, idx, score = _oracle_rows(wl, inp, mine)
        parts = [None] * world
        dist.all_gather_object(parts, (rows, idx, score))
        # the bench's aggregation: slowest rank's time, every rank's pairs
        import bench
        ms = bench.max_over_ranks(1.0 + rank, dist)
        value = bench.job_value(wl.pairs, world, ms)
        if rank == 0:
            out_q.put((parts, ms, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_sharding_is_balanced_and_complete():
    wl = _batch()
    shards = sharding.shard_sequences(wl.seq_lens, wl.q_lens, 2)
    assert sorted(shards[0] + shards[1]) == list(range(len(wl.seq_lens)))
    loads = [sum(sharding.pairs_of(wl.seq_lens[b], wl.q_lens[b]) for b in s) for s in shards]
    assert sum(loads) == wl.pairs
    biggest = max(sharding.pairs_of(L, n) for L, n in zip(wl.seq_lens, wl.q_lens))
    assert max(loads) - min(loads) <= biggest
    assert sharding.shard_sequences([5, 5, 5], None, 4)[3] == []


def test_two_gloo_ranks_reproduce_the_single_process_result():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        parts, ms, value = q.get(timeout=240)
    finally:
        for p in procs:
            p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)
    wl = _batch()
    inp = W.make_inputs(wl)
    _, ref_idx, ref_score = _oracle_rows(wl, inp, list(range(len(wl.seq_lens))))
    T = wl.total_q
    idx = sharding.unshard_rows(T, [(r, i) for r, i, _ in parts])
    score = sharding.unshard_rows(T, [(r, s) for r, _, s in parts])
    assert np.array_equal(idx, ref_idx)
    assert np.array_equal(score, ref_score)
    assert ms == 2.0                                   # max over ranks of (1.0, 2.0)
    assert value == pytest.approx(wl.pairs * 2 / 2.0e-3)
