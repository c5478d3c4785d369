"""GPU parity against the fp64 oracle at the workloads' full sizes, and at reduced sizes
that still reach every kernel instantiation those workloads launch.

This file is collected before the other GPU tests, so a run that stops at the first
failure has always compared the full-size selections with the oracle.

Which kernels each workload launches (the host planner decides):
  decode batch (bf16, 32 x 32768, 1 query):  logits <1 query per accumulator>, top-k
      clusters of 4 CTAs with 16 keys per thread, seeded by the epilogue's coarse histogram
      (rows of 16385..32768 keys);
  bf16 decode with a row longer than 32768 keys: the streaming top-k (every row);
  prefill (bf16) and long prefill (FP8): logits <8 queries per item>, the short-row kernel
      (rows within top_k) and the row-streaming top-k, whose sampled-threshold pass runs
      on rows longer than 4096 keys;
  ragged decode (FP8, 2 queries): logits <2 queries per accumulator>, the row-histogram
      pass and the streaming top-k.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_token_02_b200 import api
from sparse_attention_token_02_b200 import workloads as W

from ._parity import Uploaded, check_rows, run_indexer, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    api.dsa_version()          # the CUDA library must load
    yield
    api.dsa_check_device_errors()


# ----------------------------------------------------------------------------- full-size workloads

def test_full_decode_batch_all_rows():
    wl = W.decode()
    up = Uploaded(wl)
    idx, sc = run_indexer(up, decode=True)
    check_rows(up, idx, sc, range(wl.total_q))


def test_full_prefill_bf16_sampled_rows():
    wl = W.prefill()
    up = Uploaded(wl)
    idx, sc = run_indexer(up)
    rows = sample_rows(wl, n_mid=10) + [4095, 4096, 4097, 8191, 12000]
    check_rows(up, idx, sc, sorted(set(rows)))


def test_full_prefill_fp8_sampled_rows():
    wl = W.prefill8()
    up = Uploaded(wl)
    # the library's FP8 codes for the sampled query rows equal the oracle codec's
    rows = sorted(set(sample_rows(wl, n_mid=8) + [4097, 30000, 65000]))
    bits = up.inp["q_bits"][rows].reshape(len(rows), -1)
    codes, scale = oracle.quantize_rows(oracle.bf16_bits_to_f64(bits).astype(np.float32))
    assert np.array_equal(up.q[rows].reshape(len(rows), -1).cpu().numpy(), codes)
    assert np.array_equal(up.q_scale[rows].cpu().numpy(), scale)
    idx, sc = run_indexer(up)
    check_rows(up, idx, sc, rows)


def test_full_ragged_decode_fp8_sampled_sequences():
    wl = W.decode8()
    up = Uploaded(wl)
    idx, sc = run_indexer(up, decode=True)
    order = np.argsort(wl.seq_lens)
    seqs = [int(order[0]), int(order[-1]), int(order[len(order) // 2]), int(order[len(order) // 4])]
    rows = sorted(2 * b + j for b in seqs for j in (0, 1))
    check_rows(up, idx, sc, rows)


# ----------------------------------------------------------------------------- reduced sizes, same kernels

@pytest.mark.parametrize("q_len", [1, 2])
def test_decode_bf16_cluster_rows_of_16k_to_32k_keys(q_len):
    # rows of 16385..32768 keys: 4-CTA clusters at 16 keys a thread, the decode batch's top-k
    lens = (20000, 32768, 16385, 25000, 30001)
    wl = W.scaled(W.decode(), seq_lens=lens, q_lens=(q_len,) * len(lens), seed=60 + q_len)
    up = Uploaded(wl)
    idx, sc = run_indexer(up, decode=True)
    check_rows(up, idx, sc, range(wl.total_q))


def test_decode_bf16_rows_beyond_32k_keys_stream():
    # one row longer than a 4-CTA cluster holds sends every row of the batch to the streaming top-k
    lens = (40000, 33000, 5000, 2049, 32768, 8192, 8193)
    wl = W.scaled(W.decode(), seq_lens=lens, q_lens=(2,) * len(lens), seed=64)
    up = Uploaded(wl)
    idx, sc = run_indexer(up, decode=True)
    check_rows(up, idx, sc, range(wl.total_q))


@pytest.mark.parametrize("name", ["bf16", "fp8"])
def test_prefill_rows_beyond_4096_keys_take_the_sampled_threshold(name):
    # rows longer than 4096 keys go through the row top-k's sampled-threshold pass
    base = W.prefill() if name == "bf16" else W.prefill8()
    wl = W.scaled(base, seq_lens=(6000,), q_lens=(6000,), seed=70 if name == "bf16" else 71)
    up = Uploaded(wl)
    idx, sc = run_indexer(up)
    rng = np.random.default_rng(5)
    rows = set(range(4090, 4110)) | set(range(5980, 6000)) | set(int(x) for x in rng.integers(4097, 6000, 40))
    rows |= {0, 2046, 2047, 2048, 2049, 3000}
    check_rows(up, idx, sc, sorted(rows))


def test_ragged_decode_fp8_longest_and_shortest_rows():
    # FP8 decode: the row-histogram pass and the streaming top-k over 4096 .. 131072 keys; rows at
    # the chunk boundaries (one, two and three chunks of 4096 keys, and five)
    lens = (131072, 4096, 70001, 4097, 8192, 8193, 16385)
    wl = W.scaled(W.decode8(), seq_lens=lens, q_lens=(2,) * len(lens), seed=72)
    up = Uploaded(wl)
    idx, sc = run_indexer(up, decode=True)
    check_rows(up, idx, sc, range(wl.total_q))
