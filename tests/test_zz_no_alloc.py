"""dsa_indexer_decode_noalloc: the decode entry point for callers that may not allocate
device memory (its scratch lives in a static array inside the library).

Checked through the C ABI against the regular dsa_indexer_decode on the same inputs and
against the fp64 oracle, two calls in a row with different batches (the second call must
not be disturbed by what the first left in the shared array), and for its size limit.
This file is collected last so that a run stopping at the first failure has run every
other test.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from sparse_attention_token_02_b200 import api
from sparse_attention_token_02_b200 import workloads as W

from ._parity import RTOL, Uploaded, check_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    api.dsa_version()


def _same_selection(idx_a, sc_a, idx_b, sc_b, top_k, rtol):
    """Index sets equal except near-ties at the k-th score; scores within rtol."""
    for r in range(idx_a.shape[0]):
        va, vb = idx_a[r] >= 0, idx_b[r] >= 0
        assert va.sum() == vb.sum(), f"row {r}: valid counts differ"
        m = int(va.sum())
        a = dict(zip(idx_a[r][:m].tolist(), sc_a[r][:m].tolist()))
        b = dict(zip(idx_b[r][:m].tolist(), sc_b[r][:m].tolist()))
        kth = min(a.values()) if m == top_k else max(a.values())
        floor = max(abs(kth), 1e-30)
        for i in a.keys() & b.keys():
            assert abs(a[i] - b[i]) <= rtol * max(abs(a[i]), floor), f"row {r} index {i}"
        for i in a.keys() ^ b.keys():
            s = a.get(i, b.get(i))
            assert abs(s - kth) <= rtol * floor, f"row {r}: index {i} selected by one call only"


def test_noalloc_decode_matches_regular_decode_two_calls_in_a_row():
    cases = [W.scaled(W.decode(), seq_lens=(5000, 2049, 300, 9000), q_lens=(1,) * 4, seed=21),
             W.scaled(W.decode(), seq_lens=(4000, 3000, 2500, 1), q_lens=(2, 2, 2, 1), seed=22)]
    for wl in cases:
        up = Uploaded(wl)
        ref_i, ref_s = api.dsa_indexer_decode(up.q, up.cache, up.w, wl.seq_lens, wl.q_lens, wl.top_k,
                                              q_scale=up.q_scale, k_base=up.k_base)
        fault = torch.full((2,), 7, dtype=torch.int32, device="cuda")   # the call must clear it
        got_i, got_s = api.dsa_indexer_decode_noalloc(up.q, up.cache, up.w, wl.seq_lens, wl.q_lens, wl.top_k,
                                                      q_scale=up.q_scale, k_base=up.k_base, fault=fault)
        torch.cuda.synchronize()
        assert fault.cpu().tolist() == [0, 0]
        _same_selection(ref_i.cpu().numpy(), ref_s.cpu().numpy(), got_i.cpu().numpy(), got_s.cpu().numpy(),
                        wl.top_k, RTOL[wl.dtype])
        check_rows(up, got_i.cpu().numpy(), got_s.cpu().numpy(), range(wl.total_q))
    api.dsa_check_device_errors()


def test_noalloc_decode_fp8_and_without_fault_pointer():
    wl = W.scaled(W.decode8(), seq_lens=(6000, 2100, 3333), q_lens=(2, 2, 2))
    up = Uploaded(wl)
    ref_i, ref_s = api.dsa_indexer_decode(up.q, up.cache, up.w, wl.seq_lens, wl.q_lens, wl.top_k,
                                          q_scale=up.q_scale, k_base=up.k_base)
    for _ in range(2):
        got_i, got_s = api.dsa_indexer_decode_noalloc(up.q, up.cache, up.w, wl.seq_lens, wl.q_lens, wl.top_k,
                                                      q_scale=up.q_scale, k_base=up.k_base)
        torch.cuda.synchronize()
        _same_selection(ref_i.cpu().numpy(), ref_s.cpu().numpy(), got_i.cpu().numpy(), got_s.cpu().numpy(),
                        wl.top_k, RTOL[wl.dtype])
        check_rows(up, got_i.cpu().numpy(), got_s.cpu().numpy(), range(wl.total_q))


def test_noalloc_decode_tables_larger_than_one_parameter_chunk():
    # 300 sequences x 2 queries: the scheduling tables (about 25 KB) reach the static array
    # in two kernel-parameter chunks
    rng = np.random.default_rng(7)
    lens = tuple(int(x) for x in rng.integers(2100, 3000, 300))
    wl = W.scaled(W.decode(), seq_lens=lens, q_lens=(2,) * len(lens), seed=23)
    up = Uploaded(wl)
    got_i, got_s = api.dsa_indexer_decode_noalloc(up.q, up.cache, up.w, wl.seq_lens, wl.q_lens, wl.top_k,
                                                  q_scale=up.q_scale, k_base=up.k_base)
    torch.cuda.synchronize()
    got_i, got_s = got_i.cpu().numpy(), got_s.cpu().numpy()
    rows = list(range(0, wl.total_q, 7)) + [wl.total_q - 1]
    check_rows(up, got_i, got_s, rows)
    api.dsa_check_device_errors()


def test_noalloc_decode_rejects_batches_beyond_its_scratch():
    # 40 queries over 131072 keys each need 21 MB of score rows: more than the 16 MiB array
    L, n = 131072, 40
    cache = api.IndexerKCache.empty(L, 128, fp8=False)
    q = torch.zeros(n, 64, 128, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(n, 64, dtype=torch.float32, device="cuda")
    with pytest.raises(RuntimeError, match="INVALID_ARG.*scratch"):
        api.dsa_indexer_decode_noalloc(q, cache, w, [L] * n, [1] * n, 2048, k_base=np.zeros(n, np.int64))
