"""The selection's consumers on the GPU (latent-row gather, int64 rows, sorted order),
element by element against oracle/after_select.py on selections made by the indexer."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import after_select as A
from sparse_attention_token_02_b200 import api
from sparse_attention_token_02_b200 import workloads as W

from ._parity import Uploaded

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    api.dsa_version()
    yield
    api.dsa_check_device_errors()


@pytest.fixture(scope="module")
def selection():
    """A ragged decode selection (1-2 queries per sequence, rows shorter and longer than k)."""
    wl = W.scaled(W.decode(), seq_lens=(5000, 700, 2049, 3100), q_lens=(2, 1, 1, 2), top_k=512, seed=60)
    up = Uploaded(wl)
    idx, sc = api.dsa_indexer_decode(up.q, up.cache, up.w, wl.seq_lens, wl.q_lens, wl.top_k, k_base=up.k_base)
    api.dsa_check_device_errors()
    base = api.selection_row_base(wl.seq_lens, wl.q_lens, up.k_base)
    return wl, idx, sc, base


@pytest.mark.parametrize("row_bytes", [1024, 656])      # bf16 d_c = 512; 656-byte FP8-style rows
def test_gather_rows_bit_exact(selection, row_bytes):
    wl, idx, _, base = selection
    rows = int(sum(wl.seq_lens))
    g = torch.Generator().manual_seed(row_bytes)
    src = torch.randint(0, 256, (rows, row_bytes), dtype=torch.uint8, generator=g).cuda()
    out = api.dsa_gather_rows(src, idx, base)
    api.dsa_check_device_errors()
    ref = A.gather_rows(src.cpu().numpy(), idx.cpu().numpy(), base.cpu().numpy())
    assert np.array_equal(out.cpu().numpy(), ref)


@pytest.mark.parametrize("rows,row_bytes", [(300, 16), (40, 1024), (16, 4096), (7, 48)])
def test_gather_rows_many_batches_per_warp(rows, row_bytes):
    # synthetic selections (padding included) large enough that every warp copies several
    # 32-entry batches, over the narrowest, the widest and an odd number of vectors per row
    top_k, src_rows = 2048, 50000
    rng = np.random.default_rng(rows * row_bytes)
    idx = rng.integers(0, 40000, (rows, top_k)).astype(np.int32)
    idx[rng.random((rows, top_k)) < 0.1] = -1
    base = rng.integers(0, src_rows - 40000, rows).astype(np.int64)
    src = torch.randint(0, 256, (src_rows, row_bytes), dtype=torch.uint8,
                        generator=torch.Generator().manual_seed(rows)).cuda()
    out = api.dsa_gather_rows(src, torch.from_numpy(idx).cuda(), torch.from_numpy(base).cuda())
    api.dsa_check_device_errors()
    assert np.array_equal(out.cpu().numpy(), A.gather_rows(src.cpu().numpy(), idx, base))


def test_gather_rows_bf16_view_and_out_of_range_row(selection):
    wl, idx, _, base = selection
    rows = int(sum(wl.seq_lens))
    src = torch.randn(rows, 512, dtype=torch.bfloat16, device="cuda")
    out = api.dsa_gather_rows(src, idx, base)
    ref = A.gather_rows(src.view(torch.uint8).cpu().numpy(), idx.cpu().numpy(), base.cpu().numpy())
    assert np.array_equal(out.view(torch.uint8).cpu().numpy().reshape(ref.shape), ref)
    bad = idx.clone()
    bad[0, 0] = rows + 5                                      # past the cache: zero-filled and reported
    out = api.dsa_gather_rows(src, bad, base)
    with pytest.raises(RuntimeError, match="DEVICE_CHECK"):
        api.dsa_check_device_errors()
    assert not out[0, 0].view(torch.uint8).any()


def test_selection_rows(selection):
    _, idx, _, base = selection
    got = api.dsa_selection_rows(idx, base).cpu().numpy()
    assert np.array_equal(got, A.selection_rows(idx.cpu().numpy(), base.cpu().numpy()))


def test_sort_selection_matches_oracle_order(selection):
    _, idx, sc, _ = selection
    i2, s2 = idx.clone(), sc.clone()
    api.dsa_sort_selection(i2, s2)
    api.dsa_check_device_errors()
    ref_i, ref_s = A.sort_selection(idx.cpu().numpy(), sc.cpu().numpy())
    assert np.array_equal(i2.cpu().numpy(), ref_i)
    assert np.array_equal(s2.cpu().numpy(), ref_s)


def test_sort_selection_ties_and_sizes():
    g = torch.Generator().manual_seed(7)
    for k in (1, 3, 100, 2048, 4096):
        T = 5
        idx = torch.stack([torch.randperm(10000, generator=g)[:k] for _ in range(T)]).to(torch.int32)
        sc = torch.randint(-2, 3, (T, k), generator=g).to(torch.float32)
        idx[:, k // 2:] = torch.where(torch.rand(T, k - k // 2, generator=g) < 0.3, -1, idx[:, k // 2:])
        sc[idx < 0] = float("-inf")
        i2, s2 = idx.cuda(), sc.cuda()
        api.dsa_sort_selection(i2, s2)
        ref_i, ref_s = A.sort_selection(idx.numpy(), sc.numpy())
        assert np.array_equal(i2.cpu().numpy(), ref_i), k
        assert np.array_equal(s2.cpu().numpy(), ref_s), k
    with pytest.raises(RuntimeError, match="UNSUPPORTED"):
        api.dsa_sort_selection(torch.zeros(1, 4097, dtype=torch.int32, device="cuda"),
                               torch.zeros(1, 4097, dtype=torch.float32, device="cuda"))
