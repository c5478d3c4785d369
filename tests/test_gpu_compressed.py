"""Decode over an m-compressed key cache against oracle.decode_compressed_oracle."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import fp8_e4m3 as F
from oracle import indexer as O
from sparse_attention_token_02_b200 import api
from sparse_attention_token_02_b200 import workloads as W

from ._parity import RTOL, bits_to_bf16_tensor, check_row

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    api.dsa_version()
    yield
    api.dsa_check_device_errors()


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("m", [4, 7])
def test_compressed_decode_against_oracle(dtype, m):
    lens, q_lens, H, d, k = (9001, 4096, 130, 3, 2000), (2, 1, 2, 1, 2), 64, 128, 256
    fp8 = dtype == "fp8"
    blocks = [L // m for L in lens]
    rng = np.random.default_rng(80 + m)
    # compressed keys (the learned merge is the caller's): synthetic N(0, 1), one row per block,
    # stored with a gap of 5 rows between sequences
    k_bits = [W.f32_to_bf16_bits(rng.standard_normal((nb, d)).astype(np.float32)) for nb in blocks]
    k_base = np.cumsum([0] + [nb + 5 for nb in blocks[:-1]]).astype(np.int64)
    cache = api.IndexerKCache.empty(int(k_base[-1] + blocks[-1] + 5), d, fp8)
    for b, nb in enumerate(blocks):
        if nb:
            api.dsa_indexer_kcache_append(cache, bits_to_bf16_tensor(k_bits[b], "cuda"),
                                          torch.arange(k_base[b], k_base[b] + nb, dtype=torch.int64, device="cuda"))
    T = sum(q_lens)
    q_bits = W.f32_to_bf16_bits((rng.standard_normal((T, H, d)) / np.sqrt(d)).astype(np.float32))
    w = W.softmax_rows(rng.standard_normal((T, H)).astype(np.float32))
    q_src = bits_to_bf16_tensor(q_bits, "cuda")
    if fp8:
        codes, scale = api.dsa_quantize_rows_fp8(q_src.reshape(T, -1))
        q, q_scale = codes.reshape(T, H, d), scale
    else:
        q, q_scale = q_src, None
    idx, sc = api.dsa_indexer_decode_compressed(q, cache, torch.from_numpy(w).cuda(), lens, q_lens, m, k,
                                                q_scale=q_scale, k_base=k_base)
    api.dsa_check_device_errors()
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    # exact values the GPU scored: bf16 as given, FP8 as code * scale (the library's own codec
    # equals the oracle's, checked in test_gpu_indexer.py)
    if fp8:
        kv = []
        for bits in k_bits:
            c, s = F.quantize_rows(F.bf16_bits_to_f64(bits).astype(np.float32))
            kv.append(F.e4m3_decode(c) * s[:, None].astype(np.float64))
        c, s = F.quantize_rows(F.bf16_bits_to_f64(q_bits.reshape(T, -1)).astype(np.float32))
        qv = (F.e4m3_decode(c) * s[:, None].astype(np.float64)).reshape(T, H, d)
    else:
        kv = [F.bf16_bits_to_f64(bits) for bits in k_bits]
        qv = F.bf16_bits_to_f64(q_bits.reshape(T * H, d)).reshape(T, H, d)
    ref = O.decode_compressed_oracle(qv, kv, w.astype(np.float64), lens, q_lens, m, k)
    seq = np.repeat(np.arange(len(lens)), q_lens)
    for r in range(T):
        nv = int(ref["visible"][r])
        if nv == 0:
            assert (idx[r] == -1).all() and np.isneginf(sc[r]).all()
            continue
        orow = O.row_scores(qv[r], kv[int(seq[r])][:nv], w[r].astype(np.float64))
        check_row(idx[r], sc[r], orow, k, RTOL[dtype], what=f"compressed row {r}")


def test_compressed_decode_m_1_equals_decode():
    wl = W.scaled(W.decode(), seq_lens=(3000, 700), q_lens=(2, 1), top_k=300, seed=81)
    from ._parity import Uploaded
    up = Uploaded(wl)
    a_i, a_s = api.dsa_indexer_decode(up.q, up.cache, up.w, wl.seq_lens, wl.q_lens, wl.top_k, k_base=up.k_base)
    b_i, b_s = api.dsa_indexer_decode_compressed(up.q, up.cache, up.w, wl.seq_lens, wl.q_lens, 1, wl.top_k,
                                                 k_base=up.k_base)
    # the plain decode scores two queries per accumulator, this path one: equal up to rounding
    a_i, a_s, b_i, b_s = (t.cpu().numpy() for t in (a_i, a_s, b_i, b_s))
    for r in range(wl.total_q):
        a = dict(zip(a_i[r].tolist(), a_s[r].tolist()))
        b = dict(zip(b_i[r].tolist(), b_s[r].tolist()))
        kth = min(a.values())
        for i in a.keys() & b.keys():
            assert abs(a[i] - b[i]) <= 1e-6 * max(abs(a[i]), 1e-30)
        for i in a.keys() ^ b.keys():
            assert abs(a.get(i, b.get(i)) - kth) <= 1e-6 * max(abs(kth), 1e-30)
    from ._parity import check_rows
    check_rows(up, b_i, b_s, range(wl.total_q))


@pytest.mark.parametrize("dtype,H,d,m", [("bf16", 64, 128, 4), ("fp8", 64, 128, 7), ("bf16", 4, 64, 3)])
def test_compressed_prefill_against_oracle(dtype, H, d, m):
    # every token of each sequence is a query (q_len = seq_len); rows short of top_k blocks
    # (early positions, including ones that see no block) and rows longer than it
    lens, k = (1500, 333, 900), 64
    fp8 = dtype == "fp8"
    blocks = [L // m for L in lens]
    rng = np.random.default_rng(90 + m)
    k_bits = [W.f32_to_bf16_bits(rng.standard_normal((nb, d)).astype(np.float32)) for nb in blocks]
    k_base = np.cumsum([0] + [nb + 3 for nb in blocks[:-1]]).astype(np.int64)
    cache = api.IndexerKCache.empty(int(k_base[-1] + blocks[-1] + 3), d, fp8)
    for b, nb in enumerate(blocks):
        api.dsa_indexer_kcache_append(cache, bits_to_bf16_tensor(k_bits[b], "cuda"),
                                      torch.arange(k_base[b], k_base[b] + nb, dtype=torch.int64, device="cuda"))
    T = sum(lens)
    q_bits = W.f32_to_bf16_bits((rng.standard_normal((T, H, d)) / np.sqrt(d)).astype(np.float32))
    w = W.softmax_rows(rng.standard_normal((T, H)).astype(np.float32))
    q_src = bits_to_bf16_tensor(q_bits, "cuda")
    if fp8:
        codes, scale = api.dsa_quantize_rows_fp8(q_src.reshape(T, -1))
        q, q_scale = codes.reshape(T, H, d), scale
    else:
        q, q_scale = q_src, None
    idx, sc = api.dsa_indexer_prefill_compressed(q, cache, torch.from_numpy(w).cuda(), lens, m, k, q_scale=q_scale,
                                                 k_base=k_base)
    api.dsa_check_device_errors()
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    if fp8:
        kv = []
        for bits in k_bits:
            c, s = F.quantize_rows(F.bf16_bits_to_f64(bits).astype(np.float32))
            kv.append(F.e4m3_decode(c) * s[:, None].astype(np.float64))
        c, s = F.quantize_rows(F.bf16_bits_to_f64(q_bits.reshape(T, -1)).astype(np.float32))
        qv = (F.e4m3_decode(c) * s[:, None].astype(np.float64)).reshape(T, H, d)
    else:
        kv = [F.bf16_bits_to_f64(bits) for bits in k_bits]
        qv = F.bf16_bits_to_f64(q_bits.reshape(T * H, d)).reshape(T, H, d)
    seq = np.repeat(np.arange(len(lens)), lens)
    pos = np.concatenate([np.arange(L) for L in lens])
    rows = np.unique(np.concatenate([np.arange(0, T, 5), [0, m - 2, m - 1, T - 1]]))   # a sample of rows
    for r in rows:
        nv = O.compressed_visible(int(pos[r]), m)
        if nv == 0:
            assert (idx[r] == -1).all() and np.isneginf(sc[r]).all()
            continue
        orow = O.row_scores(qv[r], kv[int(seq[r])][:nv], w[r].astype(np.float64))
        check_row(idx[r], sc[r], orow, k, RTOL[dtype], what=f"compressed prefill row {r}")


def test_compressed_prefill_m_1_equals_prefill():
    wl = W.scaled(W.prefill(), seq_lens=(700, 1300), q_lens=(700, 1300), top_k=256, seed=91)
    from ._parity import Uploaded
    up = Uploaded(wl)
    a_i, a_s = api.dsa_indexer_prefill(up.q, up.cache, up.w, wl.seq_lens, wl.top_k, k_base=up.k_base)
    b_i, b_s = api.dsa_indexer_prefill_compressed(up.q, up.cache, up.w, wl.seq_lens, 1, wl.top_k, k_base=up.k_base)
    # m = 1 is the same launch sequence: the same scores, and the same selections up to exact
    # ties at the k-th score (which of those are kept is unspecified); both match the oracle
    a_i, a_s, b_i, b_s = (t.cpu().numpy() for t in (a_i, a_s, b_i, b_s))
    from ._parity import check_rows
    rows = list(range(0, wl.total_q, 5)) + [wl.total_q - 1]
    check_rows(up, b_i, b_s, rows)
    for r in range(wl.total_q):
        a = dict(zip(a_i[r].tolist(), a_s[r].tolist()))
        b = dict(zip(b_i[r].tolist(), b_s[r].tolist()))
        kth = min(a.values())
        for i in a.keys() & b.keys():
            assert a[i] == b[i], f"row {r} index {i}"
        for i in a.keys() ^ b.keys():
            assert a.get(i, b.get(i)) == kth, f"row {r}: index {i} selected by one call only, not an exact tie"
