"""GPU parity of the CUDA path (through the C ABI) against the fp64 CPU oracle.

Every case runs the library on seeded inputs and compares with the oracle fed the
same bits (bf16 inputs decoded exactly; FP8 codes produced by the oracle's own
codec, checked byte for byte against the library's append / quantise kernels).
Small cases compare every row; the full-size workloads compare sampled rows,
always including the first rows, the rows around the top_k boundary and the last.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_token_02_b200 import api
from sparse_attention_token_02_b200 import workloads as W

from ._parity import (RTOL, OracleInputs, Uploaded, bits_to_bf16_tensor, check_row, check_rows, run_indexer,
                      sample_rows)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    api.dsa_version()          # the CUDA library must load
    yield
    api.dsa_check_device_errors()


_run = run_indexer
_sample_rows = sample_rows
_check = check_rows


# ----------------------------------------------------------------------------- append / quantise (a1)

def test_append_bf16_copy_and_f32_rounding():
    rng = np.random.default_rng(0)
    src32 = (rng.standard_normal((300, 128)) * 3).astype(np.float32)
    cache = api.IndexerKCache.empty(1000, 128, fp8=False)
    rows = torch.from_numpy(rng.permutation(1000)[:300].astype(np.int64)).cuda()
    api.dsa_indexer_kcache_append(cache, torch.from_numpy(src32).cuda(), rows)
    got = cache.k[rows].cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, W.f32_to_bf16_bits(src32))
    bits = W.f32_to_bf16_bits(src32[::-1].copy())
    api.dsa_indexer_kcache_append(cache, bits_to_bf16_tensor(bits), rows)
    got = cache.k[rows].cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, bits)
    api.dsa_check_device_errors()


# 128: a key row (one warp each); 1040, 8192, 9008: one CTA per row with 1, 4 and 8 chunks of 8 values
# per thread, the first and last ragged; 16400: past the CTA kernel's register capacity (warp loop)
@pytest.mark.parametrize("row_len", [128, 1040, 8192, 9008, 16400])
def test_quantize_rows_fp8_bit_exact_against_oracle_codec(row_len):
    rng = np.random.default_rng(row_len)
    x = (rng.standard_normal((257, row_len)) * rng.uniform(1e-3, 50, (257, 1))).astype(np.float32)
    x[3] = 0.0
    x[4, :7] = [1e-8, -1e-8, 3e4, -3e4, 0.0, 1.0, -1.0]
    bits = W.f32_to_bf16_bits(x)
    codes, scale = api.dsa_quantize_rows_fp8(bits_to_bf16_tensor(bits))
    ref_codes, ref_scale = oracle.quantize_rows(oracle.bf16_bits_to_f64(bits).astype(np.float32))
    assert np.array_equal(scale.cpu().numpy(), ref_scale)
    assert np.array_equal(codes.cpu().numpy(), ref_codes)
    # fp32 sources too
    codes, scale = api.dsa_quantize_rows_fp8(torch.from_numpy(x).cuda())
    ref_codes, ref_scale = oracle.quantize_rows(x)
    assert np.array_equal(scale.cpu().numpy(), ref_scale)
    assert np.array_equal(codes.cpu().numpy(), ref_codes)


def test_fp8_cache_append_matches_oracle_codec():
    wl = W.scaled(W.decode8(), seq_lens=(700, 333), q_lens=(2, 2))
    up = Uploaded(wl)
    for b in range(2):
        lo = int(up.k_base[b])
        codes, scale = oracle.quantize_rows(oracle.bf16_bits_to_f64(up.inp["k_bits"][b]).astype(np.float32))
        got = up.cache.k[lo: lo + wl.seq_lens[b]].cpu().numpy()
        gs = up.cache.k_scale[lo: lo + wl.seq_lens[b]].cpu().numpy()
        assert np.array_equal(got, codes) and np.array_equal(gs, scale)


def test_append_out_of_range_row_is_reported_and_skipped():
    cache = api.IndexerKCache.empty(16, 128, fp8=True)
    src = torch.ones(2, 128, dtype=torch.bfloat16, device="cuda")
    api.dsa_indexer_kcache_append(cache, src, torch.tensor([3, 16], dtype=torch.int64, device="cuda"))
    with pytest.raises(RuntimeError, match="DEVICE_CHECK"):
        api.dsa_check_device_errors()
    assert int(cache.k[3, 0]) != 0          # the valid row was written
    api.dsa_check_device_errors()           # the flag was cleared


def test_bounded_wait_expiry_is_reported_and_the_stream_stays_usable():
    # the library's bounded wait, on a barrier that nothing completes, with a ~1 ms limit
    api.dsa_selftest_wait_expiry(2_000_000)
    with pytest.raises(RuntimeError, match="DEVICE_CHECK.*bounded wait expired"):
        api.dsa_check_device_errors()
    api.dsa_check_device_errors()           # the flag was cleared
    x = torch.arange(1024, dtype=torch.float32, device="cuda")
    assert float(x.sum()) == 1023 * 1024 / 2


# ----------------------------------------------------------------------------- prefill

def test_tiny_workload_all_rows_and_dense_scores():
    wl = W.tiny()
    up = Uploaded(wl)
    idx, sc = _run(up)
    rows = list(range(wl.total_q))
    _check(up, idx, sc, rows)
    dense = api.dsa_indexer_scores(up.q, up.cache, up.w, wl.seq_lens, k_base=up.k_base).cpu().numpy()
    for r, orow in zip(rows, up.oracle_rows(rows)):
        p = orow.shape[0]
        o_k = np.sort(orow)[::-1][min(wl.top_k, p) - 1]
        tol = RTOL["bf16"] * np.maximum(np.abs(orow), max(abs(o_k), 1e-30))
        assert np.all(np.abs(dense[r, :p] - orow) <= tol), f"row {r}"
        assert np.all(np.isneginf(dense[r, p:]))


def test_prefill_bf16_ragged_batch_chunked_and_offset_cache():
    # three sequences: a full prefill, a chunked prefill (q_len < seq_len) and a single query;
    # the cache rows of the sequences are not packed (k_base with gaps)
    wl = W.scaled(W.prefill(), seq_lens=(700, 450, 129), q_lens=(700, 200, 1), top_k=256, outlier_frac=0.01)
    inp = W.make_inputs(wl)
    up = Uploaded(wl, inp)
    base = np.array([5000, 37, 2000], dtype=np.int64)
    cache = api.IndexerKCache.empty(6000, 128, fp8=False)
    for b in range(3):
        rows = torch.arange(base[b], base[b] + wl.seq_lens[b], dtype=torch.int64, device="cuda")
        api.dsa_indexer_kcache_append(cache, bits_to_bf16_tensor(inp["k_bits"][b]), rows)
    idx, sc = api.dsa_indexer_prefill(up.q, cache, up.w, wl.seq_lens, wl.top_k, q_lens=wl.q_lens, k_base=base)
    api.dsa_check_device_errors()
    _check(up, idx.cpu().numpy(), sc.cpu().numpy(), list(range(wl.total_q)))


def test_prefill_bf16_top_k_2048_boundary_rows():
    wl = W.scaled(W.prefill(), seq_lens=(2600,), q_lens=(2600,))
    up = Uploaded(wl)
    idx, sc = _run(up)
    rows = _sample_rows(wl, n_mid=10) + list(range(2040, 2060))
    _check(up, idx, sc, sorted(set(rows)))


def test_prefill_fp8_small():
    wl = W.scaled(W.prefill8(), seq_lens=(2300, 517), q_lens=(2300, 517))
    up = Uploaded(wl)
    idx, sc = _run(up)
    _check(up, idx, sc, _sample_rows(wl, n_mid=12) + list(range(2300, 2310)))


# ----------------------------------------------------------------------------- decode

@pytest.mark.parametrize("q_len", [1, 2, 3])
def test_decode_bf16_ragged(q_len):
    lens = (5000, 130, 2049, q_len, 4096, 33, 2051)
    wl = W.scaled(W.decode(), seq_lens=lens, q_lens=(q_len,) * len(lens), seed=10 + q_len)
    up = Uploaded(wl)
    idx, sc = _run(up, decode=True)
    _check(up, idx, sc, list(range(wl.total_q)))


@pytest.mark.parametrize("q_len", [1, 2, 3])
def test_decode_fp8_ragged(q_len):
    wl = W.scaled(W.decode8(), seq_lens=(9000, 2049, 4097, 3000, 3), q_lens=(q_len,) * 5, seed=20 + q_len)
    up = Uploaded(wl)
    idx, sc = _run(up, decode=True)
    _check(up, idx, sc, list(range(wl.total_q)))


def _same_set_up_to_exact_ties(idx_a, sc_a, idx_b, sc_b, what):
    """Two selections of one row: the same scores (within 1e-6) for the indices both hold,
    and indices held by one only must score exactly the k-th score of both (a tie at the
    boundary, where the header leaves the choice open)."""
    va, vb = idx_a >= 0, idx_b >= 0
    assert va.sum() == vb.sum(), f"{what}: valid counts differ"
    a = dict(zip(idx_a[va].tolist(), sc_a[va].tolist()))
    b = dict(zip(idx_b[vb].tolist(), sc_b[vb].tolist()))
    for i in a.keys() & b.keys():
        assert abs(a[i] - b[i]) <= 1e-6 * abs(a[i]), f"{what}: index {i} scores {a[i]} vs {b[i]}"
    only = a.keys() ^ b.keys()
    if only:
        kth_a, kth_b = min(a.values()), min(b.values())
        for i in only:
            s = a[i] if i in a else b[i]
            assert s == kth_a == kth_b, f"{what}: index {i} selected by one call only and not tied at the k-th score"


def test_decode_row_equals_prefill_row():
    # the invariant of the pages' two modes: a decode step's query at position p selects what
    # the prefill's row p selects (each call is also checked against the oracle)
    wl = W.scaled(W.prefill(), seq_lens=(3000,), q_lens=(3000,), outlier_frac=0.0)
    up = Uploaded(wl)
    pidx, psc = _run(up)
    last = slice(2998, 3000)
    q_dec = up.q[last].contiguous()
    w_dec = up.w[last].contiguous()
    didx, dsc = api.dsa_indexer_decode(q_dec, up.cache, w_dec, (3000,), (2,), wl.top_k, k_base=up.k_base)
    api.dsa_check_device_errors()
    didx, dsc = didx.cpu().numpy(), dsc.cpu().numpy()
    orows = up.oracle_rows([2998, 2999])
    for j, r in enumerate((2998, 2999)):
        check_row(pidx[r], psc[r], orows[j], wl.top_k, RTOL["bf16"], what=f"prefill row {r}")
        check_row(didx[j], dsc[j], orows[j], wl.top_k, RTOL["bf16"], what=f"decode row {r}")
        _same_set_up_to_exact_ties(pidx[r], psc[r], didx[j], dsc[j], f"row {r}")


# ----------------------------------------------------------------------------- edge cases

def test_edge_top_k_larger_than_every_row_and_top_k_one():
    wl = W.scaled(W.prefill(), seq_lens=(300, 1), q_lens=(300, 1), top_k=512)
    up = Uploaded(wl)
    idx, sc = _run(up)
    _check(up, idx, sc, list(range(wl.total_q)))
    idx1, sc1 = _run(up, top_k=1)
    _check(up, idx1, sc1, list(range(wl.total_q)), top_k=1)


@pytest.mark.parametrize("decode", [False, True])
def test_short_sequence_bypass_writes_the_history_and_scores_nothing(decode):
    # every sequence within top_k: no scoring kernel, out_idx = 0 .. n_r - 1 then -1
    L, q_lens = (300, 7, 512), ((2, 1, 3) if decode else (300, 7, 512))
    wl = W.scaled(W.decode() if decode else W.prefill(), seq_lens=L, q_lens=q_lens, top_k=512)
    up = Uploaded(wl)
    run = api.dsa_indexer_decode if decode else api.dsa_indexer_prefill
    kw = dict(q_lens=q_lens) if not decode else {}
    before = api.dsa_kernel_launch_count()
    if decode:
        idx, sc = run(up.q, up.cache, up.w, L, q_lens, wl.top_k, q_scale=up.q_scale, k_base=up.k_base, scores=False)
    else:
        idx, sc = run(up.q, up.cache, up.w, L, wl.top_k, q_scale=up.q_scale, k_base=up.k_base, scores=False, **kw)
    api.dsa_check_device_errors()
    assert sc is None and api.dsa_kernel_launch_count() - before == 1
    idx = idx.cpu().numpy()
    r = 0
    for Lb, n in zip(L, q_lens):
        for j in range(n):
            hist = Lb - n + j + 1                             # the query's causal history
            want = np.where(np.arange(wl.top_k) < hist, np.arange(wl.top_k), -1)
            assert np.array_equal(idx[r], want), r
            r += 1
    # the same selection as the scored call, whose set is the whole history too
    ref_i, _ = (run(up.q, up.cache, up.w, L, q_lens, wl.top_k, q_scale=up.q_scale, k_base=up.k_base) if decode else
                run(up.q, up.cache, up.w, L, wl.top_k, q_scale=up.q_scale, k_base=up.k_base, **kw))
    assert np.array_equal(np.sort(ref_i.cpu().numpy(), axis=1), np.sort(idx, axis=1))
    with pytest.raises(RuntimeError, match="INVALID_ARG"):
        run(up.q, up.cache, up.w, L, q_lens, 16, q_scale=up.q_scale, k_base=up.k_base, scores=False) if decode else \
            run(up.q, up.cache, up.w, L, 16, q_scale=up.q_scale, k_base=up.k_base, scores=False, **kw)


@pytest.mark.parametrize("decode", [False, True])
def test_caller_workspace_matches_the_oracle_and_refuses_a_short_one(decode):
    L, q_lens = (3000, 2049, 700), ((2, 1, 1) if decode else (3000, 2049, 700))
    wl = W.scaled(W.decode() if decode else W.prefill(), seq_lens=L, q_lens=q_lens, top_k=512, seed=95)
    up = Uploaded(wl)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        ref_i, ref_s = _run(up, decode=decode)
        need = api.dsa_indexer_workspace_bytes(up.q, L, wl.top_k, q_lens=q_lens)
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        try:
            api.dsa_set_workspace(ws, stream=s)
            if decode:
                idx, sc = api.dsa_indexer_decode(up.q, up.cache, up.w, L, q_lens, wl.top_k, q_scale=up.q_scale,
                                                 k_base=up.k_base, stream=s)
            else:
                idx, sc = api.dsa_indexer_prefill(up.q, up.cache, up.w, L, wl.top_k, q_scale=up.q_scale, q_lens=q_lens,
                                                  k_base=up.k_base, stream=s)
            api.dsa_check_device_errors(s)
            # both calls against the oracle (which keys are kept among exact ties at the k-th
            # score is unspecified, so the two calls are not compared with each other)
            rows = list(range(wl.total_q))
            _check(up, ref_i, ref_s, rows)
            _check(up, idx.cpu().numpy(), sc.cpu().numpy(), rows)
            api.dsa_set_workspace(ws[: 1 << 12], stream=s)       # far too small
            with pytest.raises(RuntimeError, match="ALLOC"):
                api.dsa_indexer_decode(up.q, up.cache, up.w, L, q_lens, wl.top_k, q_scale=up.q_scale,
                                       k_base=up.k_base, stream=s) if decode else \
                    api.dsa_indexer_prefill(up.q, up.cache, up.w, L, wl.top_k, q_scale=up.q_scale, q_lens=q_lens,
                                            k_base=up.k_base, stream=s)
        finally:
            api.dsa_set_workspace(None, stream=s)
        s.synchronize()


def test_edge_ties_and_zero_and_negative_weights():
    wl = W.scaled(W.prefill(), seq_lens=(1500,), q_lens=(1500,), top_k=100)
    inp = W.make_inputs(wl)
    # integer-valued keys and queries: many exactly equal scores
    rng = np.random.default_rng(1)
    inp["k_bits"] = [W.f32_to_bf16_bits(rng.integers(-2, 3, (1500, 128)).astype(np.float32))]
    inp["q_bits"] = W.f32_to_bf16_bits(rng.integers(-1, 2, (1500, 64, 128)).astype(np.float32))
    for w in (np.full((1500, 64), 1.0 / 64, np.float32),
              np.zeros((1500, 64), np.float32),
              rng.standard_normal((1500, 64)).astype(np.float32)):
        inp["w"] = w
        up = Uploaded(wl, inp)
        idx, sc = _run(up)
        _check(up, idx, sc, [0, 1, 99, 100, 101, 500, 1499])


def test_edge_prefill_ties_in_rows_longer_than_the_gather_buffer():
    # rows of up to 9000 keys with few distinct scores: the threshold bin holds more keys
    # than one CTA gathers, so the row top-k refines it, or (zero weights: one tied value)
    # writes the tied keys directly
    L = 9000
    wl = W.scaled(W.prefill(), seq_lens=(L,), q_lens=(L,), outlier_frac=0.0, seed=43)
    inp = W.make_inputs(wl)
    rng = np.random.default_rng(3)
    inp["k_bits"] = [W.f32_to_bf16_bits(rng.integers(-2, 3, (L, 128)).astype(np.float32))]
    inp["q_bits"] = W.f32_to_bf16_bits(rng.integers(-1, 2, (L, 64, 128)).astype(np.float32))
    rows = [0, 2047, 2048, 4095, 4096, 4097, 6000, L - 1]
    for w in (np.full((L, 64), 1.0 / 64, np.float32), np.zeros((L, 64), np.float32)):
        inp["w"] = w
        up = Uploaded(wl, inp)
        idx, sc = _run(up)
        _check(up, idx, sc, rows)


def test_edge_decode_ties_zero_and_negative_weights():
    # decode rows over several chunks of the streaming top-k; with zero weights every
    # score is 0, so the threshold bin holds the whole row and the choice is all ties
    lens = (9000, 4100, 2049, 8193)
    wl = W.scaled(W.decode(), seq_lens=lens, q_lens=(2,) * len(lens), top_k=300, seed=41)
    inp = W.make_inputs(wl)
    rng = np.random.default_rng(2)
    inp["k_bits"] = [W.f32_to_bf16_bits(rng.integers(-2, 3, (L, 128)).astype(np.float32)) for L in lens]
    inp["q_bits"] = W.f32_to_bf16_bits(rng.integers(-1, 2, (wl.total_q, 64, 128)).astype(np.float32))
    T = wl.total_q
    for w in (np.full((T, 64), 1.0 / 64, np.float32), np.zeros((T, 64), np.float32),
              rng.standard_normal((T, 64)).astype(np.float32)):
        inp["w"] = w
        up = Uploaded(wl, inp)
        idx, sc = _run(up, decode=True)
        _check(up, idx, sc, list(range(T)))


def test_edge_decode_row_longer_than_one_cluster_holds():
    # 150000 keys: beyond what a cluster of 8 CTAs keeps in registers; decode streams it
    wl = W.scaled(W.decode(), seq_lens=(150000, 5000), q_lens=(1, 1), seed=42)
    up = Uploaded(wl)
    idx, sc = _run(up, decode=True)
    _check(up, idx, sc, [0, 1])


def test_edge_empty_batch_and_zero_query_sequences():
    wl = W.scaled(W.prefill(), seq_lens=(40, 10), q_lens=(0, 10), top_k=16)
    up = Uploaded(wl)
    idx, sc = _run(up)
    _check(up, idx, sc, list(range(10)))
    q = torch.zeros(0, 64, 128, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(0, 64, dtype=torch.float32, device="cuda")
    i0, s0 = api.dsa_indexer_prefill(q, up.cache, w, [], 16)
    assert i0.shape == (0, 16)


def test_edge_invalid_arguments_raise():
    up = Uploaded(W.scaled(W.decode(), seq_lens=(300,), q_lens=(1,)))
    with pytest.raises(RuntimeError, match="INVALID_ARG"):
        api.dsa_indexer_decode(up.q, up.cache, up.w, (300,), (5,), 16)       # q_len > 4
    with pytest.raises(RuntimeError, match="INVALID_ARG"):
        api.dsa_indexer_prefill(up.q, up.cache, up.w, (300,), 0, q_lens=(1,))  # top_k = 0
    with pytest.raises(RuntimeError, match="INVALID_ARG"):
        api.dsa_indexer_prefill(up.q, up.cache, up.w, (10 ** 6,), 16, q_lens=(1,))  # beyond capacity
    q32 = torch.zeros(1, 32, 128, dtype=torch.bfloat16, device="cuda")
    w32 = torch.zeros(1, 32, dtype=torch.float32, device="cuda")
    with pytest.raises(RuntimeError, match="UNSUPPORTED"):
        api.dsa_indexer_prefill(q32, up.cache, w32, (300,), 16, q_lens=(1,))


# ----------------------------------------------------------------------------- one-call host step

@pytest.mark.parametrize("name", ["bf16", "fp8"])
def test_decode_host_step_matches_the_oracle_two_calls_in_a_row(name):
    base = W.decode() if name == "bf16" else W.decode8()
    lens = [(6000, 2100, 300, 4097), (5000, 2049, 3333, 1)]
    for call, L in enumerate(lens):
        q_lens = (1, 2, 1, 1)
        wl = W.scaled(base, seq_lens=L, q_lens=q_lens, seed=50 + call)
        up = Uploaded(wl)
        # the step re-appends each sequence's newest q_len keys (same values: the cache is unchanged)
        rows = np.concatenate([up.k_base[b] + np.arange(Lb - n, Lb) for b, (Lb, n) in enumerate(zip(L, q_lens))])
        k_bits = np.concatenate(up.inp["k_bits"])[rows]
        k_h = torch.from_numpy(np.ascontiguousarray(k_bits).view(np.int16)).view(torch.bfloat16).pin_memory()
        q_h = torch.from_numpy(np.ascontiguousarray(up.inp["q_bits"]).view(np.int16)).view(torch.bfloat16).pin_memory()
        w_h = torch.from_numpy(up.inp["w"]).pin_memory()
        rows_h = torch.from_numpy(rows.astype(np.int64)).pin_memory()
        oi_h = torch.full((wl.total_q, wl.top_k), 7, dtype=torch.int32).pin_memory()
        os_h = torch.zeros((wl.total_q, wl.top_k), dtype=torch.float32).pin_memory()
        s = torch.cuda.current_stream()
        api.dsa_indexer_decode_host(q_h, w_h, k_h, rows_h, up.cache, L, q_lens, wl.top_k, oi_h, os_h,
                                    k_base=up.k_base, stream=s)
        api.dsa_check_device_errors(s)                       # synchronises the stream
        _check(up, oi_h.numpy(), os_h.numpy(), range(wl.total_q))


@pytest.mark.parametrize("name", ["bf16", "fp8"])
def test_decode_host_step_async_three_calls_in_flight(name):
    # three steps with different inputs and outputs enqueued without waiting (the third reuses
    # the first one's slot), each read back under its own completion event
    base = W.decode() if name == "bf16" else W.decode8()
    L, q_lens = (4100, 700, 2049), (2, 1, 1)
    wl = W.scaled(base, seq_lens=L, q_lens=q_lens, seed=90)
    up = Uploaded(wl)
    rows = np.concatenate([up.k_base[b] + np.arange(Lb - n, Lb) for b, (Lb, n) in enumerate(zip(L, q_lens))])
    k_bits = np.concatenate(up.inp["k_bits"])[rows]
    k_h = torch.from_numpy(np.ascontiguousarray(k_bits).view(np.int16)).view(torch.bfloat16).pin_memory()
    rows_h = torch.from_numpy(rows.astype(np.int64)).pin_memory()
    s = torch.cuda.Stream()
    steps = []
    for call in range(3):
        rng = np.random.default_rng(200 + call)
        q_bits = W.f32_to_bf16_bits((rng.standard_normal(up.inp["q_bits"].shape) / 11.3).astype(np.float32))
        w = W.softmax_rows(rng.standard_normal(up.inp["w"].shape).astype(np.float32))
        q_h = torch.from_numpy(np.ascontiguousarray(q_bits).view(np.int16)).view(torch.bfloat16).pin_memory()
        w_h = torch.from_numpy(w).pin_memory()
        oi_h = torch.full((wl.total_q, wl.top_k), 7, dtype=torch.int32).pin_memory()
        os_h = torch.zeros((wl.total_q, wl.top_k), dtype=torch.float32).pin_memory()
        ev = torch.cuda.Event()
        api.dsa_indexer_decode_host(q_h, w_h, k_h, rows_h, up.cache, L, q_lens, wl.top_k, oi_h, os_h,
                                    k_base=up.k_base, stream=s, done_event=ev)
        steps.append((q_bits, w, oi_h, os_h, ev))
    for q_bits, w, oi_h, os_h, ev in steps:
        ev.synchronize()
        # the oracle on this step's inputs (an FP8 cache: the queries through the oracle's codec,
        # which the host step's device quantisation matches bit for bit)
        ref = OracleInputs(wl, dict(up.inp, q_bits=q_bits, w=w))
        _check(ref, oi_h.numpy(), os_h.numpy(), range(wl.total_q))
    api.dsa_check_device_errors(s)


@pytest.mark.parametrize("name", ["bf16", "fp8"])
def test_prefill_host_step_matches_the_oracle_two_calls_and_three_in_flight(name):
    # whole prefills from host memory: the keys appended (quantised for an FP8 cache), bf16
    # queries uploaded (quantised on the device for an FP8 cache), the selection read back
    base = W.prefill() if name == "bf16" else W.prefill8()
    lens = (3000, 700)
    wl = W.scaled(base, seq_lens=lens, q_lens=lens, seed=120)
    up = Uploaded(wl)
    k_h = torch.from_numpy(np.ascontiguousarray(np.concatenate(up.inp["k_bits"])).view(np.int16)).view(
        torch.bfloat16).pin_memory()
    rows_h = torch.arange(wl.total_k, dtype=torch.int64).pin_memory()
    rows = list(range(0, wl.total_q, 37)) + [2047, 2048, 2999, 3000, wl.total_q - 1]
    # two synchronous calls in a row
    for call in range(2):
        q_h = torch.from_numpy(np.ascontiguousarray(up.inp["q_bits"]).view(np.int16)).view(torch.bfloat16).pin_memory()
        w_h = torch.from_numpy(up.inp["w"]).pin_memory()
        oi_h = torch.full((wl.total_q, wl.top_k), 7, dtype=torch.int32).pin_memory()
        os_h = torch.zeros((wl.total_q, wl.top_k), dtype=torch.float32).pin_memory()
        s = torch.cuda.current_stream()
        api.dsa_indexer_prefill_host(q_h, w_h, k_h, rows_h, up.cache, lens, wl.top_k, oi_h, os_h, k_base=up.k_base,
                                     stream=s)
        api.dsa_check_device_errors(s)
        _check(up, oi_h.numpy(), os_h.numpy(), rows)
    # three steps with different queries and weights in flight, each read back under its own event
    s = torch.cuda.Stream()
    steps = []
    for call in range(3):
        rng = np.random.default_rng(300 + call)
        q_bits = W.f32_to_bf16_bits(rng.standard_normal(up.inp["q_bits"].shape).astype(np.float32))
        w = W.softmax_rows(rng.standard_normal(up.inp["w"].shape).astype(np.float32))
        q_h = torch.from_numpy(np.ascontiguousarray(q_bits).view(np.int16)).view(torch.bfloat16).pin_memory()
        w_h = torch.from_numpy(w).pin_memory()
        oi_h = torch.full((wl.total_q, wl.top_k), 7, dtype=torch.int32).pin_memory()
        os_h = torch.zeros((wl.total_q, wl.top_k), dtype=torch.float32).pin_memory()
        ev = torch.cuda.Event()
        api.dsa_indexer_prefill_host(q_h, w_h, k_h, rows_h, up.cache, lens, wl.top_k, oi_h, os_h, k_base=up.k_base,
                                     stream=s, done_event=ev)
        steps.append((q_bits, w, q_h, w_h, oi_h, os_h, ev))
    for q_bits, w, q_h, w_h, oi_h, os_h, ev in steps:
        ev.synchronize()
        ref = OracleInputs(wl, dict(up.inp, q_bits=q_bits, w=w))
        _check(ref, oi_h.numpy(), os_h.numpy(), rows)
    api.dsa_check_device_errors(s)


def test_decode_host_step_rejects_bad_arguments():
    wl = W.scaled(W.decode(), seq_lens=(300,), q_lens=(1,))
    up = Uploaded(wl)
    q_h = torch.zeros(1, 64, 128, dtype=torch.bfloat16)
    w_h = torch.zeros(1, 64, dtype=torch.float32)
    oi_h = torch.zeros(1, 16, dtype=torch.int32)
    os_h = torch.zeros(1, 16, dtype=torch.float32)
    with pytest.raises(ValueError, match="host tensors"):
        api.dsa_indexer_decode_host(q_h.cuda(), w_h, None, torch.zeros(0, dtype=torch.int64), up.cache, (300,), (1,),
                                    16, oi_h, os_h)
    with pytest.raises(RuntimeError, match="INVALID_ARG"):
        api.dsa_indexer_decode_host(q_h, w_h, None, torch.zeros(0, dtype=torch.int64), up.cache, (300,), (1,),
                                    0, oi_h, os_h)


# ----------------------------------------------------------------------------- CUDA graphs

def test_graph_capture_replay_matches_the_oracle_and_unplanned_capture_is_refused():
    wl = W.scaled(W.decode(), seq_lens=(3000, 2500, 40), q_lens=(1, 1, 1), seed=31)
    up = Uploaded(wl)
    s = torch.cuda.Stream()
    out_i = torch.empty(3, wl.top_k, dtype=torch.int32, device="cuda")
    out_s = torch.empty(3, wl.top_k, dtype=torch.float32, device="cuda")
    run = lambda: api.dsa_indexer_decode(up.q, up.cache, up.w, wl.seq_lens, wl.q_lens, wl.top_k, k_base=up.k_base,
                                         out_idx=out_i, out_score=out_s, stream=s)
    with torch.cuda.stream(s):
        run()
    s.synchronize()
    eager_i, eager_s = out_i.clone(), out_s.clone()
    out_i.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s, capture_error_mode="relaxed"):
        run()
        # a batch this stream has not run uncaptured cannot be planned during capture
        with pytest.raises(RuntimeError, match="UNSUPPORTED"):
            api.dsa_indexer_decode(up.q[:2], up.cache, up.w[:2], (3000, 2500), (1, 1), wl.top_k,
                                   k_base=up.k_base[:2], stream=s)
    for _ in range(3):
        g.replay()
    s.synchronize()
    rows = range(wl.total_q)
    _check(up, eager_i.cpu().numpy(), eager_s.cpu().numpy(), rows)
    _check(up, out_i.cpu().numpy(), out_s.cpu().numpy(), rows)
    for r in rows:
        _same_set_up_to_exact_ties(out_i[r].cpu().numpy(), out_s[r].cpu().numpy(), eager_i[r].cpu().numpy(),
                                   eager_s[r].cpu().numpy(), f"replay row {r}")
    del g
    api.dsa_check_device_errors(s)
