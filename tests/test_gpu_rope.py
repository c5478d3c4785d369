"""RoPE fused into the key append and the query quantisation, against oracle/rope.py.

Rotated values are compared with the fp64 oracle to within one step of the stored format
(bf16: 8 significant bits; E4M3: 4), since the GPU rotates in fp32; a decode over RoPE'd
keys and queries is then checked row by row against the oracle's scores of the fp64-rotated,
bf16-rounded inputs.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import fp8_e4m3 as F
from oracle import indexer as O
from oracle import rope as R
from sparse_attention_token_02_b200 import api
from sparse_attention_token_02_b200 import workloads as W

from ._parity import RTOL, bits_to_bf16_tensor, check_row

pytestmark = pytest.mark.gpu

LAYOUTS = [(True, None), (False, None), (True, 64), (False, 64)]   # (interleaved, rope_dim)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    api.dsa_version()
    yield
    api.dsa_check_device_errors()


def _bf16_step(x):
    """Spacing of bf16 values around |x| (8 significant bits)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


# The GPU rotates in fp32: where a cos - b sin nearly cancels, the result is tiny while its
# rounding error still scales with |a|, |b| (about 2^-24 of them; inputs here are N(0, 1)).
ATOL_CANCEL = 2e-6


def _within_one_bf16_step(got_bf16: torch.Tensor, ref: np.ndarray):
    g = got_bf16.float().cpu().numpy().astype(np.float64)
    bound = _bf16_step(ref) + ATOL_CANCEL
    assert np.all(np.abs(g - ref) <= bound), np.max(np.abs(g - ref) / bound)


def _within_one_e4m3_step(codes: torch.Tensor, scale: torch.Tensor, ref: np.ndarray):
    s = scale.cpu().numpy().astype(np.float64)
    s = s.reshape(s.shape + (1,) * (ref.ndim - s.ndim))
    dec = F.e4m3_decode(codes.cpu().numpy().reshape(ref.shape)) * s
    step = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref) / s, 2.0 ** -9))) - 3), 2.0 ** -9) * s
    step = step + ATOL_CANCEL
    assert np.all(np.abs(dec - ref) <= step), np.max(np.abs(dec - ref) / step)


def _keys(n, d, seed):
    rng = np.random.default_rng(seed)
    bits = W.f32_to_bf16_bits(rng.standard_normal((n, d)).astype(np.float32))
    pos = np.concatenate([[0, 1, 131071, 65536], rng.integers(0, 131072, n - 4)]).astype(np.int32)
    return bits, pos


@pytest.mark.parametrize("interleaved,rope_dim", LAYOUTS)
@pytest.mark.parametrize("fp8", [False, True])
def test_append_rope_against_oracle(interleaved, rope_dim, fp8):
    n, d = 300, 128
    bits, pos = _keys(n, d, 1 + fp8)
    cache = api.IndexerKCache.empty(n + 10, d, fp8)
    rows = torch.arange(5, n + 5, dtype=torch.int64, device="cuda")
    api.dsa_indexer_kcache_append_rope(cache, bits_to_bf16_tensor(bits, "cuda"), rows,
                                       torch.from_numpy(pos).cuda(), rope_dim=rope_dim, interleaved=interleaved)
    api.dsa_check_device_errors()
    ref = R.rope_rows(F.bf16_bits_to_f64(bits), pos, rope_dim or d, interleaved=interleaved)
    if fp8:
        want_scale = np.abs(ref).max(axis=1).astype(np.float32) / np.float32(448)
        got_scale = cache.k_scale[5:n + 5].cpu().numpy()
        np.testing.assert_allclose(got_scale, want_scale, rtol=1e-6)
        _within_one_e4m3_step(cache.k[5:n + 5], cache.k_scale[5:n + 5], ref)
    else:
        _within_one_bf16_step(cache.k[5:n + 5].view(torch.bfloat16), ref)


@pytest.mark.parametrize("interleaved,rope_dim", LAYOUTS)
@pytest.mark.parametrize("fp8", [False, True])
def test_rope_queries_against_oracle(interleaved, rope_dim, fp8):
    T, H, d = 40, 64, 128
    rng = np.random.default_rng(7)
    bits = W.f32_to_bf16_bits(rng.standard_normal((T, H, d)).astype(np.float32))
    pos = rng.integers(0, 131072, T).astype(np.int32)
    res = api.dsa_rope_queries(bits_to_bf16_tensor(bits, "cuda"), torch.from_numpy(pos).cuda(), fp8=fp8,
                               rope_dim=rope_dim, interleaved=interleaved)
    ref = R.rope_heads(F.bf16_bits_to_f64(bits.reshape(T * H, d)).reshape(T, H, d), pos, rope_dim or d,
                       interleaved=interleaved)
    if fp8:
        codes, scale = res
        np.testing.assert_allclose(scale.cpu().numpy(),
                                   np.abs(ref).reshape(T, -1).max(axis=1).astype(np.float32) / np.float32(448),
                                   rtol=1e-6)
        _within_one_e4m3_step(codes, scale, ref)
    else:
        _within_one_bf16_step(res, ref)


@pytest.mark.parametrize("T,H,d,f32,fp8,interleaved,rope_dim", [
    (4000, 64, 128, False, True, False, 64),     # several tokens per shared-memory slot
    (10000, 8, 64, True, True, True, None),      # fp32 source, eight-slot rings
    (700, 128, 128, False, False, True, 64),     # the largest token (eight chunks a thread)
    (301, 3, 64, True, False, False, 32),        # heads not a multiple of the warps
])
def test_rope_queries_ring_shapes(T, H, d, f32, fp8, interleaved, rope_dim):
    rng = np.random.default_rng(T + H)
    x = rng.standard_normal((T, H, d)).astype(np.float32)
    if f32:
        src, ref_in = torch.from_numpy(x).cuda(), x.astype(np.float64)
    else:
        bits = W.f32_to_bf16_bits(x)
        src = bits_to_bf16_tensor(bits, "cuda")
        ref_in = F.bf16_bits_to_f64(bits.reshape(T * H, d)).reshape(T, H, d)
    pos = rng.integers(0, 200000, T).astype(np.int32)
    res = api.dsa_rope_queries(src, torch.from_numpy(pos).cuda(), fp8=fp8, rope_dim=rope_dim, interleaved=interleaved)
    api.dsa_check_device_errors()
    ref = R.rope_heads(ref_in, pos, rope_dim or d, interleaved=interleaved)
    if fp8:
        codes, scale = res
        np.testing.assert_allclose(scale.cpu().numpy(),
                                   np.abs(ref).reshape(T, -1).max(axis=1).astype(np.float32) / np.float32(448),
                                   rtol=1e-6)
        _within_one_e4m3_step(codes, scale, ref)
    else:
        _within_one_bf16_step(res, ref)


def test_rope_rejects_unsupported_layouts():
    cache = api.IndexerKCache.empty(8, 128, False)
    k = torch.zeros(2, 128, dtype=torch.bfloat16, device="cuda")
    rows = torch.zeros(2, dtype=torch.int64, device="cuda")
    pos = torch.zeros(2, dtype=torch.int32, device="cuda")
    with pytest.raises(RuntimeError, match="UNSUPPORTED"):
        api.dsa_indexer_kcache_append_rope(cache, k, rows, pos, rope_dim=130)
    with pytest.raises(RuntimeError, match="UNSUPPORTED"):
        api.dsa_indexer_kcache_append_rope(cache, k, rows, pos, rope_dim=24, interleaved=False)


def test_decode_over_roped_keys_and_queries_matches_oracle():
    lens, q_lens, d, H, k = (3000, 2049, 700), (2, 1, 1), 128, 64, 512
    wl = W.scaled(W.decode(), seq_lens=lens, q_lens=q_lens, top_k=k, seed=70)
    inp = W.make_inputs(wl)
    base = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
    key_pos = np.concatenate([np.arange(L) for L in lens]).astype(np.int32)
    k_bits = np.concatenate(inp["k_bits"])
    cache = api.IndexerKCache.empty(int(sum(lens)), d, False)
    api.dsa_indexer_kcache_append_rope(cache, bits_to_bf16_tensor(k_bits, "cuda"),
                                       torch.arange(int(sum(lens)), dtype=torch.int64, device="cuda"),
                                       torch.from_numpy(key_pos).cuda(), rope_dim=64, interleaved=False)
    q_pos = np.concatenate([O.query_positions(L, n) for L, n in zip(lens, q_lens)]).astype(np.int32)
    q = api.dsa_rope_queries(bits_to_bf16_tensor(inp["q_bits"], "cuda"), torch.from_numpy(q_pos).cuda(),
                             rope_dim=64, interleaved=False)
    w = torch.from_numpy(inp["w"]).cuda()
    idx, sc = api.dsa_indexer_decode(q, cache, w, lens, q_lens, k, k_base=base)
    api.dsa_check_device_errors()
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    # oracle: fp64 rotation, then the bf16 rounding the cache and the queries are stored in
    rk = R.rope_rows(F.bf16_bits_to_f64(k_bits), key_pos, 64, interleaved=False)
    rk = F.bf16_bits_to_f64(W.f32_to_bf16_bits(rk.astype(np.float32)))
    T = int(sum(q_lens))
    rq = R.rope_heads(F.bf16_bits_to_f64(inp["q_bits"].reshape(T * H, d)).reshape(T, H, d), q_pos, 64,
                      interleaved=False)
    rq = F.bf16_bits_to_f64(W.f32_to_bf16_bits(rq.astype(np.float32)).reshape(T * H, d)).reshape(T, H, d)
    seq = np.repeat(np.arange(len(lens)), q_lens)
    for r in range(T):
        b, p = int(seq[r]), int(q_pos[r])
        orow = O.row_scores(rq[r], rk[base[b]: base[b] + p + 1], inp["w"][r].astype(np.float64))
        check_row(idx[r], sc[r], orow, k, RTOL["bf16"], what=f"roped decode row {r}")
