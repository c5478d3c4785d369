"""Pins of the oracle's scores and top-k against things other than itself.

* literals summed by hand (tests/golden/hand_summed_h2_d4.json);
* closed forms: unit-vector queries (the dot product is one key coordinate) and
  rank-1 inputs (the ranking is the ranking of a known scalar per key);
* brute force over tiny rows (the top-k definition checked element by element);
* invariants the pages fix (non-negativity for w >= 0, causality, "all positions
  when p+1 <= k", positive homogeneity, head permutation, batching, decode row ==
  prefill row);
* planted mistakes: mutated copies of the score function must fail some pin.
"""

import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import decode_oracle, prefill_oracle, row_scores, topk_row
from oracle import indexer as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _f(x):
    return -math.inf if x == "-inf" else float(x)


# ----------------------------------------------------------------------------- literals

@pytest.mark.parametrize("case", [0, 1])
def test_hand_summed_literals(case):
    g = _load("hand_summed_h2_d4.json")
    c = g["cases"][case]
    q = np.array(g["q"], dtype=np.float64)
    k = np.array(g["k"], dtype=np.float64)
    w = np.array(c["w"], dtype=np.float64)
    res = prefill_oracle(q, [k], w, [3], [3], g["top_k"], keep_scores=True)
    for r in range(3):
        assert res["scores"][r].tolist() == c["scores"][r]          # exact: dyadic values
        assert res["idx"][r].tolist() == c["topk_idx"][r]
        assert res["score"][r].tolist() == [_f(x) for x in c["topk_score"][r]]


def test_decode_walkthrough_returns_every_cached_position():
    g = _load("decode_walkthrough_L8.json")
    rng = np.random.default_rng(11)
    L = g["history"] + g["q_len"]
    k = rng.standard_normal((L, g["d"]))
    q = rng.standard_normal((1, g["H"], g["d"]))
    w = np.full((1, g["H"]), 1.0 / g["H"])
    res = decode_oracle(q, [k], w, [L], 1, g["top_k"])
    valid = res["idx"][0][res["idx"][0] >= 0]
    assert valid.size == g["expected_valid"]
    assert sorted(valid.tolist()) == g["expected_index_set"]
    assert np.all(res["score"][0][valid.size:] == -np.inf)


# ----------------------------------------------------------------------------- closed forms

def test_unit_vector_queries_pick_key_coordinates():
    # q[t, i] = e_i  =>  q[t,i].k[s] = k[s, i]  =>  I = sum_i w_i * relu(k[s,i]) / sqrt(d)
    rng = np.random.default_rng(1)
    H, d, n = 5, 16, 40
    k = rng.standard_normal((n, d))
    w = rng.uniform(0.0, 1.0, H)
    q_t = np.eye(d)[:H]
    got = row_scores(q_t, k, w)
    for s in range(n):
        expect = sum(w[i] * max(k[s, i], 0.0) for i in range(H)) / 4.0   # sqrt(16) = 4
        assert got[s] == pytest.approx(expect, rel=1e-14, abs=1e-300)


def test_rank_one_inputs_rank_by_key_scalar():
    # k[s] = a_s u, q[t,i] = b_i u with |u|^2 = d: q.k/sqrt(d) = a_s b_i sqrt(d).
    # With every b_i > 0 and w_i > 0: I = sqrt(d) * a_s * sum_i w_i b_i for a_s > 0, 0 otherwise.
    rng = np.random.default_rng(2)
    d, H, L, top_k = 16, 3, 50, 7
    u = np.ones(d)                                   # |u|^2 = 16 = d
    perm = rng.permutation(L)
    a = (perm - 10).astype(np.float64)               # distinct integers, some <= 0
    k = a[:, None] * u[None, :]
    b = np.array([0.5, 1.0, 2.0])
    w = np.array([0.2, 0.3, 0.5])
    q = np.tile((b[:, None] * u[None, :])[None], (L, 1, 1))
    res = prefill_oracle(q, [k], np.tile(w, (L, 1)), [L], [L], top_k, keep_scores=True)
    c = math.sqrt(d) * float(np.dot(w, b))
    for p in range(L):
        row = res["scores"][p]
        for s in range(p + 1):
            assert row[s] == pytest.approx(c * max(a[s], 0.0), rel=1e-14, abs=0.0)
        # expected set: the positive a_s in descending order, then the zero-score ties by index
        pos = sorted([s for s in range(p + 1) if a[s] > 0], key=lambda s: -a[s])
        zeros = [s for s in range(p + 1) if a[s] <= 0]
        expect = (pos + zeros)[:top_k]
        assert res["idx"][p][: len(expect)].tolist() == expect


def test_rank_one_negative_heads_are_cut_by_relu():
    # b = (+1, -1): head 0 fires for a_s > 0, head 1 for a_s < 0.
    d = 4
    u = np.ones(d)
    a = np.array([3.0, -2.0, 0.0, 1.0])
    k = a[:, None] * u
    q_t = np.stack([u, -u])
    w = np.array([0.25, 0.75])
    got = row_scores(q_t, k, w)
    # a_s * b_i * sqrt(d) = a_s * b_i * 2
    expect = [0.25 * 6.0, 0.75 * 4.0, 0.0, 0.25 * 2.0]
    assert got.tolist() == expect


# ----------------------------------------------------------------------------- top-k by brute force

def test_topk_definition_brute_force_on_tiny_rows():
    rng = np.random.default_rng(5)
    for trial in range(300):
        n = int(rng.integers(1, 12))
        top_k = int(rng.integers(1, 14))
        row = rng.integers(-3, 4, size=n).astype(np.float64)    # many ties on purpose
        idx, val = topk_row(row, top_k)
        m = min(n, top_k)
        sel = idx[:m]
        assert np.all(idx[m:] == -1) and np.all(val[m:] == -np.inf)
        assert len(set(sel.tolist())) == m
        rest = [s for s in range(n) if s not in set(sel.tolist())]
        for s in sel:
            for r in rest:
                assert row[s] > row[r] or (row[s] == row[r] and s < r)
        assert np.array_equal(val[:m], row[sel])
        # sorted by (score desc, index asc)
        keys = [(-row[s], s) for s in sel]
        assert keys == sorted(keys)


# ----------------------------------------------------------------------------- invariants

def _random_case(rng, L=60, H=4, d=8, wpos=True):
    k = rng.standard_normal((L, d))
    q = rng.standard_normal((L, H, d))
    w = rng.uniform(0.0, 1.0, (L, H)) if wpos else rng.standard_normal((L, H))
    return q, k, w


def test_nonnegative_when_w_nonnegative_and_causal():
    rng = np.random.default_rng(6)
    q, k, w = _random_case(rng)
    res = prefill_oracle(q, [k], w, [60], [60], 16, keep_scores=True)
    for p in range(60):
        assert np.all(res["scores"][p] >= 0)
        v = res["idx"][p]
        assert np.all(v[v >= 0] <= p)
        assert (v >= 0).sum() == min(16, p + 1)
        if p + 1 <= 16:
            assert sorted(v[v >= 0].tolist()) == list(range(p + 1))


def test_positive_homogeneity_and_head_permutation():
    rng = np.random.default_rng(8)
    q, k, w = _random_case(rng, wpos=False)
    base = prefill_oracle(q, [k], w, [60], [60], 9, keep_scores=True)
    scaled = prefill_oracle(q * 2.5, [k], w, [60], [60], 9, keep_scores=True)
    perm = rng.permutation(q.shape[1])
    permuted = prefill_oracle(q[:, perm], [k], w[:, perm], [60], [60], 9, keep_scores=True)
    for p in range(60):
        tol = 1e-13 * np.abs(base["scores"][p]).max()      # w has mixed signs: cancellation
        assert np.allclose(scaled["scores"][p], 2.5 * base["scores"][p], rtol=1e-13, atol=2.5 * tol)
        assert np.allclose(permuted["scores"][p], base["scores"][p], rtol=1e-13, atol=tol)
    assert np.array_equal(scaled["idx"], base["idx"])


def test_batching_equals_separate_runs_and_decode_equals_prefill_row():
    rng = np.random.default_rng(9)
    q1, k1, w1 = _random_case(rng, L=30)
    q2, k2, w2 = _random_case(rng, L=45)
    both = prefill_oracle(np.concatenate([q1, q2]), [k1, k2], np.concatenate([w1, w2]),
                          [30, 45], [30, 45], 8)
    a = prefill_oracle(q1, [k1], w1, [30], [30], 8)
    b = prefill_oracle(q2, [k2], w2, [45], [45], 8)
    assert np.array_equal(both["idx"], np.concatenate([a["idx"], b["idx"]]))
    # a decode step of the last 2 tokens equals prefill rows 43, 44 of the second sequence
    dec = decode_oracle(q2[43:45], [k2], w2[43:45], [45], 2, 8)
    assert np.array_equal(dec["idx"], b["idx"][43:45])
    assert np.array_equal(dec["pos"], [43, 44])
    assert np.array_equal(dec["score"], b["score"][43:45])


# ----------------------------------------------------------------------------- planted mistakes

def _unit_vector_pin():
    rng = np.random.default_rng(1)
    H, d, n = 5, 16, 40
    k = rng.standard_normal((n, d))
    w = rng.uniform(0.0, 1.0, H)
    got = oracle.indexer.row_scores(np.eye(d)[:H], k, w)
    expect = [sum(w[i] * max(k[s, i], 0.0) for i in range(H)) / 4.0 for s in range(n)]
    assert np.allclose(got, expect, rtol=1e-14, atol=0)


def _pins_pass(score_fn):
    """Re-run the pins that go through the oracle with a replacement score function."""
    saved = oracle.indexer.row_scores
    oracle.indexer.row_scores = score_fn
    try:
        try:
            test_hand_summed_literals(0)
            test_hand_summed_literals(1)
            _unit_vector_pin()
            test_rank_one_inputs_rank_by_key_scalar()
        except AssertionError:
            return False
        return True
    finally:
        oracle.indexer.row_scores = saved


def _no_sqrt(q_t, k_hist, w_t):
    return np.maximum(k_hist @ q_t.T, 0.0) @ w_t


def _no_relu(q_t, k_hist, w_t):
    return ((k_hist @ q_t.T) / math.sqrt(q_t.shape[1])) @ w_t


def _relu_after_sum(q_t, k_hist, w_t):
    return np.maximum(((k_hist @ q_t.T) / math.sqrt(q_t.shape[1])) @ w_t, 0.0)


def _wrong_head_weight(q_t, k_hist, w_t):
    return np.maximum((k_hist @ q_t.T) / math.sqrt(q_t.shape[1]), 0.0) @ w_t[::-1]


def _sign_flip(q_t, k_hist, w_t):
    return np.maximum(-(k_hist @ q_t.T) / math.sqrt(q_t.shape[1]), 0.0) @ w_t


@pytest.mark.parametrize("mutant", [_no_sqrt, _no_relu, _relu_after_sum, _wrong_head_weight, _sign_flip])
def test_planted_mistakes_fail_a_pin(mutant):
    assert _pins_pass(oracle.indexer.row_scores)
    assert not _pins_pass(mutant)


def test_planted_causal_off_by_one_fails_a_pin():
    g = _load("hand_summed_h2_d4.json")
    c = g["cases"][0]
    q = np.array(g["q"], dtype=np.float64)
    k = np.array(g["k"], dtype=np.float64)
    w = np.array(c["w"], dtype=np.float64)
    # strict s < t would drop the diagonal: row 2 would lose its best key (s=2, score 1.0)
    strict = [row_scores(q[t], k[:t], w[t]) for t in range(3)]
    assert strict[2].tolist() != c["scores"][2]


# ----------------------------------------------------------------------------- m-compressed cache

def test_compressed_visible_at_block_boundaries():
    # m = 4: the block of tokens 0..3 exists from position 3 on
    assert [O.compressed_visible(p, 4) for p in (0, 2, 3, 6, 7, 8, 11)] == [0, 0, 1, 1, 2, 2, 3]
    assert [O.compressed_visible(p, 1) for p in (0, 5)] == [1, 6]


def test_compressed_decode_with_m_1_is_plain_decode():
    rng = np.random.default_rng(5)
    lens, q_lens, H, d, k = (40, 13), (2, 1), 3, 8, 6
    keys = [rng.standard_normal((L, d)) for L in lens]
    q = rng.standard_normal((sum(q_lens), H, d))
    w = rng.random((sum(q_lens), H))
    a = O.decode_compressed_oracle(q, keys, w, lens, q_lens, 1, k)
    b = O.prefill_oracle(q, keys, w, lens, q_lens, k)
    assert np.array_equal(a["idx"], b["idx"])
    assert np.array_equal(a["score"], b["score"])


def test_compressed_decode_hand_case():
    # H = 1, d = 1, w = 1: I[s] = ReLU(q k_s) / 1.  m = 2, sequence of 7 tokens -> 3 blocks.
    kc = [np.array([[1.0], [3.0], [-2.0]])]
    q = np.array([[[2.0]], [[2.0]]])
    w = np.ones((2, 1))
    res = O.decode_compressed_oracle(q, kc, w, (7,), (2,), 2, 2)
    # position 5 sees blocks 0..2 (floor(6/2) = 3); position 6 also 3 (block 3 not complete)
    assert res["visible"].tolist() == [3, 3]
    assert res["idx"][0].tolist() == [1, 0] and res["score"][0].tolist() == [6.0, 2.0]
    # with q_len 1 at the end of a 6-token sequence, floor(6/2) = 3 blocks as well
    res = O.decode_compressed_oracle(q[:1], kc, w[:1], (6,), (1,), 2, 4)
    assert res["idx"][0].tolist() == [1, 0, 2, -1]
    assert res["score"][0].tolist() == [6.0, 2.0, 0.0, -np.inf]
    # a 1-token sequence sees no block at m = 2
    res = O.decode_compressed_oracle(q[:1], [np.zeros((0, 1))], w[:1], (1,), (1,), 2, 2)
    assert res["visible"].tolist() == [0] and res["idx"][0].tolist() == [-1, -1]
