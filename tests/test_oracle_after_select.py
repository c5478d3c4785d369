"""Pins of the after-selection oracle (gather, global rows, sorted order) by hand-written cases.

Each literal below was written out by hand from the definitions in oracle/after_select.py;
a wrong base offset, a -1 that is not zero-filled, a reversed tie-break or padding sorted
into the middle each fails one of them.
"""

from __future__ import annotations

import numpy as np
import pytest

from oracle import after_select as A


def _src():
    # 5 rows of 16 bytes; row r holds bytes 16*r .. 16*r+15
    return np.arange(80, dtype=np.uint8).reshape(5, 16)


def test_gather_rows_hand_case():
    idx = np.array([[2, -1, 0], [1, 1, -1]], dtype=np.int32)
    base = np.array([1, 3], dtype=np.int64)
    out = A.gather_rows(_src(), idx, base)
    assert out.shape == (2, 3, 16)
    # row 0: base 1 -> source rows 3, (zero), 1
    assert out[0, 0, 0] == 48 and out[0, 0, 15] == 63
    assert not out[0, 1].any()
    assert out[0, 2, 0] == 16 and out[0, 2, 15] == 31
    # row 1: base 3 -> source rows 4, 4, (zero)
    assert out[1, 0, 0] == 64 and out[1, 1, 15] == 79
    assert not out[1, 2].any()


def test_gather_rows_moves_bytes_only():
    # arbitrary byte patterns (e.g. bf16 NaN payloads) come through unchanged
    src = np.array([[0xFF, 0x7F] * 8, [0x80, 0x00] * 8], dtype=np.uint8)
    out = A.gather_rows(src, np.array([[1, 0]], dtype=np.int32), np.array([0], dtype=np.int64))
    assert out[0, 0].tolist() == [0x80, 0x00] * 8
    assert out[0, 1].tolist() == [0xFF, 0x7F] * 8


def test_selection_rows_hand_case():
    idx = np.array([[0, 5, -1], [2, -1, -1]], dtype=np.int32)
    base = np.array([100, 7], dtype=np.int64)
    assert A.selection_rows(idx, base).tolist() == [[100, 105, -1], [9, -1, -1]]


def test_sort_selection_hand_case():
    idx = np.array([[4, 1, -1, 7, 2]], dtype=np.int32)
    score = np.array([[0.5, 2.0, -np.inf, 0.5, 3.0]], dtype=np.float32)
    oi, os = A.sort_selection(idx, score)
    # 3.0 (2), 2.0 (1), then the tie 0.5 by position: 4 before 7, padding last
    assert oi.tolist() == [[2, 1, 4, 7, -1]]
    assert os.tolist() == [[3.0, 2.0, 0.5, 0.5, -np.inf]]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_sort_selection_against_lexsort(seed):
    rng = np.random.default_rng(seed)
    T, k = 6, 40
    idx = np.stack([rng.permutation(100)[:k] for _ in range(T)]).astype(np.int32)
    score = rng.integers(-3, 4, (T, k)).astype(np.float32)        # many ties
    n_pad = rng.integers(0, 10, T)
    for r in range(T):
        idx[r, k - n_pad[r]:] = -1
        score[r, k - n_pad[r]:] = -np.inf
    oi, os = A.sort_selection(idx, score)
    for r in range(T):
        m = k - n_pad[r]
        order = np.lexsort((idx[r, :m], -score[r, :m]))
        assert oi[r, :m].tolist() == idx[r, :m][order].tolist()
        assert os[r, :m].tolist() == score[r, :m][order].tolist()
        assert (oi[r, m:] == -1).all() and np.isneginf(os[r, m:]).all()
