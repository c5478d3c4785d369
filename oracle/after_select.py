"""What the consumers of a selection do with it (oracle side; test infrastructure).

Only tests/, the smoke check and the bench's CPU baseline use this module; the CUDA
path shares no code with it.

* Gather of the selected latent rows ("Study MLA Indexer", section 数学流: the sparse
  MQA gathers the latent c^KV at the top-k positions; its 两条 cache 区分 table: the
  latent cache holds d_c = 512 values per token; "Lightning Indexer 详解" §1 在 DSA 中的
  角色: Core MLA attends only over the latent-cache entries of the index set I):

      out[r, j, :] = src[row_base[r] + idx[r, j], :]   for idx[r, j] >= 0
      out[r, j, :] = 0                                  for idx[r, j] == -1

  Rows are opaque bytes here (bf16, FP8 codes with scales, anything): a gather moves
  bytes and computes nothing.
* Global cache rows of a selection (for consumers that index one packed cache with
  int64 rows): row_base[r] + idx[r, j], and -1 where idx is -1.
* Sorted selection (the first page's ``torch.topk`` returns its k entries in
  descending score order, §3 step 5): each row ordered by score descending, then
  position ascending, padding (-1 / -inf) last.
"""

from __future__ import annotations

import numpy as np


def gather_rows(src: np.ndarray, idx: np.ndarray, row_base: np.ndarray) -> np.ndarray:
    """src [rows, row_bytes] uint8, idx [T, k] int32, row_base [T] int64 -> [T, k, row_bytes]."""
    src = np.asarray(src, dtype=np.uint8)
    idx = np.asarray(idx)
    row_base = np.asarray(row_base, dtype=np.int64)
    T, k = idx.shape
    out = np.zeros((T, k, src.shape[1]), dtype=np.uint8)
    for r in range(T):
        for j in range(k):
            if idx[r, j] >= 0:
                out[r, j] = src[row_base[r] + int(idx[r, j])]
    return out


def selection_rows(idx: np.ndarray, row_base: np.ndarray) -> np.ndarray:
    """int64 cache rows of a selection: row_base[r] + idx[r, j]; -1 stays -1."""
    idx = np.asarray(idx, dtype=np.int64)
    base = np.asarray(row_base, dtype=np.int64)[:, None]
    return np.where(idx >= 0, base + idx, -1)


def sort_selection(idx: np.ndarray, score: np.ndarray):
    """Each row by score descending, then position ascending; -1 entries last."""
    idx = np.asarray(idx)
    score = np.asarray(score)
    out_i = np.empty_like(idx)
    out_s = np.empty_like(score)
    for r in range(idx.shape[0]):
        entries = [(int(i), float(s)) for i, s in zip(idx[r], score[r])]
        valid = sorted((e for e in entries if e[0] >= 0), key=lambda e: (-e[1], e[0]))
        pad = [e for e in entries if e[0] < 0]
        rowv = valid + pad
        out_i[r] = [e[0] for e in rowv]
        out_s[r] = [e[1] for e in rowv]
    return out_i, out_s
