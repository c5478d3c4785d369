"""Lightning Indexer scores and top-k selection (oracle side; test infrastructure).

What is computed, and where the pages say so:

* Score (page "从原理到代码：手把手教你理解DeepSeek-V3.2的闪电索引器设计", §2.1 核心计算公式;
  page "Lightning Indexer 详解", §4 打分公式; page "Study MLA Indexer", section 数学流):

      I[t, s] = sum_{i < H} w[t, i] * ReLU( q[t, i, :] . k[s, :] / sqrt(d) )

  with ONE key vector k[s] per history token shared by all H indexer heads
  ("Lightning Indexer 详解" §4 实现要点: heads exist on the query side only;
  "Study MLA Indexer", 两条 cache 区分: the indexer K cache holds one d_idx=128 row
  per token).  The 1/sqrt(d) factor follows the first and last pages; the second
  page omits it, and it changes no index (ReLU is positively homogeneous).
* Causality (first page §3 step 5, the tril mask; "Lightning Indexer 详解" §2.4 and
  "Study MLA Indexer" 两条 cache 区分: the current key is appended to the cache
  before scoring): query at position p sees keys s = 0..p inclusive.
* Top-k (first page §3 step 5 ``torch.topk``; "Lightning Indexer 详解" §2.3: at most
  min(k, L) positions exist): the min(k, p+1) largest I[p, s]; ties are broken by
  the smaller index; the unused slots hold index -1 and score -inf.

Inputs are exact fp64 values: bf16 inputs are decoded bit-exactly, FP8 inputs are
``code value * row scale`` (see ``fp8_e4m3``).  The contraction uses a fp64 matmul
(a library primitive); everything else is written out.
"""

from __future__ import annotations

import math

import numpy as np


def query_positions(seq_len: int, q_len: int) -> np.ndarray:
    """Positions of the q_len newest tokens of a sequence of seq_len tokens.

    The cache already holds the new keys when scoring runs, so query j of the
    step sits at position seq_len - q_len + j (a decode step with q_len == 2 is
    "causal within the pair": its first query does not see the second key).
    """
    if not (0 <= q_len <= seq_len):
        raise ValueError("need 0 <= q_len <= seq_len")
    return np.arange(seq_len - q_len, seq_len, dtype=np.int64)


def row_scores(q_t: np.ndarray, k_hist: np.ndarray, w_t: np.ndarray) -> np.ndarray:
    """I[t, s] for every s in k_hist (the caller passes only the causal history).

    q_t: [H, d] fp64, k_hist: [n, d] fp64, w_t: [H] fp64.  Returns [n] fp64.
    """
    q_t = np.asarray(q_t, dtype=np.float64)
    k_hist = np.asarray(k_hist, dtype=np.float64)
    w_t = np.asarray(w_t, dtype=np.float64)
    H, d = q_t.shape
    if k_hist.ndim != 2 or k_hist.shape[1] != d or w_t.shape != (H,):
        raise ValueError("shape mismatch in row_scores")
    logits = (k_hist @ q_t.T) / math.sqrt(d)        # [n, H]: q[t,i,:].k[s,:] / sqrt(d)
    relu = np.maximum(logits, 0.0)                  # ReLU per head
    return relu @ w_t                               # sum_i w[t,i] * ReLU(...)


def topk_row(scores: np.ndarray, top_k: int) -> tuple[np.ndarray, np.ndarray]:
    """The min(top_k, n) largest entries of one causal score row, padded to top_k.

    Order: score descending, then index ascending.  Returns (idx int32 [top_k],
    score fp64 [top_k]) with -1 / -inf in the unused slots.
    """
    scores = np.asarray(scores, dtype=np.float64)
    n = scores.shape[0]
    if top_k <= 0:
        raise ValueError("top_k must be positive")
    order = np.lexsort((np.arange(n), -scores))    # last key is primary: -score, then index
    take = order[: min(top_k, n)]
    idx = np.full(top_k, -1, dtype=np.int32)
    val = np.full(top_k, -np.inf, dtype=np.float64)
    idx[: take.size] = take
    val[: take.size] = scores[take]
    return idx, val


def prefill_oracle(q: np.ndarray, k_seqs: list, w: np.ndarray, seq_lens, q_lens, top_k: int,
                   rows=None, keep_scores: bool = False) -> dict:
    """Indexer over a ragged batch.

    q:       [T_total, H, d] fp64, the queries of all sequences packed in order;
             sequence b owns q_lens[b] consecutive rows.
    k_seqs:  list of [seq_lens[b], d] fp64 key caches (keys already appended).
    w:       [T_total, H] fp64 head weights.
    rows:    optional iterable of global query rows to evaluate (default: all).
    Returns {"rows", "pos", "idx" [R, top_k] int32, "score" [R, top_k] fp64} and,
    with keep_scores, "scores": list of the full causal rows I[p, 0..p].
    """
    seq_lens = [int(x) for x in seq_lens]
    q_lens = [int(x) for x in (q_lens if q_lens is not None else seq_lens)]
    if len(seq_lens) != len(q_lens) or len(k_seqs) != len(seq_lens):
        raise ValueError("seq_lens, q_lens and k_seqs disagree on the batch size")
    T_total = sum(q_lens)
    if q.shape[0] != T_total or w.shape[0] != T_total:
        raise ValueError("q / w rows must equal sum(q_lens)")
    # map each global query row to (sequence, position)
    row_seq = np.repeat(np.arange(len(seq_lens)), q_lens)
    row_pos = np.concatenate([query_positions(L, n) for L, n in zip(seq_lens, q_lens)]) \
        if T_total else np.zeros(0, dtype=np.int64)
    sel = np.arange(T_total) if rows is None else np.asarray(list(rows), dtype=np.int64)
    out_idx = np.empty((sel.size, top_k), dtype=np.int32)
    out_val = np.empty((sel.size, top_k), dtype=np.float64)
    kept = []
    for j, r in enumerate(sel):
        b, p = int(row_seq[r]), int(row_pos[r])
        s_row = row_scores(q[r], k_seqs[b][: p + 1], w[r])
        out_idx[j], out_val[j] = topk_row(s_row, top_k)
        if keep_scores:
            kept.append(s_row)
    res = {"rows": sel, "pos": row_pos[sel], "idx": out_idx, "score": out_val}
    if keep_scores:
        res["scores"] = kept
    return res


def decode_oracle(q, k_seqs, w, seq_lens, q_len: int, top_k: int, rows=None,
                  keep_scores: bool = False) -> dict:
    """A decode step: q_len (1 or 2) new queries per sequence, at the end of each cache.

    Same definition as prefill ("Lightning Indexer 详解" §2: one query scores every
    cached position, then Top-k); only the query positions differ.
    """
    q_lens = [int(q_len)] * len(seq_lens)
    return prefill_oracle(q, k_seqs, w, seq_lens, q_lens, top_k, rows=rows, keep_scores=keep_scores)


def compressed_visible(position: int, m: int) -> int:
    """Complete blocks of m tokens a query at token position p sees: floor((p + 1) / m).

    Page "DeepSeek ... Lightning Indexer ... Lookahead Sparse Attention" (the agidaily
    survey), §三 CSA: every m consecutive tokens' cache entries are merged into one entry and
    the indexer scores those block entries instead of the raw tokens; the most recent tokens
    are covered by a separate sliding-window branch.  Reading: a block's entry exists once
    its m tokens are all in the cache, so the still-open block of the query is not scored.
    """
    return (int(position) + 1) // int(m)


def decode_compressed_oracle(q, kc_seqs, w, seq_lens, q_lens, m: int, top_k: int) -> dict:
    """Decode (or prefill: q_lens up to seq_lens) over an m-compressed key cache.

    kc_seqs[b]: [floor(seq_lens[b] / m), d] fp64 compressed keys of sequence b (block j covers
    tokens j*m .. j*m + m - 1); seq_lens / q_lens in tokens, queries at the last q_lens
    positions.  Query r at position p scores blocks 0 .. floor((p+1)/m) - 1 (same formula as
    row_scores) and keeps the top_k blocks.  Returns {"pos", "visible", "idx", "score"}.
    """
    seq_lens = [int(x) for x in seq_lens]
    q_lens = [int(x) for x in q_lens]
    row_seq = np.repeat(np.arange(len(seq_lens)), q_lens)
    row_pos = np.concatenate([query_positions(L, n) for L, n in zip(seq_lens, q_lens)])
    T = row_pos.size
    out_idx = np.empty((T, top_k), dtype=np.int32)
    out_val = np.empty((T, top_k), dtype=np.float64)
    vis = np.empty(T, dtype=np.int64)
    for r in range(T):
        b, p = int(row_seq[r]), int(row_pos[r])
        nv = compressed_visible(p, m)
        vis[r] = nv
        s_row = row_scores(q[r], kc_seqs[b][:nv], w[r]) if nv > 0 else np.zeros(0)
        out_idx[r], out_val[r] = topk_row(s_row, top_k)
    return {"pos": row_pos, "visible": vis, "idx": out_idx, "score": out_val}
