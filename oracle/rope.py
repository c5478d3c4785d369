"""Rotary position embedding of indexer keys and queries (oracle side; test infrastructure).

Only tests/, the smoke check and the bench's CPU baseline use this module; the CUDA
path shares no code with it.

The pages apply RoPE to the indexer key before it is quantised and cached, and to the
indexer query ("Study MLA Indexer", section 数学流: ``k_repr_t = RoPE(x_t W_kr) ->
quant(FP8)``, ``q_t = RoPE(x_t W_q)``; its 两条 cache 区分 table: the indexer K cache holds
the RoPE'd, quantised k_repr).  They give no further detail, so this follows the published
rotary embedding (Su et al., RoFormer): dimension pairs (a, b) of the first ``rope_dim``
values are rotated by the angle theta_i = p * base^(-2 i / rope_dim) of the token position
p,

    (a, b) -> (a cos theta_i - b sin theta_i,  a sin theta_i + b cos theta_i),

with pair i = (2i, 2i+1) ("interleaved") or (i, i + rope_dim/2) ("half"); values past
rope_dim pass through.  Everything here is fp64.
"""

from __future__ import annotations

import numpy as np


def rope_rows(x: np.ndarray, positions: np.ndarray, rope_dim: int, base: float = 10000.0,
              interleaved: bool = True) -> np.ndarray:
    """x [rows, d] (any float), positions [rows] -> rotated fp64 [rows, d]."""
    x = np.asarray(x, dtype=np.float64)
    pos = np.asarray(positions, dtype=np.float64)
    rows, d = x.shape
    assert rope_dim % 2 == 0 and 0 <= rope_dim <= d
    out = x.copy()
    half = rope_dim // 2
    for r in range(rows):
        for i in range(half):
            theta = pos[r] * base ** (-2.0 * i / rope_dim)
            c, s = np.cos(theta), np.sin(theta)
            ia, ib = (2 * i, 2 * i + 1) if interleaved else (i, i + half)
            a, b = x[r, ia], x[r, ib]
            out[r, ia] = a * c - b * s
            out[r, ib] = a * s + b * c
    return out


def rope_heads(q: np.ndarray, positions: np.ndarray, rope_dim: int, base: float = 10000.0,
               interleaved: bool = True) -> np.ndarray:
    """q [T, H, d], positions [T]: every head of token t rotated at position t's angle."""
    q = np.asarray(q, dtype=np.float64)
    T, H, d = q.shape
    flat = rope_rows(q.reshape(T * H, d), np.repeat(np.asarray(positions), H), rope_dim, base, interleaved)
    return flat.reshape(T, H, d)
