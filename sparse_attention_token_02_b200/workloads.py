"""Seeded synthetic workloads for the indexer (inputs only; none of the method's arithmetic).

Both sides of every parity check read their inputs from here: the CUDA path
uploads the arrays, the oracle decodes the same bits.  Nothing in this module
scores, quantises or selects anything.

Shapes and distributions follow the workloads the pages describe (DeepSeek-V3.2
indexer: d_I = 128, k = 2048, contexts up to 128K; "Study MLA Indexer", 关键参数):

=========  =====================================================================
tiny       1 sequence, L=512, H=4, d=64, k=32; q, k, w ~ N(0,1) fp32 from seed 0,
           w softmaxed over heads; rounded to bf16 at the boundary.
decode     32 sequences x L=32768, k[L,128] bf16 ~ N(0,1), one query per sequence
           q[64,128] bf16 ~ N(0,1/128), w = softmax of N(0,1) logits, H=64, k=2048.
prefill    1 sequence L=16384, H=64, d=128, q, k bf16 ~ N(0,1), 1% of key rows
           (chosen without replacement) scaled x4, w softmax, causal, k=2048.
prefill8   1 sequence L=65536, H=64, d=128, bf16 N(0,1) q and k sources that the
           indexer quantises to FP8-E4M3 with a per-token scale, w softmax, k=2048.
decode8    16 sequences, cache lengths uniform in [4096, 131072] (seeded), FP8 keys
           from bf16 N(0,1) sources, 2 queries per sequence (a speculative pair),
           q bf16 N(0,1) sources, H=64, d=128, k=2048.
=========  =====================================================================

Random numbers come from numpy's PCG64 through ``SeedSequence(seed).spawn``-style
keys ``(seed, tensor_id, chunk)``: every 4096-row chunk of every tensor has its own
stream, so a test can regenerate any rows of a large tensor without drawing the
rest.  Smaller variants of each workload (same recipe, fewer tokens) serve as
parity cases that the oracle finishes in seconds.
"""

from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np

CHUNK_ROWS = 4096

# tensor ids inside a workload's seed space
_T_K, _T_Q, _T_W, _T_OUTLIER, _T_LENS = 1, 2, 3, 4, 5


@dataclass(frozen=True)
class Workload:
    name: str
    seq_lens: tuple          # keys per sequence, the new tokens included
    q_lens: tuple            # queries per sequence (prefill: == seq_lens)
    H: int
    d: int
    top_k: int
    dtype: str               # "bf16" or "fp8" (what the indexer computes on)
    seed: int
    q_std: float = 1.0
    k_std: float = 1.0
    outlier_frac: float = 0.0  # fraction of key rows scaled by outlier_mult
    outlier_mult: float = 4.0
    note: str = ""
    extra: dict = field(default_factory=dict, compare=False)

    @property
    def num_seqs(self) -> int:
        return len(self.seq_lens)

    @property
    def total_q(self) -> int:
        return int(sum(self.q_lens))

    @property
    def total_k(self) -> int:
        return int(sum(self.seq_lens))

    @property
    def pairs(self) -> int:
        """Causal (query, key) pairs scored: sum over queries of (position + 1)."""
        tot = 0
        for L, n in zip(self.seq_lens, self.q_lens):
            first = L - n          # position of the first query
            tot += n * (first + 1) + n * (n - 1) // 2
        return int(tot)

    @property
    def kind(self) -> str:
        return "prefill" if tuple(self.q_lens) == tuple(self.seq_lens) else "decode"


def _ragged_lengths(seed: int, n: int, lo: int, hi: int) -> tuple:
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _T_LENS])))
    return tuple(int(x) for x in rng.integers(lo, hi + 1, size=n))


def tiny(seed: int = 0) -> Workload:
    return Workload("tiny", (512,), (512,), H=4, d=64, top_k=32, dtype="bf16", seed=seed,
                    note="fp32 N(0,1) sources rounded to bf16 at the boundary",
                    extra={"source": "fp32"})


def decode(num_seqs: int = 32, L: int = 32768, seed: int = 2) -> Workload:
    return Workload("decode", (L,) * num_seqs, (1,) * num_seqs, H=64, d=128, top_k=2048,
                    dtype="bf16", seed=seed, q_std=1.0 / np.sqrt(128.0))


def prefill(L: int = 16384, seed: int = 3) -> Workload:
    return Workload("prefill", (L,), (L,), H=64, d=128, top_k=2048, dtype="bf16", seed=seed,
                    outlier_frac=0.01)


def prefill8(L: int = 65536, seed: int = 4) -> Workload:
    return Workload("prefill8", (L,), (L,), H=64, d=128, top_k=2048, dtype="fp8", seed=seed)


def decode8(num_seqs: int = 16, lo: int = 4096, hi: int = 131072, seed: int = 5) -> Workload:
    lens = _ragged_lengths(seed, num_seqs, lo, hi)
    return Workload("decode8", lens, (2,) * num_seqs, H=64, d=128, top_k=2048, dtype="fp8",
                    seed=seed)


def scaled(wl: Workload, **kw) -> Workload:
    """Same recipe, other sizes (for parity cases the oracle finishes quickly)."""
    return replace(wl, **kw)


# ----------------------------------------------------------------------------- generators

def _rng(seed: int, tensor_id: int, chunk: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor_id, chunk])))


def normal_rows(seed: int, tensor_id: int, row_begin: int, row_end: int, row_len: int,
                std: float = 1.0) -> np.ndarray:
    """fp32 N(0, std^2) rows [row_begin, row_end) of a chunked tensor."""
    out = np.empty((row_end - row_begin, row_len), dtype=np.float32)
    c0, c1 = row_begin // CHUNK_ROWS, (row_end - 1) // CHUNK_ROWS if row_end > row_begin else -1
    for c in range(c0, c1 + 1):
        chunk = _rng(seed, tensor_id, c).standard_normal((CHUNK_ROWS, row_len), dtype=np.float32)
        lo = max(row_begin, c * CHUNK_ROWS)
        hi = min(row_end, (c + 1) * CHUNK_ROWS)
        out[lo - row_begin: hi - row_begin] = chunk[lo - c * CHUNK_ROWS: hi - c * CHUNK_ROWS]
    if std != 1.0:
        out *= np.float32(std)
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even) and return the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def softmax_rows(logits: np.ndarray) -> np.ndarray:
    """Head weights as the pages draw them: softmax over heads (first page §2.1, w_i)."""
    z = logits.astype(np.float64)
    z = z - z.max(axis=-1, keepdims=True)
    e = np.exp(z)
    return (e / e.sum(axis=-1, keepdims=True)).astype(np.float32)


def key_rows(wl: Workload, b: int, row_begin: int = 0, row_end: int | None = None) -> np.ndarray:
    """Key source rows of sequence b as fp32 values (rounded to bf16 at the boundary by the caller)."""
    L = wl.seq_lens[b]
    row_end = L if row_end is None else row_end
    x = normal_rows(wl.seed * 1000 + b, _T_K, row_begin, row_end, wl.d, wl.k_std)
    if wl.outlier_frac > 0:
        n_out = int(round(wl.outlier_frac * L))
        rng = _rng(wl.seed * 1000 + b, _T_OUTLIER, 0)
        rows = np.sort(rng.choice(L, size=n_out, replace=False))
        sel = rows[(rows >= row_begin) & (rows < row_end)] - row_begin
        x[sel] *= np.float32(wl.outlier_mult)
    return x


def query_rows(wl: Workload, row_begin: int, row_end: int) -> np.ndarray:
    """Query source rows [row_begin, row_end) of the packed [T_total, H, d] tensor (fp32)."""
    x = normal_rows(wl.seed, _T_Q, row_begin, row_end, wl.H * wl.d, wl.q_std)
    return x.reshape(row_end - row_begin, wl.H, wl.d)


def weight_rows(wl: Workload, row_begin: int, row_end: int) -> np.ndarray:
    """Head weights [row_begin, row_end) x H, fp32 softmax of N(0,1) logits."""
    return softmax_rows(normal_rows(wl.seed, _T_W, row_begin, row_end, wl.H))


def make_inputs(wl: Workload) -> dict:
    """All inputs of a workload, host side.

    Returns {"q_bits" uint16 [T,H,d], "k_bits": list of uint16 [L_b, d],
    "w" fp32 [T,H]} (bf16 bit patterns; FP8 workloads quantise these sources in
    the indexer's own append / quantise step).
    """
    T = wl.total_q
    q = query_rows(wl, 0, T)
    w = weight_rows(wl, 0, T)
    ks = [f32_to_bf16_bits(key_rows(wl, b)) for b in range(wl.num_seqs)]
    return {"q_bits": f32_to_bf16_bits(q), "k_bits": ks, "w": w}
