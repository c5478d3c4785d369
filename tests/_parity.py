"""Helpers shared by the GPU parity tests: input upload and the comparison rule.

Comparison rule for one query row (tolerance `rtol`: 2e-3 for bf16, 3e-2 for FP8):
  * exactly min(top_k, p+1) valid entries, distinct, inside 0..p; the rest are -1 / -inf;
  * every returned score is within rtol * max(|oracle score|, |o_k|) of the oracle's
    score of that index, where o_k is the oracle's k-th largest score of the row
    (the row maximum when every position is returned);
  * the index set equals the oracle's except for indices whose oracle score lies
    within rtol * max(|o_k|, 1e-30) of o_k (near-ties at the selection boundary).
"""

from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_attention_token_02_b200 import workloads as W
from sparse_attention_token_02_b200.api import IndexerKCache, dsa_indexer_kcache_append, dsa_quantize_rows_fp8

RTOL = {"bf16": 2e-3, "fp8": 3e-2}


def bits_to_bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


class OracleInputs:
    """The exact fp64 values the oracle sees for a workload's host inputs (bf16 bits
    decoded exactly; FP8 sources through the oracle's own codec)."""

    def __init__(self, wl: W.Workload, inputs: dict | None = None):
        self.wl = wl
        self.inp = inputs if inputs is not None else W.make_inputs(wl)

    def oracle_keys(self, b: int) -> np.ndarray:
        bits = self.inp["k_bits"][b]
        if self.wl.dtype == "fp8":
            codes, scale = oracle.quantize_rows(oracle.bf16_bits_to_f64(bits).astype(np.float32))
            return oracle.e4m3_decode(codes) * scale[:, None].astype(np.float64)
        return oracle.bf16_bits_to_f64(bits)

    def oracle_queries(self, rows) -> np.ndarray:
        bits = self.inp["q_bits"][rows]
        if self.wl.dtype == "fp8":
            flat = oracle.bf16_bits_to_f64(bits.reshape(len(rows), -1)).astype(np.float32)
            codes, scale = oracle.quantize_rows(flat)
            vals = oracle.e4m3_decode(codes) * scale[:, None].astype(np.float64)
            return vals.reshape(bits.shape)
        return oracle.bf16_bits_to_f64(bits)

    def row_meta(self):
        """(sequence, position) of every packed query row."""
        seq, pos = [], []
        for b, (Lb, n) in enumerate(zip(self.wl.seq_lens, self.wl.q_lens)):
            seq += [b] * n
            pos += list(range(Lb - n, Lb))
        return np.array(seq, dtype=np.int64), np.array(pos, dtype=np.int64)

    def oracle_rows(self, rows):
        """Full causal score rows I[p, 0..p] (fp64) of the given packed query rows."""
        seq, pos = self.row_meta()
        rows = list(rows)
        qv = self.oracle_queries(np.array(rows, dtype=np.int64))
        w = self.inp["w"][rows].astype(np.float64)
        keys = {}
        out = []
        for j, r in enumerate(rows):
            b = int(seq[r])
            if b not in keys:
                keys[b] = self.oracle_keys(b)
            out.append(oracle.row_scores(qv[j], keys[b][: pos[r] + 1], w[j]))
        return out


class Uploaded(OracleInputs):
    """A workload's inputs on the device (through the library's own append / quantise)
    plus the exact fp64 values the oracle must see."""

    def __init__(self, wl: W.Workload, inputs: dict | None = None, device="cuda"):
        super().__init__(wl, inputs)
        inp = self.inp
        fp8 = wl.dtype == "fp8"
        L = list(wl.seq_lens)
        self.k_base = np.concatenate([[0], np.cumsum(L)[:-1]]).astype(np.int64) if L else np.zeros(0, np.int64)
        total = int(sum(L))
        self.cache = IndexerKCache.empty(max(total, 1), wl.d, fp8, device)
        if total:
            k_src = bits_to_bf16_tensor(np.concatenate(inp["k_bits"]), device)
            rows = torch.arange(total, dtype=torch.int64, device=device)
            dsa_indexer_kcache_append(self.cache, k_src, rows)
        q_src = bits_to_bf16_tensor(inp["q_bits"], device)
        if fp8:
            codes, scale = dsa_quantize_rows_fp8(q_src.reshape(q_src.shape[0], -1))
            self.q = codes.reshape(q_src.shape)
            self.q_scale = scale
        else:
            self.q = q_src
            self.q_scale = None
        self.w = torch.from_numpy(inp["w"]).to(device)
        torch.cuda.synchronize()


def check_row(gpu_idx: np.ndarray, gpu_score: np.ndarray, orow: np.ndarray, top_k: int, rtol: float,
              what: str = "") -> None:
    n = orow.shape[0]
    m = min(top_k, n)
    valid = gpu_idx >= 0
    assert valid.sum() == m, f"{what}: {valid.sum()} valid entries, expected {m}"
    assert np.all(valid[:m]), f"{what}: valid entries are not first"
    assert np.all(gpu_idx[m:] == -1) and np.all(np.isneginf(gpu_score[m:])), f"{what}: bad padding"
    sel = gpu_idx[:m].astype(np.int64)
    assert len(np.unique(sel)) == m, f"{what}: duplicate indices"
    assert sel.min() >= 0 and sel.max() < n, f"{what}: index outside the causal range"
    ref_idx, _ = oracle.topk_row(orow, top_k)
    ref = ref_idx[:m].astype(np.int64)
    o_k = orow[ref[-1]] if n > top_k else np.max(orow)
    floor = max(abs(o_k), 1e-30)
    err = np.abs(gpu_score[:m].astype(np.float64) - orow[sel])
    bound = rtol * np.maximum(np.abs(orow[sel]), floor)
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} scores off; worst rel {np.max(err / np.maximum(bound / rtol, 1e-300)):.3e}")
    diff = np.setxor1d(sel, ref)
    if diff.size:
        gap = np.abs(orow[diff] - o_k)
        assert np.all(gap <= rtol * floor), (f"{what}: {diff.size} indices differ from the oracle's set and "
                                             f"are not near-ties (max gap {gap.max() / floor:.3e} of o_k)")


def run_indexer(up: Uploaded, decode: bool = False, top_k: int | None = None, stream=None):
    """One prefill or decode call of the library on an uploaded workload; host copies of
    (out_idx, out_score)."""
    from sparse_attention_token_02_b200 import api
    wl = up.wl
    k = wl.top_k if top_k is None else top_k
    if decode:
        idx, sc = api.dsa_indexer_decode(up.q, up.cache, up.w, wl.seq_lens, wl.q_lens, k, q_scale=up.q_scale,
                                         k_base=up.k_base, stream=stream)
    else:
        idx, sc = api.dsa_indexer_prefill(up.q, up.cache, up.w, wl.seq_lens, k, q_scale=up.q_scale,
                                          q_lens=wl.q_lens, k_base=up.k_base, stream=stream)
    api.dsa_check_device_errors(stream)
    return idx.cpu().numpy(), sc.cpu().numpy()


def sample_rows(wl: W.Workload, n_mid: int = 8, seed: int = 0):
    """Packed query rows to check on a large workload: the first and last rows, the rows
    around the top_k boundary, and n_mid seeded random rows."""
    T = wl.total_q
    rng = np.random.default_rng(seed)
    picks = {0, 1, T - 1, T - 2}
    k = wl.top_k
    seq_pos = []
    for Lb, n in zip(wl.seq_lens, wl.q_lens):
        seq_pos += list(range(Lb - n, Lb))
    seq_pos = np.array(seq_pos)
    for target in (k - 2, k - 1, k, k + 1, 2 * k + 5):
        hit = np.nonzero(seq_pos == target)[0]
        if hit.size:
            picks.add(int(hit[0]))
    picks.update(int(x) for x in rng.integers(0, T, size=n_mid))
    return sorted(p for p in picks if 0 <= p < T)


def check_rows(up: Uploaded, idx, sc, rows, top_k=None):
    """check_row against the oracle for each of the given packed query rows."""
    k = up.wl.top_k if top_k is None else top_k
    rtol = RTOL[up.wl.dtype]
    rows = list(rows)
    for r, orow in zip(rows, up.oracle_rows(rows)):
        check_row(idx[r], sc[r], orow, k, rtol, what=f"{up.wl.name} row {r}")
