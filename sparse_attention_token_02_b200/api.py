"""Python binding of the indexer's C ABI: torch tensors in, pointers out.

Argument marshalling only.  torch provides device memory and the current CUDA
stream; every step of the indexer runs in the CUDA library.  Names follow the C
entry points (include/dsa_indexer.h).
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass

import numpy as np
import torch

from . import _lib
from ._lib import DSA_BF16, DSA_F32, DSA_FP8_E4M3, Batch, KCache, Query, check


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DSA_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return DSA_FP8_E4M3
    if t.dtype == torch.float32:
        return DSA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _require_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("device tensors must be contiguous CUDA tensors")


@dataclass
class IndexerKCache:
    """An indexer key cache: ``k`` [capacity, d_I] bf16 or uint8 (E4M3 codes), ``k_scale`` [capacity] fp32 (FP8)."""
    k: torch.Tensor
    k_scale: torch.Tensor | None = None

    @staticmethod
    def empty(capacity: int, d_I: int, fp8: bool, device="cuda") -> "IndexerKCache":
        if fp8:
            return IndexerKCache(torch.zeros(capacity, d_I, dtype=torch.uint8, device=device),
                                 torch.ones(capacity, dtype=torch.float32, device=device))
        return IndexerKCache(torch.zeros(capacity, d_I, dtype=torch.bfloat16, device=device), None)

    @property
    def fp8(self) -> bool:
        return self.k.dtype in (torch.uint8, torch.float8_e4m3fn)

    def c(self) -> KCache:
        _require_cuda(self.k, self.k_scale)
        return KCache(self.k.data_ptr(), self.k_scale.data_ptr() if self.k_scale is not None else None,
                      self.k.shape[0], self.k.shape[1], DSA_FP8_E4M3 if self.fp8 else DSA_BF16)


def _query(q: torch.Tensor, q_scale) -> Query:
    _require_cuda(q, q_scale)
    if q.dim() != 3:
        raise ValueError("q must be [T_total, H_I, d_I]")
    code = _dtype_code(q)
    return Query(q.data_ptr(), q_scale.data_ptr() if q_scale is not None else None, code, q.shape[1], q.shape[2])


class _HostBatch:
    """Keeps the host arrays of a dsa_batch_t alive for the duration of a call.  Built once
    with host_batch() it can be passed in place of ``seq_lens`` to the calls that take one,
    so a loop over steps with the same batch does not convert the lists every step."""

    def __init__(self, seq_lens, q_lens, k_base):
        self.seq = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
        self.ql = None if q_lens is None else np.ascontiguousarray(np.asarray(q_lens, dtype=np.int32))
        self.kb = None if k_base is None else np.ascontiguousarray(np.asarray(k_base, dtype=np.int64))
        self.c = Batch(len(self.seq), self.seq.ctypes.data,
                       None if self.ql is None else self.ql.ctypes.data,
                       None if self.kb is None else self.kb.ctypes.data)

    @property
    def total_q(self) -> int:
        return int(self.seq.sum() if self.ql is None else self.ql.sum())


def host_batch(seq_lens, q_lens=None, k_base=None) -> _HostBatch:
    """A reusable batch description (seq_lens, q_lens, k_base as for the calls)."""
    return _HostBatch(seq_lens, q_lens, k_base)


def _batch(seq_lens, q_lens, k_base) -> _HostBatch:
    if isinstance(seq_lens, _HostBatch):
        if q_lens is not None or k_base is not None:
            raise ValueError("pass q_lens / k_base to host_batch(), not with a prebuilt batch")
        return seq_lens
    return _HostBatch(seq_lens, q_lens, k_base)


def dsa_indexer_kcache_append(cache: IndexerKCache, k_new: torch.Tensor, dst_rows: torch.Tensor, stream=None):
    """Write (bf16 cache) or quantise and write (FP8 cache) rows ``k_new`` [n, d_I] to ``dst_rows`` (int64)."""
    _require_cuda(k_new, dst_rows)
    if dst_rows.dtype != torch.int64:
        raise TypeError("dst_rows must be int64")
    kc = cache.c()
    check(_lib.load().dsa_indexer_kcache_append(ctypes.byref(kc), _ptr(k_new), _dtype_code(k_new), _ptr(dst_rows),
                                                k_new.shape[0], _stream(stream)))


def dsa_quantize_rows_fp8(src: torch.Tensor, dst=None, scale=None, stream=None):
    """Per-row FP8 E4M3 quantisation of ``src`` [rows, ...] (bf16 / fp32): returns (codes uint8, scale fp32 [rows])."""
    _require_cuda(src, dst, scale)
    rows = src.shape[0]
    row_len = src.numel() // max(rows, 1) if rows else 0
    if dst is None:
        dst = torch.empty(src.shape, dtype=torch.uint8, device=src.device)
    if scale is None:
        scale = torch.empty(rows, dtype=torch.float32, device=src.device)
    check(_lib.load().dsa_quantize_rows_fp8(_ptr(src), _dtype_code(src), rows, row_len, _ptr(dst), _ptr(scale),
                                            _stream(stream)))
    return dst, scale


def _run(fn_name, q, q_scale, cache, w, seq_lens, q_lens, k_base, top_k, out_idx, out_score, stream,
         scores=True):
    b = _batch(seq_lens, q_lens, k_base)
    T = b.total_q
    _require_cuda(w)
    if w.dtype != torch.float32:
        raise TypeError("w must be fp32")
    if out_idx is None:
        out_idx = torch.empty(T, top_k, dtype=torch.int32, device=q.device)
    if out_score is None and scores:
        out_score = torch.empty(T, top_k, dtype=torch.float32, device=q.device)
    _require_cuda(out_idx, out_score)
    qq, kc = _query(q, q_scale), cache.c()
    fn = getattr(_lib.load(), fn_name)
    check(fn(ctypes.byref(qq), ctypes.byref(kc), _ptr(w), ctypes.byref(b.c), top_k, _ptr(out_idx), _ptr(out_score),
             _stream(stream)))
    return out_idx, out_score


def dsa_indexer_prefill(q, cache: IndexerKCache, w, seq_lens, top_k, q_scale=None, q_lens=None, k_base=None,
                        out_idx=None, out_score=None, stream=None, scores=True):
    """Scores + top-k for every query of a ragged batch; returns (out_idx int32, out_score fp32) [T_total, top_k].
    ``scores=False`` (every sequence at most top_k long): the short-sequence bypass, no scoring,
    returns (out_idx, None)."""
    return _run("dsa_indexer_prefill", q, q_scale, cache, w, seq_lens, q_lens, k_base, top_k, out_idx, out_score,
                stream, scores)


def dsa_indexer_decode(q, cache: IndexerKCache, w, seq_lens, q_lens, top_k, q_scale=None, k_base=None,
                       out_idx=None, out_score=None, stream=None, scores=True):
    """A decode step (1..4 queries per sequence at the end of each cache); returns (out_idx, out_score).
    ``scores=False``: the short-sequence bypass, as for dsa_indexer_prefill."""
    return _run("dsa_indexer_decode", q, q_scale, cache, w, seq_lens, q_lens, k_base, top_k, out_idx, out_score,
                stream, scores)


def dsa_indexer_decode_noalloc(q, cache: IndexerKCache, w, seq_lens, q_lens, top_k, q_scale=None, k_base=None,
                               out_idx=None, out_score=None, fault=None, stream=None):
    """dsa_indexer_decode for callers that may not allocate device memory: the library
    keeps its scratch in a fixed static device array (16 MiB per device) instead of a
    cudaMalloc'd workspace.  ``fault`` (optional int32 [2] CUDA tensor) receives the
    first device fault.  Calls that overlap on the GPU share that array and race."""
    b = _HostBatch(seq_lens, q_lens, k_base)
    T = b.total_q
    _require_cuda(w, fault)
    if w.dtype != torch.float32:
        raise TypeError("w must be fp32")
    if out_idx is None:
        out_idx = torch.empty(T, top_k, dtype=torch.int32, device=q.device)
    if out_score is None:
        out_score = torch.empty(T, top_k, dtype=torch.float32, device=q.device)
    _require_cuda(out_idx, out_score)
    qq, kc = _query(q, q_scale), cache.c()
    check(_lib.load().dsa_indexer_decode_noalloc(ctypes.byref(qq), ctypes.byref(kc), _ptr(w), ctypes.byref(b.c),
                                                 top_k, _ptr(out_idx), _ptr(out_score), _ptr(fault),
                                                 _stream(stream)))
    return out_idx, out_score


def _host_step(fn_name, q_host, w_host, k_new_host, dst_rows_host, cache, batch, top_k, out_idx_host,
               out_score_host, q_scale_host, stream, done_event):
    for t in (q_host, w_host, k_new_host, dst_rows_host, out_idx_host, out_score_host, q_scale_host):
        if t is not None and (t.is_cuda or not t.is_contiguous()):
            raise ValueError(f"{fn_name} takes contiguous host tensors")
    if w_host.dtype != torch.float32 or out_score_host.dtype != torch.float32 or out_idx_host.dtype != torch.int32:
        raise TypeError("w and out_score must be fp32, out_idx int32")
    if dst_rows_host.dtype != torch.int64:
        raise TypeError("dst_rows must be int64")
    if q_host.dim() != 3:
        raise ValueError("q must be [T_total, H_I, d_I]")
    qq = Query(q_host.data_ptr(), q_scale_host.data_ptr() if q_scale_host is not None else None, _dtype_code(q_host),
               q_host.shape[1], q_host.shape[2])
    kc = cache.c()
    n_new = int(k_new_host.shape[0]) if k_new_host is not None else 0
    args = (ctypes.byref(qq), ctypes.byref(kc), _ptr(w_host), _ptr(k_new_host),
            _dtype_code(k_new_host) if n_new else DSA_BF16, _ptr(dst_rows_host), n_new, ctypes.byref(batch.c), top_k,
            _ptr(out_idx_host), _ptr(out_score_host), _stream(stream))
    if done_event is None:
        check(getattr(_lib.load(), fn_name)(*args))
        return
    if not done_event.cuda_event:               # torch creates its events on their first record
        done_event.record(torch.cuda.current_stream() if stream is None else stream)
    check(getattr(_lib.load(), fn_name + "_async")(*args, ctypes.c_void_p(done_event.cuda_event)))


def dsa_indexer_decode_host(q_host, w_host, k_new_host, dst_rows_host, cache: IndexerKCache, seq_lens, q_lens,
                            top_k, out_idx_host, out_score_host, q_scale_host=None, k_base=None, stream=None,
                            done_event=None):
    """One decode step from HOST tensors in a single library call (dsa_indexer_decode_host):
    upload the new keys (bf16 or fp32 [n_new, d_I], cache rows ``dst_rows_host`` int64), queries
    [T, H_I, d_I] (bf16, or uint8 E4M3 codes with ``q_scale_host``) and weights [T, H_I] fp32,
    append, score + select, and copy the selection into ``out_idx_host`` int32 / ``out_score_host``
    fp32 [T, top_k].  ``seq_lens`` may be a prebuilt host_batch() (q_lens and k_base then None).
    Returns at once; the host outputs are complete when ``stream`` has finished,
    or, with ``done_event`` (a torch.cuda.Event; dsa_indexer_decode_host_async), once that event
    has completed, while ``stream`` goes on without waiting for the read-back.  Pinned host
    tensors keep the copies asynchronous."""
    _host_step("dsa_indexer_decode_host", q_host, w_host, k_new_host, dst_rows_host, cache,
               _batch(seq_lens, q_lens, k_base), top_k, out_idx_host, out_score_host, q_scale_host, stream, done_event)


def dsa_indexer_prefill_host(q_host, w_host, k_new_host, dst_rows_host, cache: IndexerKCache, seq_lens, top_k,
                             out_idx_host, out_score_host, q_scale_host=None, q_lens=None, k_base=None, stream=None,
                             done_event=None):
    """One prefill step from HOST tensors in a single library call (dsa_indexer_prefill_host):
    the same uploads, append and read-back as dsa_indexer_decode_host around the prefill's
    scoring and selection (q_lens None: every key of a sequence has its query).  With
    ``done_event`` the read-back of one step overlaps the next step's kernels."""
    _host_step("dsa_indexer_prefill_host", q_host, w_host, k_new_host, dst_rows_host, cache,
               _batch(seq_lens, q_lens, k_base), top_k, out_idx_host, out_score_host, q_scale_host, stream, done_event)


def dsa_selftest_wait_expiry(limit_cycles=100000, stream=None):
    """Run the bounded-wait self-test (a wait on a barrier nothing completes, given up after
    limit_cycles); the expiry then shows in dsa_check_device_errors."""
    check(_lib.load().dsa_selftest_wait_expiry(int(limit_cycles), _stream(stream)))


def dsa_indexer_decode_compressed(q, cache: IndexerKCache, w, seq_lens, q_lens, m, top_k, q_scale=None,
                                  k_base=None, out_idx=None, out_score=None, stream=None):
    """Decode over an m-compressed key cache (block j of sequence b at cache row k_base[b] + j);
    seq_lens / q_lens in tokens.  Returns (block indices int32 [T, k], scores fp32 [T, k])."""
    return _run_compressed("dsa_indexer_decode_compressed", q, cache, w, seq_lens, q_lens, m, top_k, q_scale, k_base,
                           out_idx, out_score, stream)


def dsa_indexer_prefill_compressed(q, cache: IndexerKCache, w, seq_lens, m, top_k, q_scale=None, q_lens=None,
                                   k_base=None, out_idx=None, out_score=None, stream=None):
    """Prefill over an m-compressed key cache (as dsa_indexer_decode_compressed, any q_lens;
    None: every token of each sequence is a query)."""
    return _run_compressed("dsa_indexer_prefill_compressed", q, cache, w, seq_lens, q_lens, m, top_k, q_scale, k_base,
                           out_idx, out_score, stream)


def _run_compressed(fn_name, q, cache, w, seq_lens, q_lens, m, top_k, q_scale, k_base, out_idx, out_score, stream):
    b = _HostBatch(seq_lens, q_lens, k_base)
    T = b.total_q
    _require_cuda(w)
    if out_idx is None:
        out_idx = torch.empty(T, top_k, dtype=torch.int32, device=q.device)
    if out_score is None:
        out_score = torch.empty(T, top_k, dtype=torch.float32, device=q.device)
    _require_cuda(out_idx, out_score)
    qq, kc = _query(q, q_scale), cache.c()
    check(getattr(_lib.load(), fn_name)(ctypes.byref(qq), ctypes.byref(kc), _ptr(w), ctypes.byref(b.c), int(m), top_k,
                                        _ptr(out_idx), _ptr(out_score), _stream(stream)))
    return out_idx, out_score


def _rope(d, rope_dim, base, interleaved):
    from ._lib import Rope
    return Rope(d if rope_dim is None else int(rope_dim), 1 if interleaved else 0, float(base))


def dsa_indexer_kcache_append_rope(cache: IndexerKCache, k_new, dst_rows, positions, rope_dim=None, base=10000.0,
                                   interleaved=True, stream=None):
    """Rotate pre-RoPE key rows k_new [n, d_I] (bf16/fp32) at ``positions`` (int32 [n]) and append
    them at cache rows ``dst_rows`` (int64 [n]); FP8 caches get the quantised rows + scales.
    rope_dim None rotates the whole vector."""
    _require_cuda(k_new, dst_rows, positions)
    if dst_rows.dtype != torch.int64 or positions.dtype != torch.int32:
        raise TypeError("dst_rows must be int64 and positions int32")
    r = _rope(cache.k.shape[1], rope_dim, base, interleaved)
    kc = cache.c()
    check(_lib.load().dsa_indexer_kcache_append_rope(ctypes.byref(kc), _ptr(k_new.contiguous()), _dtype_code(k_new),
                                                     _ptr(dst_rows), _ptr(positions), int(k_new.shape[0]),
                                                     ctypes.byref(r), _stream(stream)))


def dsa_rope_queries(q_src, positions, fp8=False, rope_dim=None, base=10000.0, interleaved=True, out=None,
                     scale=None, stream=None):
    """Rotate pre-RoPE queries q_src [T, H, d] (bf16/fp32) at ``positions`` (int32 [T]); returns
    bf16 [T, H, d], or (uint8 E4M3 codes [T, H, d], fp32 scale [T]) with fp8=True."""
    _require_cuda(q_src, positions, out, scale)
    if positions.dtype != torch.int32:
        raise TypeError("positions must be int32")
    T, H, d = q_src.shape
    if out is None:
        out = torch.empty(T, H, d, dtype=torch.uint8 if fp8 else torch.bfloat16, device=q_src.device)
    if fp8 and scale is None:
        scale = torch.empty(T, dtype=torch.float32, device=q_src.device)
    r = _rope(d, rope_dim, base, interleaved)
    src = q_src.contiguous()
    check(_lib.load().dsa_rope_queries(_ptr(src), _dtype_code(src), T, H, d, _ptr(positions), ctypes.byref(r),
                                       _ptr(out), DSA_FP8_E4M3 if fp8 else DSA_BF16, _ptr(scale), _stream(stream)))
    return (out, scale) if fp8 else out


def selection_row_base(seq_lens, q_lens=None, k_base=None, device="cuda"):
    """int64 [T_total] device tensor: the cache row of position 0 of each packed query row's
    sequence (what dsa_gather_rows / dsa_selection_rows add to the selected positions).
    k_base None: sequences packed back to back from row 0; q_lens None: prefill (q_len = seq_len)."""
    seq = np.asarray(seq_lens, dtype=np.int64)
    ql = seq if q_lens is None else np.asarray(q_lens, dtype=np.int64)
    base = np.concatenate([[0], np.cumsum(seq)[:-1]]) if k_base is None else np.asarray(k_base, dtype=np.int64)
    return torch.from_numpy(np.repeat(base, ql).astype(np.int64)).to(device)


def dsa_gather_rows(src, idx, row_base, out=None, stream=None):
    """Gather the selected rows: out[r, j] = src[row_base[r] + idx[r, j]] (zeros for -1).
    src [rows, ...] any dtype, contiguous, rows of a multiple of 16 bytes; idx int32 [T, k];
    row_base int64 [T] (device).  Returns [T, k, ...] with src's dtype."""
    _require_cuda(src, idx, row_base, out)
    if idx.dtype != torch.int32 or row_base.dtype != torch.int64:
        raise TypeError("idx must be int32 and row_base int64")
    if not (src.is_contiguous() and idx.is_contiguous() and row_base.is_contiguous()):
        raise ValueError("src, idx and row_base must be contiguous")
    T, k = idx.shape
    row_bytes = src[0].numel() * src.element_size() if src.shape[0] else 0
    if out is None:
        out = torch.empty((T, k) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
    check(_lib.load().dsa_gather_rows(_ptr(src), src.shape[0], row_bytes, _ptr(idx), _ptr(row_base), T, k, _ptr(out),
                                      _stream(stream)))
    return out


def dsa_selection_rows(idx, row_base, out=None, stream=None):
    """int64 [T, k] cache rows of a selection: row_base[r] + idx[r, j], -1 where idx is -1."""
    _require_cuda(idx, row_base, out)
    T, k = idx.shape
    if out is None:
        out = torch.empty(T, k, dtype=torch.int64, device=idx.device)
    check(_lib.load().dsa_selection_rows(_ptr(idx), _ptr(row_base), T, k, _ptr(out), _stream(stream)))
    return out


def dsa_sort_selection(idx, score, stream=None):
    """Sort each row of a selection in place: score descending, then position ascending, padding last."""
    _require_cuda(idx, score)
    T, k = idx.shape
    check(_lib.load().dsa_sort_selection(_ptr(idx), _ptr(score), T, k, _stream(stream)))
    return idx, score


def dsa_indexer_scores(q, cache: IndexerKCache, w, seq_lens, q_scale=None, q_lens=None, k_base=None, ld=None,
                       out=None, stream=None):
    """Dense scores [T_total, ld] (entries after each query's position are left as they were: -inf here)."""
    b = _HostBatch(seq_lens, q_lens, k_base)
    if ld is None:
        ld = (int(b.seq.max()) + 3) // 4 * 4 if len(b.seq) else 4
    if out is None:
        out = torch.full((b.total_q, ld), float("-inf"), dtype=torch.float32, device=q.device)
    _require_cuda(w, out)
    qq, kc = _query(q, q_scale), cache.c()
    check(_lib.load().dsa_indexer_scores(ctypes.byref(qq), ctypes.byref(kc), _ptr(w), ctypes.byref(b.c), _ptr(out),
                                         ld, _stream(stream)))
    return out


def dsa_indexer_workspace_bytes(q, seq_lens, top_k, q_lens=None) -> int:
    b = _HostBatch(seq_lens, q_lens, None)
    qq = Query(0, None, _dtype_code(q), q.shape[1], q.shape[2])
    return int(_lib.load().dsa_indexer_workspace_bytes(ctypes.byref(qq), ctypes.byref(b.c), top_k))


def dsa_set_workspace(buf: torch.Tensor | None, stream=None):
    if buf is None:
        check(_lib.load().dsa_set_workspace(None, 0, _stream(stream)))
    else:
        _require_cuda(buf)
        check(_lib.load().dsa_set_workspace(_ptr(buf), buf.numel() * buf.element_size(), _stream(stream)))


def dsa_check_device_errors(stream=None):
    """Synchronise the stream and raise if one of the library's kernels recorded a fault."""
    check(_lib.load().dsa_check_device_errors(_stream(stream)))


def dsa_set_profile_events(begin=None, mid=None, end=None):
    """Register torch.cuda.Event objects (timing enabled) recorded around the next calls' kernels."""
    v = [None if e is None else ctypes.c_void_p(e.cuda_event) for e in (begin, mid, end)]
    check(_lib.load().dsa_set_profile_events(*v))


def dsa_kernel_launch_count() -> int:
    return int(_lib.load().dsa_kernel_launch_count())


def dsa_version() -> str:
    return _lib.load().dsa_version().decode()
