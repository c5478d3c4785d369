/*
 * dsa_indexer.h -- C ABI of the DeepSeek Sparse Attention Lightning Indexer on B200.
 *
 * The operation (page "从原理到代码：手把手教你理解DeepSeek-V3.2的闪电索引器设计" §2.1 and §3;
 * page "Lightning Indexer 详解" §2 and §4; page "Study MLA Indexer", section 数学流):
 *
 *     I[t, s] = sum_{i < H_I} w[t, i] * ReLU( q[t, i, :] . k[s, :] / sqrt(d_I) )
 *
 * for every query t and every cached key s at or before t's position, with ONE
 * d_I-dimensional indexer key per token shared by all H_I heads; then the
 * top_k largest I[t, s] per query (DeepSeek-V3.2 uses top_k = 2048).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers named "device" are CUDA device pointers on the current device;
 *   "host" pointers are read synchronously during the call and may be reused
 *   as soon as it returns -- except the *_host buffers of the host-step calls
 *   (dsa_indexer_decode_host, dsa_indexer_prefill_host and their _async forms),
 *   which are copied asynchronously and stay in use until the step completes.  Device pointers passed to the
 *   tensor-core path (the cache, the queries) must be 16-byte aligned.
 * - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every call
 *   only enqueues work on it; outputs are valid once the stream has reached
 *   that point.  Calls that share a stream may be issued back to back.
 * - Ownership: the library never frees or keeps caller memory.  It owns a
 *   workspace per (device, stream), grown on demand with cudaMalloc, unless
 *   the caller supplies one with dsa_set_workspace().
 * - Errors: argument problems are found before anything is enqueued and
 *   returned as a status; dsa_get_last_error() then holds a message (per
 *   thread).  Faults detected inside kernels (a cache row out of range, a
 *   bounded wait that expired, a broken selection invariant) are recorded in
 *   a device flag and reported by dsa_check_device_errors().
 * - Positions: the keys of a step are appended BEFORE scoring ("Study MLA
 *   Indexer", 两条 cache 区分), so a sequence with seq_len keys and q_len
 *   queries has its query j at position p = seq_len - q_len + j and that
 *   query sees keys 0..p (itself included).
 * - Output: for query row r, out_idx[r*top_k + j] (int32) are 0-based key
 *   positions inside the query's sequence and out_score[r*top_k + j] (fp32)
 *   their scores.  The min(top_k, p+1) valid entries come first; the rest are
 *   -1 / -inf.  The order of the valid entries is unspecified: the result is
 *   the index SET of "Lightning Indexer 详解" §1.  Among keys whose scores are
 *   exactly equal at the k-th place, which ones are kept is unspecified.
 */
#ifndef DSA_INDEXER_H
#define DSA_INDEXER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DSA_INDEXER_ABI_VERSION 1

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

typedef enum {
  DSA_BF16 = 0,      /* bfloat16 */
  DSA_FP8_E4M3 = 1,  /* OCP FP8 E4M3 ("e4m3fn") with one fp32 scale per row */
  DSA_F32 = 2        /* fp32, accepted as an append / quantise SOURCE only */
} dsa_dtype_t;

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, inconsistent batch, misalignment */
  DSA_ERR_UNSUPPORTED = 2,   /* valid request this build has no kernel for (H_I, d_I, dtype) */
  DSA_ERR_ALLOC = 3,         /* the library could not allocate its workspace */
  DSA_ERR_CUDA = 4,          /* a CUDA runtime call failed (message has the CUDA error) */
  DSA_ERR_DEVICE_CHECK = 5   /* a kernel recorded a fault (see dsa_check_device_errors) */
} dsa_status_t;

/* One layer's indexer key cache, packed by rows.  Sequences live at arbitrary
 * row ranges (see dsa_batch_t.k_base).  Row r holds the key of one token. */
typedef struct {
  void* k;                /* device [capacity_rows, d_I] bf16 or e4m3 bytes, row-major        */
  float* k_scale;         /* device [capacity_rows] fp32 per-row scale (FP8), NULL for bf16    */
  int64_t capacity_rows;  /* rows allocated in k (and k_scale)                                */
  int32_t d_I;            /* key width: 128 (DeepSeek-V3.2) or 64                              */
  dsa_dtype_t dtype;      /* DSA_BF16 or DSA_FP8_E4M3                                          */
} dsa_kcache_t;

/* Queries of all sequences, packed in sequence order: sequence b owns q_lens[b]
 * consecutive rows. */
typedef struct {
  const void* data;       /* device [T_total, H_I, d_I] bf16 or e4m3 bytes                     */
  const float* scale;     /* device [T_total] fp32 per-token scale (FP8), NULL for bf16        */
  dsa_dtype_t dtype;      /* must equal the cache dtype                                        */
  int32_t H_I;            /* indexer heads (64 in DeepSeek-V3.2)                               */
  int32_t d_I;            /* must equal the cache d_I                                          */
} dsa_query_t;

/* The ragged batch, described on the host. */
typedef struct {
  int32_t num_seqs;
  const int32_t* seq_lens;  /* host [num_seqs]: cached keys of each sequence, this step's included */
  const int32_t* q_lens;    /* host [num_seqs]: queries of each sequence; NULL means q_len == seq_len */
  const int64_t* k_base;    /* host [num_seqs]: cache row holding key position 0 of each sequence;
                               NULL means the sequences are packed back to back from row 0           */
} dsa_batch_t;

/*
 * Append keys to the cache ("Lightning Indexer 详解" §2.1 and §2.4: each new token's
 * key becomes the next cache row, history is never recomputed; "Study MLA
 * Indexer", 数学流: the K path is quantised to FP8 before the write).
 *   k_new     device [n, d_I] source rows, dtype src_dtype (DSA_BF16 or DSA_F32)
 *   dst_rows  device int64 [n]: destination cache row of each source row
 * bf16 cache: a copy (fp32 sources rounded to nearest even).  FP8 cache: each row
 * is quantised with its own scale = absmax / 448 (IEEE fp32 division), codes =
 * E4M3(x / scale) rounded to nearest even and saturated to +-448; an all-zero
 * row gets scale 1.  A destination outside [0, capacity_rows) is skipped and
 * recorded as a device fault.
 */
DSA_API dsa_status_t dsa_indexer_kcache_append(const dsa_kcache_t* kc, const void* k_new, dsa_dtype_t src_dtype,
                                       const int64_t* dst_rows, int32_t n, void* stream);

/*
 * Per-row FP8 quantisation, the routine the cache append uses; it also
 * quantises queries with one scale per token over all H_I * d_I values
 * (row_len = H_I * d_I).
 *   src    device [rows, row_len] DSA_BF16 or DSA_F32
 *   dst    device uint8 [rows, row_len] E4M3 codes
 *   scale  device fp32 [rows]
 * row_len must be a positive multiple of 16.
 */
DSA_API dsa_status_t dsa_quantize_rows_fp8(const void* src, dsa_dtype_t src_dtype, int64_t rows, int32_t row_len,
                                   uint8_t* dst, float* scale, void* stream);

/*
 * Prefill: score every query of every sequence against its causal history and
 * select the top_k keys ("从原理到代码…" §3: scores for all query/key pairs, causal
 * mask, topk; "Study MLA Indexer", 数学流: [L, L] logits then arg top-k [L, k]).
 *   q, kc     queries and cache as above (same dtype, same d_I)
 *   w         device fp32 [T_total, H_I] head weights (any sign; softmax output in
 *             DeepSeek-V3.2, "从原理到代码…" §2.1)
 *   batch     host description; T_total = sum(q_lens)
 *   top_k     >= 1
 *   out_idx   device int32 [T_total, top_k]
 *   out_score device fp32  [T_total, top_k], or NULL when every sequence has seq_len <=
 *             top_k: the short-sequence bypass ("Study MLA Indexer", 三个 why: with every
 *             sequence within k the selection is the whole causal history and the scores
 *             go unused), which launches no scoring kernel and writes out_idx[r] =
 *             0 .. n_r - 1, then -1.  NULL with a longer sequence is DSA_ERR_INVALID_ARG.
 * Supported shapes: (H_I, d_I) = (64, 128) in bf16 or FP8, (4, 64) in bf16.
 */
DSA_API dsa_status_t dsa_indexer_prefill(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w,
                                 const dsa_batch_t* batch, int32_t top_k, int32_t* out_idx, float* out_score,
                                 void* stream);

/*
 * Decode: the same scoring and selection for a step of 1 to 4 new queries per
 * sequence at the end of each cache ("Lightning Indexer 详解" §2: one query scores
 * every cached position, linear in L per step).  Arguments as for prefill;
 * every q_lens[b] must be in 1..4 (q_lens may not be NULL).  The key range of
 * each sequence is split across the GPU so few long sequences still fill it.
 * Supported shapes: (H_I, d_I) = (64, 128) in bf16 or FP8.
 */
DSA_API dsa_status_t dsa_indexer_decode(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w,
                                const dsa_batch_t* batch, int32_t top_k, int32_t* out_idx, float* out_score,
                                void* stream);

/*
 * One whole decode step from host memory (the serving loop of the second page, §2: append
 * the new token's key, score it and the cache, select), enqueued on `stream` without
 * waiting for it:
 *   1. copies k_new_host [n_new, d_I] (k_new_dtype: DSA_BF16 or DSA_F32) and
 *      dst_rows_host [n_new] to the device and appends them as dsa_indexer_kcache_append;
 *   2. copies q->data [T, H_I, d_I] (q->dtype), q->scale [T] (FP8) and w_host [T, H_I]
 *      to the device and scores + selects as dsa_indexer_decode (T = sum of q_lens);
 *      bf16 queries against an FP8 cache are first quantised on the device as
 *      dsa_quantize_rows_fp8 does (one scale per token);
 *   3. copies the selection back into out_idx_host / out_score_host [T, top_k].
 * Here q->data and q->scale are HOST pointers, like every *_host argument.  Page-locked
 * host memory keeps the copies asynchronous; pageable memory works, with CUDA staging it.
 * The copies run on two copy streams of the library (one per direction) and the device
 * copies live in two library-owned slots of `stream` used in turn, so the uploads of one
 * call overlap the kernels of the previous one; events order everything against `stream`.
 * The host inputs must stay unchanged, and the host outputs are complete, once `stream`
 * has finished (e.g. dsa_check_device_errors).  n_new may be 0.  Not capturable in a CUDA
 * graph (DSA_ERR_UNSUPPORTED while `stream` is capturing).
 */
DSA_API dsa_status_t dsa_indexer_decode_host(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w_host,
                                             const void* k_new_host, dsa_dtype_t k_new_dtype,
                                             const int64_t* dst_rows_host, int32_t n_new, const dsa_batch_t* batch,
                                             int32_t top_k, int32_t* out_idx_host, float* out_score_host,
                                             void* stream);

/*
 * dsa_indexer_decode_host without the read-back on `stream`: the device-to-host copies of
 * the selection are ordered only on the library's copy stream, and done_event (a
 * cudaEvent_t the caller created, required) is recorded there once out_idx_host and
 * out_score_host are complete; wait on it (cudaEventSynchronize, cudaStreamWaitEvent)
 * before reading them.  `stream` does not wait for the read-back, so the read-back of one
 * step overlaps the kernels of the next.  Two calls in flight use the two slots: a third
 * call waits on the device for the first one's read-back before reusing its slot.
 */
DSA_API dsa_status_t dsa_indexer_decode_host_async(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w_host,
                                                   const void* k_new_host, dsa_dtype_t k_new_dtype,
                                                   const int64_t* dst_rows_host, int32_t n_new,
                                                   const dsa_batch_t* batch, int32_t top_k, int32_t* out_idx_host,
                                                   float* out_score_host, void* stream, void* done_event);

/*
 * The prefill counterparts of the two host-step calls above: the same copies, slots, copy
 * streams and ordering, with the scoring and selection of dsa_indexer_prefill (any q_lens,
 * q_lens may be NULL: every key of a sequence has its query).  A prefill step moves much more
 * than a decode step (the 65 536-token FP8 prefill uploads 1 GB of bf16 queries and reads 1 GB
 * of selection back), so the copies of one step overlap the kernels of its neighbours: the
 * uploads of step i+1 and the read-back of step i-1 (with the _async form) run while step i
 * scores.  Each slot holds a step's inputs and outputs on the device (both slots together about
 * 2 x (bf16 queries + selection) bytes, grown on demand with cudaMalloc).
 * ("Study MLA Indexer", 数学流: [L, L] logits then arg top-k [L, k], for a prompt of L tokens.)
 */
DSA_API dsa_status_t dsa_indexer_prefill_host(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w_host,
                                              const void* k_new_host, dsa_dtype_t k_new_dtype,
                                              const int64_t* dst_rows_host, int32_t n_new, const dsa_batch_t* batch,
                                              int32_t top_k, int32_t* out_idx_host, float* out_score_host,
                                              void* stream);
DSA_API dsa_status_t dsa_indexer_prefill_host_async(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w_host,
                                                    const void* k_new_host, dsa_dtype_t k_new_dtype,
                                                    const int64_t* dst_rows_host, int32_t n_new,
                                                    const dsa_batch_t* batch, int32_t top_k, int32_t* out_idx_host,
                                                    float* out_score_host, void* stream, void* done_event);

/*
 * The scores alone, without selection (the first page's index_scores, §3):
 * out_scores[r * ld + s] = I[p_r, s] for s = 0..p_r.  Entries with s > p_r are
 * not written.  ld >= max(seq_lens) and ld % 4 == 0.
 */
DSA_API dsa_status_t dsa_indexer_scores(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w,
                                const dsa_batch_t* batch, float* out_scores, int64_t ld, void* stream);

/*
 * Decode that allocates no device memory.  (The pages have no counterpart: this
 * is a library entry point for callers that may not allocate.)
 *
 * The decode step for callers that must not allocate device memory at all: a server
 * whose device memory belongs to its own pool (an allocation behind the pool's back can
 * fail or fragment it), code under a device-memory budget enforced outside CUDA, or a host
 * that forbids allocator calls on its hot path.  dsa_indexer_decode grows a workspace with
 * cudaMalloc; this call instead keeps the score rows and the scheduling tables in one
 * static 16 MiB __device__ array inside the library, which every GPU that loads the
 * library holds until the process exits.  It calls no cudaMalloc, cudaFree or other
 * allocating routine, and stages nothing through host memory: its tables reach the array
 * inside kernel parameters.
 *
 * Arguments as for dsa_indexer_decode, with these differences:
 *   fault      optional device int32[2]: cleared by the call, then receives the first
 *              device fault (code, info) as dsa_check_device_errors would report it;
 *              with NULL, faults are kept in the static array and not reported.
 *   out_score  required (the short-sequence bypass of dsa_indexer_decode is not offered).
 * The selection is the same (same rule, same tolerance of exact ties at the k-th score);
 * the route differs: after the logits kernel, one cluster of CTAs per row selects from
 * the row's scores alone (no coarse histogram from the logits epilogue), so a row may hold
 * at most 131072 keys (DSA_ERR_UNSUPPORTED beyond).
 * Limits: the batch must fit the array: 4 bytes per cached key of every query (rounded
 * up to 4 keys per query) plus its tables, else DSA_ERR_INVALID_ARG says how much it
 * needs.  Every call shares the one array (per device) and leaves its contents behind, so
 * calls that overlap on the GPU (other streams, other host threads) race; serialise them.
 * Set-up: the array is reserved on a device when the library's device code is loaded
 * there -- with CUDA's lazy module loading (the default) that happens during the first
 * call on the device, which can therefore fail with a CUDA out-of-memory error on a device
 * that is already full.  The first call on a device also looks up the array's device
 * address (cudaGetSymbolAddress) with that device current.  Make one call at
 * initialisation, before any stream capture.
 */
DSA_API dsa_status_t dsa_indexer_decode_noalloc(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w,
                                                const dsa_batch_t* batch, int32_t top_k, int32_t* out_idx,
                                                float* out_score, int32_t* fault, void* stream);

/*
 * Decode over an m-compressed indexer key cache (the agidaily survey of DSA and its
 * successors, §三 CSA: every m consecutive tokens' entries are merged into one, and the
 * indexer scores those block entries; the merge itself is learned and is the caller's).
 *   kc      cache of compressed keys: row k_base[b] + j holds block j of sequence b,
 *           i.e. tokens j*m .. j*m + m - 1 (bf16 or FP8 + scale, as for dsa_indexer_decode)
 *   batch   seq_lens / q_lens in TOKENS; the queries sit at the last q_lens positions;
 *           k_base = first compressed row of each sequence (NULL: sequences' blocks packed
 *           back to back from row 0, floor(seq_len / m) rows each)
 *   m       tokens per block (>= 1; m = 1 is dsa_indexer_decode)
 * A query at token position p sees the complete blocks j < floor((p + 1) / m): its own
 * still-open block is not scored (the sliding-window branch covers it).  out_idx holds
 * block indices j, out_score their scores; a query that sees no block gets only -1 / -inf.
 * Every q_lens[b] is 1..4.  The decode kernels run unchanged with each query's causal limit
 * moved to its last complete block; the queries of a sequence share every key tile.
 */
DSA_API dsa_status_t dsa_indexer_decode_compressed(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w,
                                                   const dsa_batch_t* batch, int32_t m, int32_t top_k,
                                                   int32_t* out_idx, float* out_score, void* stream);

/*
 * Prefill over an m-compressed cache: the same arguments and visibility as
 * dsa_indexer_decode_compressed, for any q_lens (0 .. seq_len, the queries at the last
 * q_lens positions, as for dsa_indexer_prefill); the prefill kernels run with each query's
 * causal limit moved to its last complete block.  out_score is required.
 */
DSA_API dsa_status_t dsa_indexer_prefill_compressed(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w,
                                                    const dsa_batch_t* batch, int32_t m, int32_t top_k,
                                                    int32_t* out_idx, float* out_score, void* stream);

/*
 * Rotary position embedding of indexer keys and queries, fused into the cache append and
 * the query quantisation (page "Study MLA Indexer", section 数学流: the key is RoPE'd, then
 * quantised and written to the indexer K cache; the query is RoPE'd).  The pages give no
 * RoPE detail; this is the published rotary embedding: pair i of the first rope_dim values
 * of each d_I-vector turns by theta_i = position * base^(-2i / rope_dim),
 * (a, b) -> (a cos - b sin, a sin + b cos); later values pass through.
 */
typedef struct {
  int32_t rope_dim;     /* leading values that rotate: even, <= d_I (0: none)               */
  int32_t interleaved;  /* 1: pairs (2i, 2i+1); 0: pairs (i, i + rope_dim/2), which needs     */
                        /*    rope_dim / 2 = 2^m * d_I / 32 and a multiple of 8                 */
                        /*    (d_I = 128: rope_dim 16, 32, 64, 128; d_I = 64: 16, 32, 64)       */
  double base;          /* 10000 in the published form                                        */
} dsa_rope_t;

/*
 * dsa_indexer_kcache_append with the rotation first: key row r (k_new [n, d_I], bf16 or
 * fp32, pre-RoPE) is rotated at position positions[r] (device int32 [n]) and stored at cache
 * row dst_rows[r] as bf16 or quantised E4M3 + scale, like dsa_indexer_kcache_append.
 */
DSA_API dsa_status_t dsa_indexer_kcache_append_rope(const dsa_kcache_t* kc, const void* k_new, dsa_dtype_t src_dtype,
                                                    const int64_t* dst_rows, const int32_t* positions, int32_t n,
                                                    const dsa_rope_t* rope, void* stream);

/*
 * Queries q_src [T, H_I, d_I] (bf16 or fp32, pre-RoPE, device): every head of token t is
 * rotated at positions[t] (device int32 [T]) and written to q_dst [T, H_I, d_I] as bf16
 * (dst_dtype DSA_BF16) or as E4M3 codes with one scale per token in q_scale [T]
 * (DSA_FP8_E4M3, as dsa_quantize_rows_fp8).  H_I <= 128, d_I 64 or 128; q_src and q_dst
 * 16-byte aligned (DSA_ERR_INVALID_ARG otherwise).  A timed-out copy wait inside the kernel
 * is reported by dsa_check_device_errors.
 */
DSA_API dsa_status_t dsa_rope_queries(const void* q_src, dsa_dtype_t src_dtype, int64_t T, int32_t H_I, int32_t d_I,
                                      const int32_t* positions, const dsa_rope_t* rope, void* q_dst,
                                      dsa_dtype_t dst_dtype, float* q_scale, void* stream);

/*
 * After the selection (what its consumers do with it).
 *
 * dsa_gather_rows: the sparse attention's read of the latent cache at the selected
 * positions (page "Study MLA Indexer", section 数学流, and its 两条 cache 区分 table:
 * c^KV, d_c = 512 per token; "Lightning Indexer 详解" §1):
 *     dst[r, j, :] = src[row_base[r] + idx[r, j], :]   for idx[r, j] >= 0,
 *     dst[r, j, :] = 0                                  for idx[r, j] == -1,
 * with rows of row_bytes bytes (any element type; a multiple of 16, at most 4096).
 *   src       device [src_rows, row_bytes], 16-byte aligned (e.g. the latent cache)
 *   idx       device int32 [rows, top_k] (a selection from prefill / decode)
 *   row_base  device int64 [rows]: cache row of position 0 of each query row's sequence
 *   dst       device [rows, top_k, row_bytes], 16-byte aligned
 * A source row outside [0, src_rows) is zero-filled and recorded as a device fault
 * (dsa_check_device_errors).
 *
 * dsa_selection_rows: out[r, j] = row_base[r] + idx[r, j] (int64), -1 where idx is -1 —
 * global cache rows for consumers that gather from one packed cache by int64 index.
 *
 * dsa_sort_selection: sorts every row of a selection in place by score descending, then
 * position ascending, padding (-1 / -inf) last — the order torch.topk returns
 * (-0.0 counts as, and is returned as, +0.0).  top_k <= 4096 (else DSA_ERR_UNSUPPORTED).
 *
 * All three only enqueue on `stream`.
 */
DSA_API dsa_status_t dsa_gather_rows(const void* src, int64_t src_rows, int32_t row_bytes, const int32_t* idx,
                                     const int64_t* row_base, int64_t rows, int32_t top_k, void* dst, void* stream);
DSA_API dsa_status_t dsa_selection_rows(const int32_t* idx, const int64_t* row_base, int64_t rows, int32_t top_k,
                                        int64_t* out, void* stream);
DSA_API dsa_status_t dsa_sort_selection(int32_t* idx, float* score, int64_t rows, int32_t top_k, void* stream);

/* Workspace bytes a call with this batch needs (scores plus scheduling tables). */
DSA_API size_t dsa_indexer_workspace_bytes(const dsa_query_t* q, const dsa_batch_t* batch, int32_t top_k);

/*
 * Use caller memory (device, 256-byte aligned) as the workspace of `stream` on
 * the current device instead of library allocations; ptr == NULL returns to
 * library-owned memory.  A call whose workspace does not fit returns
 * DSA_ERR_ALLOC.  The memory must stay valid while work using it is pending.
 */
DSA_API dsa_status_t dsa_set_workspace(void* ptr, size_t bytes, void* stream);

/*
 * Synchronises `stream`, then reports and clears any device fault recorded by
 * this library's kernels on that stream: DSA_OK or DSA_ERR_DEVICE_CHECK (the
 * message names the fault).
 */
DSA_API dsa_status_t dsa_check_device_errors(void* stream);

/*
 * Self-test of failure detection: one kernel waits, with the same bounded wait every kernel
 * of this library uses, on a barrier that nothing completes, giving up after limit_cycles SM
 * clock cycles (1 .. 2e9).  The expiry is recorded like any device fault: the next
 * dsa_check_device_errors(stream) returns DSA_ERR_DEVICE_CHECK ("a bounded wait expired")
 * and clears it; the stream stays usable.
 */
DSA_API dsa_status_t dsa_selftest_wait_expiry(int64_t limit_cycles, void* stream);

/*
 * Profiling hook.  Registers three cudaEvent_t for the calling thread (NULL
 * clears them): every later prefill / decode / scores call on this thread
 * records ev_begin right before its logits kernel, ev_mid right after it and
 * ev_end after its last kernel, all on the call's stream.  Timing one step's
 * kernels this way needs no profiler.
 */
DSA_API dsa_status_t dsa_set_profile_events(void* ev_begin, void* ev_mid, void* ev_end);

/* Number of kernels this library has launched from the calling thread so far. */
DSA_API uint64_t dsa_kernel_launch_count(void);

/* Message of the last failed call on this thread ("" if none). */
DSA_API const char* dsa_get_last_error(void);

/* Library version string. */
DSA_API const char* dsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_INDEXER_H */
