// C ABI of the indexer: argument validation, the host-side planner (work items for
// the logits kernel, score-row layout, top-k launch classes), per-stream workspace
// and the launch sequence.  See include/dsa_indexer.h for the contract.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <queue>
#include <string>
#include <utility>
#include <vector>

#include "dsa_indexer.h"
#include "internal.h"

namespace dsa {

int logits_queries_per_item(int H, int D, bool prefill, int max_q_len);

namespace {

thread_local std::string g_last_error;
thread_local cudaEvent_t g_prof[3] = {nullptr, nullptr, nullptr};
thread_local uint64_t g_launches = 0;

dsa_status_t fail(dsa_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

dsa_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(DSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define DSA_CUDA_TRY(expr, what)                 \
  do {                                           \
    cudaError_t e_ = (expr);                     \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

constexpr size_t kAlign = 256;
size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }
int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }
int next_pow2(int64_t x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

// ----------------------------------------------------------------------------- plans

struct Plan {
  // logits
  int tpa = 1, ng = 1;
  std::vector<LogitsItem> items;     // grouped by CTA
  std::vector<int32_t> cta_items;    // [grid + 1]
  // score rows
  std::vector<int64_t> row_off;
  std::vector<int32_t> row_pos;
  int64_t score_elems = 0;
  bool stream_topk = false;          // decode: coarse histograms + the streaming top-k
  // top-k launches: rows grouped by (ept, cluster); short rows separately
  struct TopkClass {
    int ept, cluster;
    int64_t first, count;            // range in topk_rows
  };
  std::vector<int32_t> topk_rows;
  std::vector<TopkClass> classes;
  std::vector<TopkChunk> chunks;     // streaming top-k (then `classes` is empty)
  bool cluster_topk = false;         // decode: `classes` (clusters seeded by the histograms), no chunks
  int64_t rows_first = 0, rows_count = 0;   // row-streaming top-k: range in topk_rows
  int64_t short_first = 0, short_count = 0;
};

// Packs the tables into one host blob whose layout mirrors the device copy.
struct MetaLayout {
  size_t items = 0, cta = 0, row_off = 0, row_pos = 0, topk_rows = 0, chunks = 0, total = 0;
};

// Score workspace: the score rows, then (streaming top-k) the coarse histograms and row
// counters, zeroed together every call, and the candidate buffers laid out like the rows.
struct WsLayout {
  size_t hist = 0, hist1 = 0, ctr = 0, zero_bytes = 0, cand_key = 0, cand_idx = 0, total = 0;
};

WsLayout ws_layout(int64_t score_elems, int64_t rows, bool stream_topk) {
  WsLayout w;
  size_t o = align_up(size_t(score_elems) * sizeof(float));
  if (stream_topk) {
    w.hist = o;
    w.hist1 = w.hist + size_t(rows) * kHistBins * sizeof(uint32_t);
    w.ctr = w.hist1 + size_t(rows) * kTopkBins * sizeof(uint32_t);
    w.zero_bytes = size_t(rows) * (kHistBins + kTopkBins + 4) * sizeof(uint32_t);
    o = align_up(o + w.zero_bytes);
    w.cand_key = o;
    o = align_up(o + size_t(score_elems) * sizeof(uint32_t));
    w.cand_idx = o;
    o = align_up(o + size_t(score_elems) * sizeof(int32_t));
  }
  w.total = o;
  return w;
}

// ----------------------------------------------------------------------------- per-stream context

constexpr int kRing = 4;

struct Ctx {
  int device = 0;
  cudaStream_t stream = nullptr;
  int* d_err = nullptr;            // [2]: code, info
  void* d_meta = nullptr;
  size_t meta_cap = 0;
  float* d_scores = nullptr;
  size_t scores_cap = 0;           // bytes
  void* user_ws = nullptr;         // caller workspace (dsa_set_workspace)
  size_t user_ws_bytes = 0;
  void* h_stage[kRing] = {};
  size_t h_cap[kRing] = {};
  cudaEvent_t h_event[kRing] = {};
  bool h_used[kRing] = {};
  int ring = 0;
  // plan cache: the tables of the last planned batch are still in d_meta
  bool meta_valid = false;
  std::vector<int64_t> plan_key;
  // a CUDA graph captured calls that read d_meta / d_scores: never free or overwrite them
  bool frozen = false;
  std::vector<void*> graveyard;   // device buffers a captured graph may still use
  Plan plan;
  MetaLayout layout;
  void* cur_meta = nullptr;       // tables of the cached plan
  float* cur_scores = nullptr;    // score workspace of the cached plan
  // dsa_indexer_decode_host: device copies of a step's inputs and outputs, in two slots used in
  // turn, filled and read back on the context's own copy streams so that the copies of one
  // step overlap the compute of its neighbours
  struct StepSlot {
    void* d = nullptr;
    size_t cap = 0;
    cudaEvent_t in_done = nullptr;    // the inputs have landed
    cudaEvent_t computed = nullptr;   // the step's kernels are done with the slot's inputs and outputs
    cudaEvent_t out_done = nullptr;   // the outputs have been copied to the host
    bool used = false;
  };
  StepSlot step[2];
  int step_next = 0;
  cudaStream_t copy_in = nullptr, copy_out = nullptr;
};

std::mutex g_mu;
std::map<std::pair<int, cudaStream_t>, Ctx*> g_ctx;

dsa_status_t get_ctx(cudaStream_t stream, Ctx** out) {
  int dev = 0;
  DSA_CUDA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
  std::lock_guard<std::mutex> lk(g_mu);
  auto key = std::make_pair(dev, stream);
  auto it = g_ctx.find(key);
  if (it != g_ctx.end()) {
    *out = it->second;
    return DSA_OK;
  }
  Ctx* c = new Ctx();
  c->device = dev;
  c->stream = stream;
  cudaError_t e = cudaMalloc(&c->d_err, 2 * sizeof(int));
  if (e != cudaSuccess) {
    delete c;
    return fail(DSA_ERR_ALLOC, "cudaMalloc(error flag): %s", cudaGetErrorString(e));
  }
  e = cudaMemset(c->d_err, 0, 2 * sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(error flag)");
  for (int i = 0; i < kRing; ++i) {
    e = cudaEventCreateWithFlags(&c->h_event[i], cudaEventDisableTiming);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventCreate");
  }
  g_ctx[key] = c;
  *out = c;
  return DSA_OK;
}

// Device memory for one call: metadata tables and the score workspace.
dsa_status_t reserve(Ctx* c, size_t meta_bytes, size_t score_bytes, void** meta, float** scores) {
  if (c->user_ws) {
    const size_t need = align_up(meta_bytes) + align_up(score_bytes);
    if (need > c->user_ws_bytes)
      return fail(DSA_ERR_ALLOC, "caller workspace holds %zu bytes, this call needs %zu", c->user_ws_bytes, need);
    *meta = c->user_ws;
    *scores = reinterpret_cast<float*>(static_cast<char*>(c->user_ws) + align_up(meta_bytes));
    return DSA_OK;
  }
  if (c->frozen) {
    // a captured graph reads the current tables: the new plan goes to fresh memory
    if (c->d_meta) c->graveyard.push_back(c->d_meta);
    c->d_meta = nullptr;
    c->meta_cap = 0;
  }
  if ((meta_bytes > c->meta_cap && c->d_meta) || (score_bytes > c->scores_cap && c->d_scores)) {
    // buffers are in use by work already on this stream: wait for it before replacing them
    DSA_CUDA_TRY(cudaStreamSynchronize(c->stream), "cudaStreamSynchronize");
  }
  if (meta_bytes > c->meta_cap) {
    if (c->d_meta) cudaFree(c->d_meta);
    c->d_meta = nullptr;
    c->meta_cap = 0;
    const size_t cap = align_up(std::max(meta_bytes + meta_bytes / 4, size_t(1) << 20));
    cudaError_t e = cudaMalloc(&c->d_meta, cap);
    if (e != cudaSuccess) return fail(DSA_ERR_ALLOC, "cudaMalloc(%zu) for tables: %s", cap, cudaGetErrorString(e));
    c->meta_cap = cap;
  }
  if (score_bytes > c->scores_cap) {
    if (c->d_scores) {
      if (c->frozen)
        c->graveyard.push_back(c->d_scores);
      else
        cudaFree(c->d_scores);
    }
    c->d_scores = nullptr;
    c->scores_cap = 0;
    const size_t cap = align_up(std::max(score_bytes + score_bytes / 8, size_t(1) << 20));
    cudaError_t e = cudaMalloc(reinterpret_cast<void**>(&c->d_scores), cap);
    if (e != cudaSuccess) return fail(DSA_ERR_ALLOC, "cudaMalloc(%zu) for scores: %s", cap, cudaGetErrorString(e));
    c->scores_cap = cap;
  }
  c->frozen = false;
  *meta = c->d_meta;
  *scores = c->d_scores;
  return DSA_OK;
}

// Pinned staging slot for the host tables of one call (reused once its copy is done).
dsa_status_t stage_upload(Ctx* c, const void* host, size_t bytes, void* dev) {
  if (bytes == 0) return DSA_OK;
  const int i = c->ring;
  c->ring = (c->ring + 1) % kRing;
  if (c->h_used[i]) DSA_CUDA_TRY(cudaEventSynchronize(c->h_event[i]), "cudaEventSynchronize");
  if (bytes > c->h_cap[i]) {
    if (c->h_stage[i]) cudaFreeHost(c->h_stage[i]);
    c->h_stage[i] = nullptr;
    c->h_cap[i] = 0;
    const size_t cap = align_up(std::max(bytes + bytes / 4, size_t(1) << 16));
    DSA_CUDA_TRY(cudaHostAlloc(&c->h_stage[i], cap, cudaHostAllocDefault), "cudaHostAlloc");
    c->h_cap[i] = cap;
  }
  std::memcpy(c->h_stage[i], host, bytes);
  DSA_CUDA_TRY(cudaMemcpyAsync(dev, c->h_stage[i], bytes, cudaMemcpyHostToDevice, c->stream), "cudaMemcpyAsync");
  DSA_CUDA_TRY(cudaEventRecord(c->h_event[i], c->stream), "cudaEventRecord");
  c->h_used[i] = true;
  return DSA_OK;
}

// ----------------------------------------------------------------------------- TMA descriptors

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

dsa_status_t get_encoder(EncodeTiledFn* fn) {
  static EncodeTiledFn cached = nullptr;
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  if (!cached) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || p == nullptr)
      return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cached = reinterpret_cast<EncodeTiledFn>(p);
  }
  *fn = cached;
  return DSA_OK;
}

// 2-D row-major [rows, row_elems] tensor, box = [box_rows, 128 bytes], 128-byte swizzle.
dsa_status_t encode_rows(CUtensorMap* map, const void* base, bool fp8, int64_t rows, int row_elems, int box_rows) {
  EncodeTiledFn enc;
  dsa_status_t st = get_encoder(&enc);
  if (st != DSA_OK) return st;
  const int esz = fp8 ? 1 : 2;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_elems), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_elems) * esz};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esz), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return DSA_OK;
}

// ----------------------------------------------------------------------------- validation

struct BatchView {
  int num_seqs = 0;
  std::vector<int32_t> seq_len, q_len;
  std::vector<int64_t> k_base;
  std::vector<int64_t> q_off;   // first packed query row of each sequence
  int64_t total_q = 0;
  int32_t max_seq_len = 0;
  int32_t max_q_len = 0;
  int32_t cmp = 1;              // 1: one cache row per token; m > 1: one per m tokens (compressed)
  // keys a query at position p sees
  int32_t visible(int32_t p) const { return (p + 1) / cmp; }
};

dsa_status_t check_cache(const dsa_kcache_t* kc) {
  if (!kc) return fail(DSA_ERR_INVALID_ARG, "kcache is NULL");
  if (!kc->k) return fail(DSA_ERR_INVALID_ARG, "kcache.k is NULL");
  if (kc->dtype != DSA_BF16 && kc->dtype != DSA_FP8_E4M3)
    return fail(DSA_ERR_INVALID_ARG, "kcache.dtype must be DSA_BF16 or DSA_FP8_E4M3");
  if (kc->dtype == DSA_FP8_E4M3 && !kc->k_scale) return fail(DSA_ERR_INVALID_ARG, "FP8 cache needs k_scale");
  if (kc->d_I != 64 && kc->d_I != 128) return fail(DSA_ERR_UNSUPPORTED, "d_I must be 64 or 128 (got %d)", kc->d_I);
  if (kc->capacity_rows <= 0 || kc->capacity_rows >= (int64_t(1) << 31))
    return fail(DSA_ERR_INVALID_ARG, "capacity_rows must be in [1, 2^31)");
  if (reinterpret_cast<uintptr_t>(kc->k) % 16) return fail(DSA_ERR_INVALID_ARG, "kcache.k must be 16-byte aligned");
  return DSA_OK;
}

dsa_status_t check_batch(const dsa_batch_t* b, const dsa_kcache_t* kc, bool decode, BatchView* v, int32_t cmp = 1) {
  if (!b) return fail(DSA_ERR_INVALID_ARG, "batch is NULL");
  if (cmp < 1) return fail(DSA_ERR_INVALID_ARG, "m must be >= 1");
  v->cmp = cmp;
  if (b->num_seqs < 0) return fail(DSA_ERR_INVALID_ARG, "num_seqs < 0");
  if (b->num_seqs > 0 && !b->seq_lens) return fail(DSA_ERR_INVALID_ARG, "batch.seq_lens is NULL");
  if (decode && b->num_seqs > 0 && !b->q_lens) return fail(DSA_ERR_INVALID_ARG, "decode needs batch.q_lens");
  v->num_seqs = b->num_seqs;
  int64_t row = 0, qoff = 0;
  for (int i = 0; i < b->num_seqs; ++i) {
    const int32_t L = b->seq_lens[i];
    const int32_t n = b->q_lens ? b->q_lens[i] : L;
    if (L < 0 || n < 0 || n > L)
      return fail(DSA_ERR_INVALID_ARG, "sequence %d: need 0 <= q_len (%d) <= seq_len (%d)", i, n, L);
    if (decode && (n < 1 || n > 4))
      return fail(DSA_ERR_INVALID_ARG, "decode: sequence %d has q_len %d, expected 1..4", i, n);
    const int64_t base = b->k_base ? b->k_base[i] : row;
    const int64_t rows = L / cmp;               // cache rows of the sequence
    if (base < 0 || base + rows > kc->capacity_rows)
      return fail(DSA_ERR_INVALID_ARG, "sequence %d: rows [%lld, %lld) exceed the cache capacity %lld", i,
                  static_cast<long long>(base), static_cast<long long>(base + rows),
                  static_cast<long long>(kc->capacity_rows));
    v->seq_len.push_back(L);
    v->q_len.push_back(n);
    v->k_base.push_back(base);
    v->q_off.push_back(qoff);
    qoff += n;
    row += rows;
    v->max_seq_len = std::max(v->max_seq_len, L);
    v->max_q_len = std::max(v->max_q_len, n);
  }
  v->total_q = qoff;
  if (v->total_q >= (int64_t(1) << 31) / 64) return fail(DSA_ERR_INVALID_ARG, "too many queries in one call");
  return DSA_OK;
}

dsa_status_t check_query(const dsa_query_t* q, const dsa_kcache_t* kc) {
  if (!q) return fail(DSA_ERR_INVALID_ARG, "query is NULL");
  if (!q->data) return fail(DSA_ERR_INVALID_ARG, "query.data is NULL");
  if (q->dtype != kc->dtype) return fail(DSA_ERR_INVALID_ARG, "query and cache dtypes differ");
  if (q->d_I != kc->d_I) return fail(DSA_ERR_INVALID_ARG, "query d_I (%d) != cache d_I (%d)", q->d_I, kc->d_I);
  if (q->dtype == DSA_FP8_E4M3 && !q->scale) return fail(DSA_ERR_INVALID_ARG, "FP8 queries need query.scale");
  if (q->H_I <= 0) return fail(DSA_ERR_INVALID_ARG, "H_I must be positive");
  if (reinterpret_cast<uintptr_t>(q->data) % 16) return fail(DSA_ERR_INVALID_ARG, "query.data must be 16-byte aligned");
  return DSA_OK;
}

// ----------------------------------------------------------------------------- planning

void plan_rows(const BatchView& v, bool dense, int64_t ld, Plan* p) {
  p->row_off.resize(v.total_q);
  p->row_pos.resize(v.total_q);
  int64_t off = 0;
  for (int b = 0; b < v.num_seqs; ++b) {
    const int32_t pos0 = v.seq_len[b] - v.q_len[b];
    for (int j = 0; j < v.q_len[b]; ++j) {
      const int64_t r = v.q_off[b] + j;
      const int32_t n = v.visible(pos0 + j);   // the row's keys (-1 below: none)
      p->row_pos[r] = n - 1;
      if (dense) {
        p->row_off[r] = r * ld;
      } else {
        p->row_off[r] = off;
        off += round_up(n, 4);
      }
    }
  }
  p->score_elems = dense ? 0 : off;
}

// Prefill: items of `nt` consecutive queries with their whole causal key range;
// longest-processing-time-first assignment onto `max_ctas` persistent CTAs.
void plan_prefill_items(const BatchView& v, int nt, int groups_per_item, int max_ctas, Plan* p) {
  std::vector<LogitsItem> raw;
  std::vector<int64_t> cost;
  for (int b = 0; b < v.num_seqs; ++b) {
    const int32_t pos0 = v.seq_len[b] - v.q_len[b];
    for (int j = 0; j < v.q_len[b]; j += nt) {
      LogitsItem it{};
      it.k_row0 = v.k_base[b];
      it.q_row0 = static_cast<int32_t>(v.q_off[b] + j);
      it.n_tok = std::min(nt, v.q_len[b] - j);
      it.pos0 = pos0 + j;
      it.kt_begin = 0;
      const int32_t n_last = v.visible(it.pos0 + it.n_tok - 1);   // keys of the item's last query
      if (n_last == 0) continue;                                   // no query of the item sees a key
      it.kt_end = static_cast<int32_t>((n_last + kKeyTile - 1) / kKeyTile);
      it.cmp = v.cmp;
      raw.push_back(it);
      const int groups = (it.n_tok + (nt / groups_per_item) - 1) / (nt / groups_per_item);
      cost.push_back(int64_t(it.kt_end) * (groups + 1));   // +1: the tile load and item overhead
    }
  }
  const int grid = static_cast<int>(std::min<int64_t>(raw.size(), max_ctas));
  std::vector<int> order(raw.size());
  for (size_t i = 0; i < order.size(); ++i) order[i] = static_cast<int>(i);
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cost[a] > cost[b]; });
  using Load = std::pair<int64_t, int>;
  std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
  for (int c = 0; c < grid; ++c) heap.push({0, c});
  std::vector<std::vector<int>> per(grid);
  for (int i : order) {
    Load l = heap.top();
    heap.pop();
    per[l.second].push_back(i);
    heap.push({l.first + cost[i], l.second});
  }
  p->items.clear();
  p->cta_items.assign(1, 0);
  for (int c = 0; c < grid; ++c) {
    for (int i : per[c]) p->items.push_back(raw[i]);
    p->cta_items.push_back(static_cast<int32_t>(p->items.size()));
  }
}

// Decode: all queries of a sequence in one group; the concatenated key tiles of
// all sequences are cut into `max_ctas` nearly equal contiguous ranges.
void plan_decode_items(const BatchView& v, int max_ctas, Plan* p) {
  int64_t total = 0;
  std::vector<int32_t> tiles(v.num_seqs);
  for (int b = 0; b < v.num_seqs; ++b) {
    tiles[b] = (v.visible(v.seq_len[b] - 1) + kKeyTile - 1) / kKeyTile;   // the last query sees the most
    if (v.q_len[b] == 0) tiles[b] = 0;
    total += tiles[b];
  }
  p->items.clear();
  p->cta_items.assign(1, 0);
  if (total == 0) return;
  const int grid = static_cast<int>(std::min<int64_t>(total, max_ctas));
  int b = 0;
  int32_t t = 0;   // next tile of sequence b
  for (int c = 0; c < grid; ++c) {
    int64_t quota = total * (c + 1) / grid - total * c / grid;
    while (quota > 0) {
      while (b < v.num_seqs && t >= tiles[b]) {
        ++b;
        t = 0;
      }
      if (b >= v.num_seqs) break;
      const int32_t take = static_cast<int32_t>(std::min<int64_t>(quota, tiles[b] - t));
      LogitsItem it{};
      it.k_row0 = v.k_base[b];
      it.q_row0 = static_cast<int32_t>(v.q_off[b]);
      it.n_tok = v.q_len[b];
      it.pos0 = v.seq_len[b] - v.q_len[b];
      it.kt_begin = t;
      it.kt_end = t + take;
      it.cmp = v.cmp;
      p->items.push_back(it);
      t += take;
      quota -= take;
    }
    p->cta_items.push_back(static_cast<int32_t>(p->items.size()));
  }
}

dsa_status_t plan_topk(const BatchView& v, int top_k, int sms, Plan* p, int max_cs = 8) {
  std::vector<int32_t> shorts, longs;
  for (int64_t r = 0; r < v.total_q; ++r) (p->row_pos[r] + 1 <= top_k ? shorts : longs).push_back(static_cast<int32_t>(r));
  const int64_t n_long = static_cast<int64_t>(longs.size());
  int cs_par = 1;
  if (n_long > 0 && n_long < 2 * sms) cs_par = std::min(max_cs, next_pow2((2 * sms + n_long - 1) / n_long));
  std::map<std::pair<int, int>, std::vector<int32_t>> cls;
  for (int32_t r : longs) {
    const int64_t n = int64_t(p->row_pos[r]) + 1;
    int cs = std::max(cs_par, next_pow2((n + 32 * kTopkThreads - 1) / (32 * kTopkThreads)));
    if (cs > 8) return fail(DSA_ERR_UNSUPPORTED, "a row of %lld keys exceeds the top-k kernel's limit", (long long)n);
    int ept = next_pow2((n + int64_t(cs) * kTopkThreads - 1) / (int64_t(cs) * kTopkThreads));
    ept = std::max(4, ept);
    cls[{ept, cs}].push_back(r);
  }
  p->topk_rows.clear();
  p->classes.clear();
  p->short_first = 0;
  p->short_count = static_cast<int64_t>(shorts.size());
  p->topk_rows.insert(p->topk_rows.end(), shorts.begin(), shorts.end());
  for (auto& kv : cls) {
    auto& rows = kv.second;
    std::stable_sort(rows.begin(), rows.end(),
                     [&](int32_t a, int32_t b) { return p->row_pos[a] > p->row_pos[b]; });   // longest first
    Plan::TopkClass c{kv.first.first, kv.first.second, static_cast<int64_t>(p->topk_rows.size()),
                      static_cast<int64_t>(rows.size())};
    p->topk_rows.insert(p->topk_rows.end(), rows.begin(), rows.end());
    p->classes.push_back(c);
  }
  return DSA_OK;
}

// Decode rows: chunks of kStreamChunk keys for the streaming top-k (no length limit).
// Decode rows (the coarse histograms given).  A bf16 batch whose rows are at most 32768
// keys long takes one cluster per row (the cluster kernel seeded by the histogram: no
// global counters, fence or ticket between the CTAs of a row); FP8 batches and longer rows
// stream 4096-key chunks (the FP8 histogram pass needs those chunks anyway, and 32 keys a
// thread leave the clusters slower there).
void plan_topk_stream(const BatchView& v, int top_k, int sms, bool fp8, Plan* p) {
  p->topk_rows.clear();
  p->classes.clear();
  p->chunks.clear();
  int64_t longest = 0;
  for (int64_t r = 0; r < v.total_q; ++r) longest = std::max(longest, int64_t(p->row_pos[r]) + 1);
  // clusters of at most 4 CTAs: they find room on the SMs the logits kernel frees as it drains
  // (the step overlaps better: 55.5-56.6 us against 60.0 us with clusters of 8), and rows up
  // to 4 x 16 x 512 keys keep 16 keys a thread
  constexpr int kMaxCs = 4;
  p->cluster_topk = !fp8 && longest <= int64_t(kMaxCs) * 16 * kTopkThreads &&
                    plan_topk(v, top_k, sms, p, kMaxCs) == DSA_OK;
  if (p->cluster_topk) return;
  p->topk_rows.clear();
  p->classes.clear();
  for (int64_t r = 0; r < v.total_q; ++r) {
    const int32_t n = p->row_pos[r] + 1;
    if (n <= top_k) {
      p->topk_rows.push_back(static_cast<int32_t>(r));
      continue;
    }
    const int32_t nch = (n + kStreamChunk - 1) / kStreamChunk;
    for (int32_t c = 0; c < nch; ++c)
      p->chunks.push_back(TopkChunk{static_cast<int32_t>(r), c * kStreamChunk, std::min(n, (c + 1) * kStreamChunk), nch});
  }
  p->short_first = 0;
  p->short_count = static_cast<int64_t>(p->topk_rows.size());
}

// Prefill rows: one CTA each in the row-streaming top-k, longest rows first.
void plan_topk_rows(const BatchView& v, int top_k, Plan* p) {
  std::vector<int32_t> longs;
  p->topk_rows.clear();
  p->classes.clear();
  p->chunks.clear();
  for (int64_t r = 0; r < v.total_q; ++r)
    (p->row_pos[r] + 1 <= top_k ? p->topk_rows : longs).push_back(static_cast<int32_t>(r));
  p->short_first = 0;
  p->short_count = static_cast<int64_t>(p->topk_rows.size());
  std::stable_sort(longs.begin(), longs.end(), [&](int32_t x, int32_t y) { return p->row_pos[x] > p->row_pos[y]; });
  p->rows_first = p->short_count;
  p->rows_count = static_cast<int64_t>(longs.size());
  p->topk_rows.insert(p->topk_rows.end(), longs.begin(), longs.end());
}

MetaLayout layout_of(const Plan& p) {
  MetaLayout m;
  size_t o = 0;
  m.items = o;     o = align_up(o + p.items.size() * sizeof(LogitsItem));
  m.cta = o;       o = align_up(o + p.cta_items.size() * sizeof(int32_t));
  m.row_off = o;   o = align_up(o + p.row_off.size() * sizeof(int64_t));
  m.row_pos = o;   o = align_up(o + p.row_pos.size() * sizeof(int32_t));
  m.topk_rows = o; o = align_up(o + p.topk_rows.size() * sizeof(int32_t));
  m.chunks = o;    o = align_up(o + p.chunks.size() * sizeof(TopkChunk));
  m.total = o;
  return m;
}

std::vector<uint8_t> pack(const Plan& p, const MetaLayout& m) {
  std::vector<uint8_t> blob(m.total, 0);
  auto put = [&](size_t off, const void* src, size_t n) { if (n) std::memcpy(blob.data() + off, src, n); };
  put(m.items, p.items.data(), p.items.size() * sizeof(LogitsItem));
  put(m.cta, p.cta_items.data(), p.cta_items.size() * sizeof(int32_t));
  put(m.row_off, p.row_off.data(), p.row_off.size() * sizeof(int64_t));
  put(m.row_pos, p.row_pos.data(), p.row_pos.size() * sizeof(int32_t));
  put(m.topk_rows, p.topk_rows.data(), p.topk_rows.size() * sizeof(int32_t));
  put(m.chunks, p.chunks.data(), p.chunks.size() * sizeof(TopkChunk));
  return blob;
}

int g_sms = 0;

// ----------------------------------------------------------------------------- the indexer call

enum class Mode { Prefill, Decode, Scores };

dsa_status_t run_indexer(Mode mode, const dsa_query_t* q, const dsa_kcache_t* kc, const float* w,
                         const dsa_batch_t* batch, int32_t top_k, int32_t* out_idx, float* out_score,
                         float* dense_out, int64_t ld, void* stream_v, int32_t cmp = 1) {
  g_last_error.clear();
  dsa_status_t st = check_cache(kc);
  if (st != DSA_OK) return st;
  BatchView v;
  if ((st = check_batch(batch, kc, mode == Mode::Decode, &v, cmp)) != DSA_OK) return st;
  if (cmp > 1 && (mode == Mode::Scores || !out_score))
    return fail(DSA_ERR_INVALID_ARG, "a compressed cache needs the scores and the selection");
  if (mode != Mode::Scores && top_k < 1) return fail(DSA_ERR_INVALID_ARG, "top_k must be >= 1");
  if (v.total_q == 0) return DSA_OK;          // nothing to score: no pointer is touched
  if ((st = check_query(q, kc)) != DSA_OK) return st;
  if (!w) return fail(DSA_ERR_INVALID_ARG, "w is NULL");
  const bool fp8 = kc->dtype == DSA_FP8_E4M3;
  if (mode == Mode::Scores) {
    if (!dense_out) return fail(DSA_ERR_INVALID_ARG, "out_scores is NULL");
    if (ld < v.max_seq_len || ld % 4) return fail(DSA_ERR_INVALID_ARG, "ld must be >= max(seq_lens) and a multiple of 4");
  } else if (!out_idx) {
    return fail(DSA_ERR_INVALID_ARG, "out_idx is NULL");
  } else if (!out_score && v.max_seq_len > top_k) {
    return fail(DSA_ERR_INVALID_ARG, "out_score is NULL while a sequence is longer than top_k");
  }
  // short-sequence bypass: no scores wanted and every row keeps its whole history
  const bool bypass = mode != Mode::Scores && !out_score;
  const bool decode_sched = mode == Mode::Decode || (mode == Mode::Scores && v.max_q_len <= 4 &&
                                                     q->H_I == 64 && kc->d_I == 128);
  const int H = q->H_I, D = kc->d_I;
  int tpa, ng;
  if (decode_sched) {
    tpa = logits_queries_per_item(H, D, false, v.max_q_len);
    ng = 1;
  } else if (H == 4) {
    tpa = 64;
    ng = 1;
  } else {
    tpa = 4;
    ng = 2;
  }
  const bool prefill_items = !decode_sched && H != 4;
  if (!logits_config_supported(H, D, fp8, tpa, ng, prefill_items))
    return fail(DSA_ERR_UNSUPPORTED, "no %s kernel for H_I=%d, d_I=%d, dtype=%s", decode_sched ? "decode" : "prefill",
                H, D, fp8 ? "fp8" : "bf16");

  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  Ctx* c = nullptr;
  if ((st = get_ctx(stream, &c)) != DSA_OK) return st;
  if (g_sms == 0) g_sms = num_sms(c->device);

  // The plan depends only on the batch description, so a repeated batch reuses the
  // tables already on the device (decode loops, graph capture).
  std::vector<int64_t> key = {static_cast<int64_t>(mode), H, D, fp8, top_k, ld, v.num_seqs,
                              reinterpret_cast<int64_t>(c->user_ws), v.cmp};
  for (int b = 0; b < v.num_seqs; ++b) {
    key.push_back(v.seq_len[b]);
    key.push_back(v.q_len[b]);
    key.push_back(v.k_base[b]);
  }
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  DSA_CUDA_TRY(cudaStreamIsCapturing(stream, &cap), "cudaStreamIsCapturing");
  const bool capturing = cap != cudaStreamCaptureStatusNone;
  if (!(c->meta_valid && key == c->plan_key)) {
    if (capturing)
      return fail(DSA_ERR_UNSUPPORTED, "a call can be captured in a CUDA graph only after an uncaptured call "
                                       "with the same batch on the same stream");
    Plan np;
    np.tpa = tpa;
    np.ng = ng;
    plan_rows(v, mode == Mode::Scores, ld, &np);
    if (decode_sched)
      plan_decode_items(v, g_sms, &np);
    else
      plan_prefill_items(v, tpa * ng, ng, g_sms, &np);
    // decode: the logits epilogue bins each row and the top-k streams it (rows are few and long)
    np.stream_topk = mode == Mode::Decode;
    if (np.stream_topk)
      plan_topk_stream(v, top_k, g_sms, fp8, &np);
    else if (mode == Mode::Prefill)
      plan_topk_rows(v, top_k, &np);
    const MetaLayout nm = layout_of(np);
    const std::vector<uint8_t> blob = pack(np, nm);
    c->meta_valid = false;
    void* dm = nullptr;
    float* ds = nullptr;
    const size_t ws_bytes = ws_layout(np.score_elems, v.total_q, np.stream_topk).total;
    if ((st = reserve(c, nm.total, ws_bytes, &dm, &ds)) != DSA_OK) return st;
    if ((st = stage_upload(c, blob.data(), blob.size(), dm)) != DSA_OK) return st;
    if (np.stream_topk) {
      // the histograms and row counters start clear; from then on the top-k kernels clear
      // each row's after use, so a repeated call needs no memset between its launches
      const WsLayout nw = ws_layout(np.score_elems, v.total_q, true);
      DSA_CUDA_TRY(cudaMemsetAsync(reinterpret_cast<char*>(ds) + nw.hist, 0, nw.zero_bytes, stream), "cudaMemsetAsync");
    }
    c->plan = std::move(np);
    c->layout = nm;
    c->plan_key = key;
    c->meta_valid = true;
    c->cur_meta = dm;
    c->cur_scores = ds;
  }
  if (capturing) c->frozen = true;
  const Plan& p = c->plan;
  const MetaLayout& m = c->layout;
  float* d_scores = c->cur_scores;
  char* mb = static_cast<char*>(c->cur_meta);
  const WsLayout wl = ws_layout(p.score_elems, v.total_q, p.stream_topk);
  char* wsb = reinterpret_cast<char*>(d_scores);
  if (bypass) {
    // every row holds at most top_k keys: the selection is its whole history, no scoring
    TopkArgs s{};
    s.row_pos = reinterpret_cast<const int32_t*>(mb + m.row_pos);
    s.top_k = top_k;
    s.out_idx = out_idx;
    s.rows = reinterpret_cast<const int32_t*>(mb + m.topk_rows) + p.short_first;
    s.n_rows = static_cast<int32_t>(p.short_count);
    DSA_CUDA_TRY(launch_topk_short(s, stream), "top-k (short rows) launch");
    ++g_launches;
    return DSA_OK;
  }
  uint32_t* d_hist = p.stream_topk ? reinterpret_cast<uint32_t*>(wsb + wl.hist) : nullptr;
  // from the scoring launch on, a failed enqueue leaves histograms uncleared: plan afresh next time
  struct Replan {
    Ctx* c;
    bool armed;
    ~Replan() { if (armed) c->meta_valid = false; }
  } replan{c, d_hist != nullptr};

  CUtensorMap tk, tq;
  if ((st = encode_rows(&tk, kc->k, fp8, kc->capacity_rows, D, kKeyTile)) != DSA_OK) return st;
  if ((st = encode_rows(&tq, q->data, fp8, v.total_q * H, D, tpa * H)) != DSA_OK) return st;

  LogitsArgs la{};
  la.items = reinterpret_cast<const LogitsItem*>(mb + m.items);
  la.cta_items = reinterpret_cast<const int32_t*>(mb + m.cta);
  la.row_off = reinterpret_cast<const int64_t*>(mb + m.row_off);
  la.w = w;
  la.q_scale = fp8 ? q->scale : nullptr;
  la.k_scale = fp8 ? kc->k_scale : nullptr;
  la.k_capacity = kc->capacity_rows;
  la.scores = mode == Mode::Scores ? dense_out : d_scores;
  la.row_hist = d_hist;
  la.inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  la.err = c->d_err;
  LogitsLaunch L{H, D, fp8, tpa, ng, static_cast<int>(p.cta_items.size()) - 1, stream, prefill_items};
  // inside a capture the events must become event-record nodes of the graph
  const unsigned ev_flags = capturing ? cudaEventRecordExternal : cudaEventRecordDefault;
  if (g_prof[0]) DSA_CUDA_TRY(cudaEventRecordWithFlags(g_prof[0], stream, ev_flags), "cudaEventRecord");
  DSA_CUDA_TRY(launch_logits(L, tk, tq, la), "logits kernel launch");
  g_launches += L.grid > 0;
  if (g_prof[1]) DSA_CUDA_TRY(cudaEventRecordWithFlags(g_prof[1], stream, ev_flags), "cudaEventRecord");
  if (mode == Mode::Scores) {
    if (g_prof[2]) DSA_CUDA_TRY(cudaEventRecordWithFlags(g_prof[2], stream, ev_flags), "cudaEventRecord");
    return DSA_OK;
  }

  TopkArgs ta{};
  ta.scores = d_scores;
  ta.row_off = la.row_off;
  ta.row_pos = reinterpret_cast<const int32_t*>(mb + m.row_pos);
  ta.top_k = top_k;
  ta.out_idx = out_idx;
  ta.out_score = out_score;
  ta.err = c->d_err;
  const int32_t* rows = reinterpret_cast<const int32_t*>(mb + m.topk_rows);
  if (p.short_count) {
    TopkArgs s = ta;
    s.rows = rows + p.short_first;
    s.n_rows = static_cast<int32_t>(p.short_count);
    s.row_hist = d_hist;                      // decode: cleared for the next call
    DSA_CUDA_TRY(launch_topk_short(s, stream), "top-k (short rows) launch");
    ++g_launches;
  }
  if (!p.chunks.empty()) {
    TopkArgs s = ta;
    s.chunks = reinterpret_cast<const TopkChunk*>(mb + m.chunks);
    s.n_chunks = static_cast<int32_t>(p.chunks.size());
    s.row_hist = d_hist;
    s.row_hist1 = reinterpret_cast<uint32_t*>(wsb + wl.hist1);
    s.row_ctr = reinterpret_cast<uint32_t*>(wsb + wl.ctr);
    s.cand_key = reinterpret_cast<uint32_t*>(wsb + wl.cand_key);
    s.cand_idx = reinterpret_cast<int32_t*>(wsb + wl.cand_idx);
    if (!logits_bins_rows(H, D, fp8, tpa, ng, prefill_items)) {
      // this logits configuration leaves the coarse histograms to a pass over the score rows
      DSA_CUDA_TRY(launch_row_hist(s, stream), "row histogram launch");
      ++g_launches;
    }
    DSA_CUDA_TRY(launch_topk_stream(s, stream), "top-k (streaming) launch");
    ++g_launches;
  }
  for (const auto& cl : p.classes) {
    TopkArgs s = ta;
    s.rows = rows + cl.first;
    s.n_rows = static_cast<int32_t>(cl.count);
    s.row_hist = p.stream_topk ? d_hist : nullptr;   // decode: the clusters start from the coarse histogram
    DSA_CUDA_TRY(launch_topk(s, cl.ept, cl.cluster, stream), "top-k launch");
    ++g_launches;
  }
  if (p.rows_count) {
    TopkArgs s = ta;
    s.rows = rows + p.rows_first;
    s.n_rows = static_cast<int32_t>(p.rows_count);
    DSA_CUDA_TRY(launch_topk_rows(s, stream), "top-k (row-streaming) launch");
    ++g_launches;
  }
  if (g_prof[2]) DSA_CUDA_TRY(cudaEventRecordWithFlags(g_prof[2], stream, ev_flags), "cudaEventRecord");
  replan.armed = false;
  return DSA_OK;
}

}  // namespace

// RoPE parameters for the kernels, with the pair frequencies base^(-2i / rope_dim) in fp64
RopeParams rope_params(const dsa_rope_t& r) {
  RopeParams p{};
  p.rope_dim = r.rope_dim;
  p.interleaved = r.interleaved;
  p.base = r.base;
  for (int i = 0; i < kRopeMaxPairs; ++i)
    p.inv_freq[i] = (r.rope_dim > 0 && r.base > 0.0) ? std::pow(r.base, -2.0 * i / r.rope_dim) : 0.0;
  return p;
}

int num_sms(int device) {
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || n <= 0) n = 148;
  return n;
}

}  // namespace dsa

// ============================================================================= C ABI

using namespace dsa;

extern "C" {

dsa_status_t dsa_indexer_kcache_append(const dsa_kcache_t* kc, const void* k_new, dsa_dtype_t src_dtype,
                                       const int64_t* dst_rows, int32_t n, void* stream_v) {
  g_last_error.clear();
  dsa_status_t st = check_cache(kc);
  if (st != DSA_OK) return st;
  if (n < 0) return fail(DSA_ERR_INVALID_ARG, "n < 0");
  if (n == 0) return DSA_OK;
  if (!k_new || !dst_rows) return fail(DSA_ERR_INVALID_ARG, "k_new / dst_rows is NULL");
  if (src_dtype != DSA_BF16 && src_dtype != DSA_F32) return fail(DSA_ERR_INVALID_ARG, "src_dtype must be DSA_BF16 or DSA_F32");
  if (reinterpret_cast<uintptr_t>(k_new) % 16) return fail(DSA_ERR_INVALID_ARG, "k_new must be 16-byte aligned");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  Ctx* c = nullptr;
  if ((st = get_ctx(stream, &c)) != DSA_OK) return st;
  const int f32 = src_dtype == DSA_F32;
  cudaError_t e;
  if (kc->dtype == DSA_FP8_E4M3)
    e = launch_quantize_rows_fp8(k_new, f32, n, kc->d_I, static_cast<uint8_t*>(kc->k), kc->k_scale, dst_rows,
                                 kc->capacity_rows, c->d_err, stream);
  else
    e = launch_append_bf16(k_new, f32, n, kc->d_I, static_cast<uint16_t*>(kc->k), dst_rows, kc->capacity_rows,
                           c->d_err, stream);
  if (e != cudaSuccess) return cuda_fail(e, "append kernel launch");
  ++g_launches;
  return DSA_OK;
}

dsa_status_t dsa_quantize_rows_fp8(const void* src, dsa_dtype_t src_dtype, int64_t rows, int32_t row_len,
                                   uint8_t* dst, float* scale, void* stream_v) {
  g_last_error.clear();
  if (rows < 0) return fail(DSA_ERR_INVALID_ARG, "rows < 0");
  if (row_len <= 0 || row_len % 16) return fail(DSA_ERR_INVALID_ARG, "row_len must be a positive multiple of 16");
  if (rows == 0) return DSA_OK;
  if (!src || !dst || !scale) return fail(DSA_ERR_INVALID_ARG, "src / dst / scale is NULL");
  if (src_dtype != DSA_BF16 && src_dtype != DSA_F32) return fail(DSA_ERR_INVALID_ARG, "src_dtype must be DSA_BF16 or DSA_F32");
  if (reinterpret_cast<uintptr_t>(src) % 16 || reinterpret_cast<uintptr_t>(dst) % 16)
    return fail(DSA_ERR_INVALID_ARG, "src and dst must be 16-byte aligned");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  Ctx* c = nullptr;
  dsa_status_t st = get_ctx(stream, &c);
  if (st != DSA_OK) return st;
  cudaError_t e = launch_quantize_rows_fp8(src, src_dtype == DSA_F32, rows, row_len, dst, scale, nullptr, rows,
                                           c->d_err, stream);
  if (e != cudaSuccess) return cuda_fail(e, "quantise kernel launch");
  ++g_launches;
  return DSA_OK;
}

dsa_status_t dsa_indexer_prefill(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w,
                                 const dsa_batch_t* batch, int32_t top_k, int32_t* out_idx, float* out_score,
                                 void* stream) {
  return run_indexer(Mode::Prefill, q, kc, w, batch, top_k, out_idx, out_score, nullptr, 0, stream);
}

dsa_status_t dsa_indexer_decode(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w,
                                const dsa_batch_t* batch, int32_t top_k, int32_t* out_idx, float* out_score,
                                void* stream) {
  return run_indexer(Mode::Decode, q, kc, w, batch, top_k, out_idx, out_score, nullptr, 0, stream);
}

// Copy streams and slot events of the host step, created on first use.
static dsa_status_t ensure_step_streams(Ctx* c) {
  if (c->copy_in) return DSA_OK;
  DSA_CUDA_TRY(cudaStreamCreateWithFlags(&c->copy_in, cudaStreamNonBlocking), "cudaStreamCreate(copy in)");
  DSA_CUDA_TRY(cudaStreamCreateWithFlags(&c->copy_out, cudaStreamNonBlocking), "cudaStreamCreate(copy out)");
  for (auto& sl : c->step) {
    DSA_CUDA_TRY(cudaEventCreateWithFlags(&sl.in_done, cudaEventDisableTiming), "cudaEventCreate");
    DSA_CUDA_TRY(cudaEventCreateWithFlags(&sl.computed, cudaEventDisableTiming), "cudaEventCreate");
    DSA_CUDA_TRY(cudaEventCreateWithFlags(&sl.out_done, cudaEventDisableTiming), "cudaEventCreate");
  }
  return DSA_OK;
}

// The host step (decode, or prefill with the same copies).  Slot i % 2 holds step i's inputs
// and outputs:
//   copy_in : [wait computed(i-2)] H2D inputs            [record in_done(i)]
//   stream  : [wait in_done(i), out_done(i-2)] append, quantise, decode   [record computed(i)]
//   copy_out: [wait computed(i)] D2H outputs             [record out_done(i), done_event]
// With join, `stream` then waits for out_done(i), so the host outputs are complete when the
// stream is (the uploads of the next call still overlap this call's compute); without, the
// caller waits on done_event.
static dsa_status_t host_step(bool prefill, const dsa_query_t* q, const dsa_kcache_t* kc, const float* w_host,
                              const void* k_new_host, dsa_dtype_t k_new_dtype, const int64_t* dst_rows_host,
                              int32_t n_new, const dsa_batch_t* batch, int32_t top_k, int32_t* out_idx_host,
                              float* out_score_host, void* stream_v, cudaEvent_t done_event, bool join) {
  const char* name = prefill ? "dsa_indexer_prefill_host" : "dsa_indexer_decode_host";
  g_last_error.clear();
  dsa_status_t st = check_cache(kc);
  if (st != DSA_OK) return st;
  if (!q || !batch || !w_host || !out_idx_host || !out_score_host || !q->data)
    return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (n_new < 0 || (n_new > 0 && (!k_new_host || !dst_rows_host)))
    return fail(DSA_ERR_INVALID_ARG, "n_new < 0, or k_new_host / dst_rows_host is NULL");
  if (k_new_dtype != DSA_BF16 && k_new_dtype != DSA_F32) return fail(DSA_ERR_INVALID_ARG, "k_new_dtype must be DSA_BF16 or DSA_F32");
  if (q->dtype != DSA_BF16 && q->dtype != DSA_FP8_E4M3) return fail(DSA_ERR_INVALID_ARG, "q->dtype must be DSA_BF16 or DSA_FP8_E4M3");
  if (q->dtype == DSA_FP8_E4M3 && !q->scale) return fail(DSA_ERR_INVALID_ARG, "FP8 queries need q->scale");
  // bf16 queries against an FP8 cache are quantised on the device after the upload
  const bool quantise_q = q->dtype == DSA_BF16 && kc->dtype == DSA_FP8_E4M3;
  if (q->H_I <= 0 || q->d_I <= 0 || top_k <= 0) return fail(DSA_ERR_INVALID_ARG, "H_I, d_I and top_k must be positive");
  if (batch->num_seqs < 0 || (batch->num_seqs > 0 && (!batch->seq_lens || (!prefill && !batch->q_lens))))
    return fail(DSA_ERR_INVALID_ARG, prefill ? "prefill needs batch.seq_lens" : "decode needs batch.seq_lens and batch.q_lens");
  int64_t T = 0;
  for (int i = 0; i < batch->num_seqs; ++i) T += batch->q_lens ? batch->q_lens[i] : batch->seq_lens[i];
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  DSA_CUDA_TRY(cudaStreamIsCapturing(stream, &cap), "cudaStreamIsCapturing");
  if (cap != cudaStreamCaptureStatusNone) return fail(DSA_ERR_UNSUPPORTED, "%s cannot be captured", name);
  Ctx* c = nullptr;
  if ((st = get_ctx(stream, &c)) != DSA_OK) return st;
  if ((st = ensure_step_streams(c)) != DSA_OK) return st;

  // slot layout: [k_new | dst_rows | q | q_scale | w | out_idx | out_score | q8 | q8_scale],
  // 256-byte aligned parts (the last two only when bf16 queries meet an FP8 cache)
  const size_t esz_k = k_new_dtype == DSA_F32 ? 4 : 2, esz_q = q->dtype == DSA_FP8_E4M3 ? 1 : 2;
  const size_t q_elems = size_t(T) * q->H_I * q->d_I;
  const size_t b_k = size_t(n_new) * kc->d_I * esz_k, b_rows = size_t(n_new) * sizeof(int64_t);
  const size_t b_q = q_elems * esz_q, b_qs = q->dtype == DSA_FP8_E4M3 ? size_t(T) * 4 : 0;
  const size_t b_w = size_t(T) * q->H_I * 4, b_out = size_t(T) * top_k * 4;
  const size_t o_rows = align_up(b_k), o_q = o_rows + align_up(b_rows), o_qs = o_q + align_up(b_q);
  const size_t o_w = o_qs + align_up(b_qs), o_oi = o_w + align_up(b_w), o_os = o_oi + align_up(b_out);
  const size_t o_q8 = o_os + align_up(b_out), o_q8s = o_q8 + (quantise_q ? align_up(q_elems) : 0);
  const size_t total = o_q8s + (quantise_q ? align_up(size_t(T) * 4) : 0);
  Ctx::StepSlot& sl = c->step[c->step_next];
  if (total > sl.cap) {
    if (sl.d) {
      DSA_CUDA_TRY(cudaEventSynchronize(sl.out_done), "cudaEventSynchronize");   // its last step is over
      DSA_CUDA_TRY(cudaFree(sl.d), "cudaFree");
      sl.d = nullptr;
      sl.cap = 0;
    }
    DSA_CUDA_TRY(cudaMalloc(&sl.d, total), "cudaMalloc(host-step staging)");
    sl.cap = total;
  }
  char* d = static_cast<char*>(sl.d);
  if (sl.used) DSA_CUDA_TRY(cudaStreamWaitEvent(c->copy_in, sl.computed, 0), "cudaStreamWaitEvent");
  auto h2d = [&](size_t off, const void* src, size_t bytes) -> cudaError_t {
    return bytes ? cudaMemcpyAsync(d + off, src, bytes, cudaMemcpyHostToDevice, c->copy_in) : cudaSuccess;
  };
  DSA_CUDA_TRY(h2d(0, k_new_host, b_k), "cudaMemcpyAsync(k_new)");
  DSA_CUDA_TRY(h2d(o_rows, dst_rows_host, b_rows), "cudaMemcpyAsync(dst_rows)");
  DSA_CUDA_TRY(h2d(o_q, q->data, b_q), "cudaMemcpyAsync(q)");
  DSA_CUDA_TRY(h2d(o_qs, q->scale, b_qs), "cudaMemcpyAsync(q_scale)");
  DSA_CUDA_TRY(h2d(o_w, w_host, b_w), "cudaMemcpyAsync(w)");
  DSA_CUDA_TRY(cudaEventRecord(sl.in_done, c->copy_in), "cudaEventRecord");
  DSA_CUDA_TRY(cudaStreamWaitEvent(stream, sl.in_done, 0), "cudaStreamWaitEvent");
  if (sl.used) DSA_CUDA_TRY(cudaStreamWaitEvent(stream, sl.out_done, 0), "cudaStreamWaitEvent");
  sl.used = true;
  c->step_next ^= 1;
  if (n_new > 0 &&
      (st = dsa_indexer_kcache_append(kc, d, k_new_dtype, reinterpret_cast<const int64_t*>(d + o_rows), n_new,
                                      stream_v)) != DSA_OK)
    return st;
  dsa_query_t qd = *q;
  qd.data = d + o_q;
  qd.scale = b_qs ? reinterpret_cast<const float*>(d + o_qs) : nullptr;
  if (quantise_q && T > 0) {
    if ((st = dsa_quantize_rows_fp8(d + o_q, DSA_BF16, T, q->H_I * q->d_I, reinterpret_cast<uint8_t*>(d + o_q8),
                                    reinterpret_cast<float*>(d + o_q8s), stream_v)) != DSA_OK)
      return st;
    qd.data = d + o_q8;
    qd.scale = reinterpret_cast<const float*>(d + o_q8s);
    qd.dtype = DSA_FP8_E4M3;
  }
  int32_t* oi = reinterpret_cast<int32_t*>(d + o_oi);
  float* os = reinterpret_cast<float*>(d + o_os);
  const float* wd = reinterpret_cast<const float*>(d + o_w);
  if ((st = prefill ? dsa_indexer_prefill(&qd, kc, wd, batch, top_k, oi, os, stream_v)
                    : dsa_indexer_decode(&qd, kc, wd, batch, top_k, oi, os, stream_v)) != DSA_OK)
    return st;
  DSA_CUDA_TRY(cudaEventRecord(sl.computed, stream), "cudaEventRecord");
  DSA_CUDA_TRY(cudaStreamWaitEvent(c->copy_out, sl.computed, 0), "cudaStreamWaitEvent");
  if (b_out) {
    DSA_CUDA_TRY(cudaMemcpyAsync(out_idx_host, oi, b_out, cudaMemcpyDeviceToHost, c->copy_out), "cudaMemcpyAsync(out_idx)");
    DSA_CUDA_TRY(cudaMemcpyAsync(out_score_host, os, b_out, cudaMemcpyDeviceToHost, c->copy_out),
                 "cudaMemcpyAsync(out_score)");
  }
  DSA_CUDA_TRY(cudaEventRecord(sl.out_done, c->copy_out), "cudaEventRecord");
  if (done_event) DSA_CUDA_TRY(cudaEventRecord(done_event, c->copy_out), "cudaEventRecord(done_event)");
  if (join) DSA_CUDA_TRY(cudaStreamWaitEvent(stream, sl.out_done, 0), "cudaStreamWaitEvent");
  return DSA_OK;
}

dsa_status_t dsa_indexer_decode_host(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w_host,
                                     const void* k_new_host, dsa_dtype_t k_new_dtype, const int64_t* dst_rows_host,
                                     int32_t n_new, const dsa_batch_t* batch, int32_t top_k, int32_t* out_idx_host,
                                     float* out_score_host, void* stream_v) {
  return host_step(false, q, kc, w_host, k_new_host, k_new_dtype, dst_rows_host, n_new, batch, top_k, out_idx_host,
                   out_score_host, stream_v, nullptr, true);
}

dsa_status_t dsa_indexer_decode_host_async(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w_host,
                                           const void* k_new_host, dsa_dtype_t k_new_dtype,
                                           const int64_t* dst_rows_host, int32_t n_new, const dsa_batch_t* batch,
                                           int32_t top_k, int32_t* out_idx_host, float* out_score_host,
                                           void* stream_v, void* done_event) {
  if (!done_event) {
    g_last_error.clear();
    return fail(DSA_ERR_INVALID_ARG, "done_event is NULL");
  }
  return host_step(false, q, kc, w_host, k_new_host, k_new_dtype, dst_rows_host, n_new, batch, top_k, out_idx_host,
                   out_score_host, stream_v, static_cast<cudaEvent_t>(done_event), false);
}

dsa_status_t dsa_indexer_prefill_host(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w_host,
                                      const void* k_new_host, dsa_dtype_t k_new_dtype, const int64_t* dst_rows_host,
                                      int32_t n_new, const dsa_batch_t* batch, int32_t top_k, int32_t* out_idx_host,
                                      float* out_score_host, void* stream_v) {
  return host_step(true, q, kc, w_host, k_new_host, k_new_dtype, dst_rows_host, n_new, batch, top_k, out_idx_host,
                   out_score_host, stream_v, nullptr, true);
}

dsa_status_t dsa_indexer_prefill_host_async(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w_host,
                                            const void* k_new_host, dsa_dtype_t k_new_dtype,
                                            const int64_t* dst_rows_host, int32_t n_new, const dsa_batch_t* batch,
                                            int32_t top_k, int32_t* out_idx_host, float* out_score_host,
                                            void* stream_v, void* done_event) {
  if (!done_event) {
    g_last_error.clear();
    return fail(DSA_ERR_INVALID_ARG, "done_event is NULL");
  }
  return host_step(true, q, kc, w_host, k_new_host, k_new_dtype, dst_rows_host, n_new, batch, top_k, out_idx_host,
                   out_score_host, stream_v, static_cast<cudaEvent_t>(done_event), false);
}

// Over a cache of one key per m tokens the same kernels run with every query's causal limit
// mapped to the blocks its position completes (the logits epilogue masks keys past
// (p + 1) / m - 1, the planner sizes key ranges and score rows by it).
dsa_status_t dsa_indexer_decode_compressed(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w,
                                           const dsa_batch_t* batch, int32_t m, int32_t top_k, int32_t* out_idx,
                                           float* out_score, void* stream_v) {
  if (m < 1) {
    g_last_error.clear();
    return fail(DSA_ERR_INVALID_ARG, "m must be >= 1");
  }
  return run_indexer(Mode::Decode, q, kc, w, batch, top_k, out_idx, out_score, nullptr, 0, stream_v, m);
}

dsa_status_t dsa_indexer_prefill_compressed(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w,
                                            const dsa_batch_t* batch, int32_t m, int32_t top_k, int32_t* out_idx,
                                            float* out_score, void* stream_v) {
  if (m < 1) {
    g_last_error.clear();
    return fail(DSA_ERR_INVALID_ARG, "m must be >= 1");
  }
  return run_indexer(Mode::Prefill, q, kc, w, batch, top_k, out_idx, out_score, nullptr, 0, stream_v, m);
}

dsa_status_t dsa_selftest_wait_expiry(int64_t limit_cycles, void* stream_v) {
  g_last_error.clear();
  if (limit_cycles < 1 || limit_cycles > 2000000000LL) return fail(DSA_ERR_INVALID_ARG, "limit_cycles must be in 1 .. 2e9");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  Ctx* c = nullptr;
  dsa_status_t st = get_ctx(stream, &c);
  if (st != DSA_OK) return st;
  DSA_CUDA_TRY(launch_wait_expiry(limit_cycles, c->d_err, stream), "self-test kernel launch");
  ++g_launches;
  return DSA_OK;
}

dsa_status_t dsa_indexer_kcache_append_rope(const dsa_kcache_t* kc, const void* k_new, dsa_dtype_t src_dtype,
                                            const int64_t* dst_rows, const int32_t* positions, int32_t n,
                                            const dsa_rope_t* rope, void* stream_v) {
  g_last_error.clear();
  dsa_status_t st = check_cache(kc);
  if (st != DSA_OK) return st;
  if (n < 0) return fail(DSA_ERR_INVALID_ARG, "n < 0");
  if (n == 0) return DSA_OK;
  if (!k_new || !dst_rows || !positions || !rope) return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (src_dtype != DSA_BF16 && src_dtype != DSA_F32) return fail(DSA_ERR_INVALID_ARG, "src_dtype must be DSA_BF16 or DSA_F32");
  const RopeParams rp = rope_params(*rope);
  if (!rope_shape_supported(kc->d_I, 1, rp)) return fail(DSA_ERR_UNSUPPORTED, "unsupported RoPE layout for d_I = %d", kc->d_I);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  Ctx* c = nullptr;
  if ((st = get_ctx(stream, &c)) != DSA_OK) return st;
  const int fp8 = kc->dtype == DSA_FP8_E4M3;
  DSA_CUDA_TRY(launch_rope_append(k_new, src_dtype == DSA_F32, n, kc->d_I, dst_rows, positions, kc->capacity_rows, rp,
                                  fp8, kc->k, kc->k_scale, c->d_err, stream),
               "RoPE append kernel launch");
  ++g_launches;
  return DSA_OK;
}

dsa_status_t dsa_rope_queries(const void* q_src, dsa_dtype_t src_dtype, int64_t T, int32_t H, int32_t d,
                              const int32_t* positions, const dsa_rope_t* rope, void* q_dst, dsa_dtype_t dst_dtype,
                              float* q_scale, void* stream_v) {
  g_last_error.clear();
  if (T < 0) return fail(DSA_ERR_INVALID_ARG, "T < 0");
  if (T == 0) return DSA_OK;
  if (!q_src || !positions || !rope || !q_dst) return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (src_dtype != DSA_BF16 && src_dtype != DSA_F32) return fail(DSA_ERR_INVALID_ARG, "src_dtype must be DSA_BF16 or DSA_F32");
  if (dst_dtype != DSA_BF16 && dst_dtype != DSA_FP8_E4M3) return fail(DSA_ERR_INVALID_ARG, "dst_dtype must be DSA_BF16 or DSA_FP8_E4M3");
  if (dst_dtype == DSA_FP8_E4M3 && !q_scale) return fail(DSA_ERR_INVALID_ARG, "FP8 output needs q_scale");
  if (T > 0x7FFFFFFF) return fail(DSA_ERR_UNSUPPORTED, "too many tokens for one launch");
  const RopeParams rp = rope_params(*rope);
  if (!rope_shape_supported(d, H, rp)) return fail(DSA_ERR_UNSUPPORTED, "unsupported RoPE shape (H_I %d, d_I %d)", H, d);
  if (reinterpret_cast<uintptr_t>(q_src) % 16 || reinterpret_cast<uintptr_t>(q_dst) % 16)
    return fail(DSA_ERR_INVALID_ARG, "q_src and q_dst must be 16-byte aligned");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  Ctx* c = nullptr;
  dsa_status_t st = get_ctx(stream, &c);
  if (st != DSA_OK) return st;
  if (!g_sms) g_sms = num_sms(c->device);
  DSA_CUDA_TRY(launch_rope_queries(q_src, src_dtype == DSA_F32, T, H, d, positions, rp, dst_dtype == DSA_FP8_E4M3,
                                   q_dst, q_scale, c->d_err, g_sms, stream),
               "RoPE query kernel launch");
  ++g_launches;
  return DSA_OK;
}

dsa_status_t dsa_gather_rows(const void* src, int64_t src_rows, int32_t row_bytes, const int32_t* idx,
                             const int64_t* row_base, int64_t rows, int32_t top_k, void* dst, void* stream_v) {
  g_last_error.clear();
  if (rows < 0 || top_k < 0 || src_rows < 0) return fail(DSA_ERR_INVALID_ARG, "negative size");
  if (rows == 0 || top_k == 0) return DSA_OK;
  if (!src || !idx || !row_base || !dst) return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!gather_row_bytes_supported(row_bytes))
    return fail(DSA_ERR_INVALID_ARG, "row_bytes must be a positive multiple of 16, at most 4096");
  if (reinterpret_cast<uintptr_t>(src) % 16 || reinterpret_cast<uintptr_t>(dst) % 16)
    return fail(DSA_ERR_INVALID_ARG, "src and dst must be 16-byte aligned");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  Ctx* c = nullptr;
  dsa_status_t st = get_ctx(stream, &c);
  if (st != DSA_OK) return st;
  if (!g_sms) g_sms = num_sms(c->device);
  DSA_CUDA_TRY(launch_gather_rows(src, src_rows, row_bytes, idx, row_base, rows, top_k, dst, c->d_err, g_sms, stream),
               "gather kernel launch");
  ++g_launches;
  return DSA_OK;
}

dsa_status_t dsa_selection_rows(const int32_t* idx, const int64_t* row_base, int64_t rows, int32_t top_k,
                                int64_t* out, void* stream_v) {
  g_last_error.clear();
  if (rows < 0 || top_k < 0) return fail(DSA_ERR_INVALID_ARG, "negative size");
  if (rows == 0 || top_k == 0) return DSA_OK;
  if (!idx || !row_base || !out) return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  Ctx* c = nullptr;
  dsa_status_t st = get_ctx(stream, &c);
  if (st != DSA_OK) return st;
  if (!g_sms) g_sms = num_sms(c->device);
  DSA_CUDA_TRY(launch_selection_rows(idx, row_base, rows, top_k, out, g_sms, stream), "selection-rows kernel launch");
  ++g_launches;
  return DSA_OK;
}

dsa_status_t dsa_sort_selection(int32_t* idx, float* score, int64_t rows, int32_t top_k, void* stream_v) {
  g_last_error.clear();
  if (rows < 0 || top_k < 0) return fail(DSA_ERR_INVALID_ARG, "negative size");
  if (rows == 0 || top_k <= 1) return DSA_OK;
  if (!idx || !score) return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (top_k > sort_selection_max()) return fail(DSA_ERR_UNSUPPORTED, "dsa_sort_selection takes top_k <= %d", sort_selection_max());
  if (rows > 0x7FFFFFFF) return fail(DSA_ERR_UNSUPPORTED, "too many rows for one launch");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  Ctx* c = nullptr;
  dsa_status_t st = get_ctx(stream, &c);
  if (st != DSA_OK) return st;
  DSA_CUDA_TRY(launch_sort_selection(idx, score, rows, top_k, stream), "sort kernel launch");
  ++g_launches;
  return DSA_OK;
}

dsa_status_t dsa_indexer_scores(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w,
                                const dsa_batch_t* batch, float* out_scores, int64_t ld, void* stream) {
  return run_indexer(Mode::Scores, q, kc, w, batch, 1, nullptr, nullptr, out_scores, ld, stream);
}

size_t dsa_indexer_workspace_bytes(const dsa_query_t* q, const dsa_batch_t* batch, int32_t top_k) {
  if (!q || !batch || batch->num_seqs < 0 || (batch->num_seqs > 0 && !batch->seq_lens)) return 0;
  int64_t rows = 0, elems = 0, tiles = 0;
  for (int i = 0; i < batch->num_seqs; ++i) {
    const int32_t L = batch->seq_lens[i];
    const int32_t n = batch->q_lens ? batch->q_lens[i] : L;
    for (int32_t j = 0; j < n; ++j) elems += round_up(L - n + j + 1, 4);
    rows += n;
    tiles += (L + kKeyTile - 1) / kKeyTile;
  }
  (void)top_k;
  const int64_t items = rows + tiles + 4096;   // bound on the number of work items
  const int64_t chunks = elems / kStreamChunk + rows;   // bound on the streaming top-k's chunks
  const size_t meta = align_up(items * sizeof(LogitsItem)) + align_up((items + 2) * 4) + align_up(rows * 8) +
                      align_up(rows * 4) + align_up(rows * 4) + align_up(chunks * sizeof(TopkChunk));
  return align_up(meta) + ws_layout(elems, rows, true).total;
}

dsa_status_t dsa_set_workspace(void* ptr, size_t bytes, void* stream_v) {
  g_last_error.clear();
  if (ptr && reinterpret_cast<uintptr_t>(ptr) % 256) return fail(DSA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  Ctx* c = nullptr;
  dsa_status_t st = get_ctx(static_cast<cudaStream_t>(stream_v), &c);
  if (st != DSA_OK) return st;
  c->user_ws = ptr;
  c->user_ws_bytes = ptr ? bytes : 0;
  c->meta_valid = false;
  return DSA_OK;
}

dsa_status_t dsa_check_device_errors(void* stream_v) {
  g_last_error.clear();
  Ctx* c = nullptr;
  dsa_status_t st = get_ctx(static_cast<cudaStream_t>(stream_v), &c);
  if (st != DSA_OK) return st;
  DSA_CUDA_TRY(cudaStreamSynchronize(c->stream), "cudaStreamSynchronize");
  int h[2] = {0, 0};
  DSA_CUDA_TRY(cudaMemcpy(h, c->d_err, sizeof(h), cudaMemcpyDeviceToHost), "cudaMemcpy(error flag)");
  if (h[0] == 0) return DSA_OK;
  DSA_CUDA_TRY(cudaMemset(c->d_err, 0, sizeof(h)), "cudaMemset(error flag)");
  const char* what = h[0] == DSA_DEVERR_TIMEOUT ? "a bounded wait expired in block"
                     : h[0] == DSA_DEVERR_BOUNDS ? "cache append destination out of range for source row"
                     : h[0] == DSA_DEVERR_TOPK   ? "top-k selection invariant broken on row"
                                                 : "unknown device fault, info";
  return fail(DSA_ERR_DEVICE_CHECK, "device fault %d: %s %d", h[0], what, h[1]);
}

dsa_status_t dsa_set_profile_events(void* ev_begin, void* ev_mid, void* ev_end) {
  g_prof[0] = static_cast<cudaEvent_t>(ev_begin);
  g_prof[1] = static_cast<cudaEvent_t>(ev_mid);
  g_prof[2] = static_cast<cudaEvent_t>(ev_end);
  return DSA_OK;
}

uint64_t dsa_kernel_launch_count(void) { return g_launches; }

const char* dsa_get_last_error(void) { return g_last_error.c_str(); }

const char* dsa_version(void) { return "dsa_indexer 0.1 (sm_100a)"; }

}  // extern "C"

// ============================================================================= decode without device allocation
//
// dsa_indexer_decode obtains its workspace with cudaMalloc the first time a stream
// needs it.  Some callers may not allocate at all: a serving process whose device
// memory is carved up in advance by its own pool (an allocation behind its back can
// fail or fragment that pool), code that runs under a device-memory budget enforced
// outside CUDA, or an embedding that forbids allocator calls on its hot path.  For
// them, dsa_indexer_decode_noalloc keeps the score rows and scheduling tables in one
// file-scope __device__ array instead.  The array is part of this library's device
// image, so every GPU that loads the library holds it until the process exits.

namespace dsa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB on every device
constexpr size_t kNoAllocFaultBytes = 256;                  // fault words at the front of the array

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array on the current device.  In host code the symbol is
// only a stand-in, so the address is looked up once per device with that device
// current, and kept.
dsa_status_t noalloc_scratch(void** out) {
  int dev = 0;
  DSA_CUDA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
  static std::mutex mu;
  static std::map<int, void*> addr;
  std::lock_guard<std::mutex> lk(mu);
  auto it = addr.find(dev);
  if (it == addr.end()) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    if (p == nullptr) return fail(DSA_ERR_CUDA, "cudaGetSymbolAddress(static scratch) returned NULL");
    it = addr.emplace(dev, p).first;
  }
  *out = it->second;
  return DSA_OK;
}

// The call's scheduling tables travel to the array inside kernel parameters, in chunks of
// kTableChunk bytes: a parameter block is copied when the launch is enqueued, so the host
// blob may be freed as soon as the call returns, and nothing is staged through host memory
// that the driver would have to allocate or pin.
constexpr int kTableChunk = 16384;
struct __align__(16) TableChunk {
  unsigned char bytes[kTableChunk];
};

// Copies `n` bytes (a multiple of 16) of the chunk to dst; the first chunk of a call also
// clears the call's two fault words.
__global__ void __launch_bounds__(256) noalloc_tables_kernel(const __grid_constant__ TableChunk chunk, int n,
                                                             unsigned char* __restrict__ dst, int* fault_words) {
  const uint4* src = reinterpret_cast<const uint4*>(chunk.bytes);
  uint4* out = reinterpret_cast<uint4*>(dst);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n / 16; i += gridDim.x * blockDim.x) out[i] = src[i];
  if (fault_words != nullptr && blockIdx.x == 0 && threadIdx.x < 2) fault_words[threadIdx.x] = 0;
}

dsa_status_t noalloc_upload(const std::vector<uint8_t>& blob, unsigned char* dst, int* fault_words,
                            cudaStream_t stream) {
  static thread_local TableChunk chunk;
  size_t off = 0;
  do {
    const size_t n = std::min(blob.size() - off, static_cast<size_t>(kTableChunk));
    if (n) std::memcpy(chunk.bytes, blob.data() + off, n);
    const int blocks = static_cast<int>((n / 16 + 255) / 256) > 0 ? static_cast<int>((n / 16 + 255) / 256) : 1;
    noalloc_tables_kernel<<<blocks, 256, 0, stream>>>(chunk, static_cast<int>(n), dst + off,
                                                      off == 0 ? fault_words : nullptr);
    DSA_CUDA_TRY(cudaGetLastError(), "table upload kernel launch");
    ++g_launches;
    off += n;
  } while (off < blob.size());
  return DSA_OK;
}

}  // namespace
}  // namespace dsa

extern "C" dsa_status_t dsa_indexer_decode_noalloc(const dsa_query_t* q, const dsa_kcache_t* kc, const float* w,
                                                   const dsa_batch_t* batch, int32_t top_k, int32_t* out_idx,
                                                   float* out_score, int32_t* fault, void* stream_v) {
  using namespace dsa;
  g_last_error.clear();
  dsa_status_t st = check_cache(kc);
  if (st != DSA_OK) return st;
  BatchView v;
  if ((st = check_batch(batch, kc, true, &v)) != DSA_OK) return st;
  if (top_k < 1) return fail(DSA_ERR_INVALID_ARG, "top_k must be >= 1");
  if (v.total_q == 0) return DSA_OK;
  if ((st = check_query(q, kc)) != DSA_OK) return st;
  if (!w) return fail(DSA_ERR_INVALID_ARG, "w is NULL");
  if (!out_idx || !out_score) return fail(DSA_ERR_INVALID_ARG, "out_idx / out_score is NULL");
  const bool fp8 = kc->dtype == DSA_FP8_E4M3;
  const int H = q->H_I, D = kc->d_I;
  const int tpa = logits_queries_per_item(H, D, false, v.max_q_len);
  if (!logits_config_supported(H, D, fp8, tpa, 1, false))
    return fail(DSA_ERR_UNSUPPORTED, "no decode kernel for H_I=%d, d_I=%d, dtype=%s", H, D, fp8 ? "fp8" : "bf16");

  int dev = 0;
  DSA_CUDA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
  const int sms = num_sms(dev);
  Plan p;
  p.tpa = tpa;
  p.ng = 1;
  plan_rows(v, false, 0, &p);
  plan_decode_items(v, sms, &p);
  if ((st = plan_topk(v, top_k, sms, &p)) != DSA_OK) return st;
  const MetaLayout m = layout_of(p);
  const size_t need = kNoAllocFaultBytes + align_up(m.total) + align_up(size_t(p.score_elems) * sizeof(float));
  if (need > kNoAllocScratchBytes)
    return fail(DSA_ERR_INVALID_ARG,
                "this batch needs %zu bytes of scratch; dsa_indexer_decode_noalloc has a fixed %zu "
                "(score rows take 4 bytes per cached key, rounded up to 4 keys per query)",
                need, kNoAllocScratchBytes);

  void* base = nullptr;
  if ((st = noalloc_scratch(&base)) != DSA_OK) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  int* err = fault ? reinterpret_cast<int*>(fault) : static_cast<int*>(base);
  char* mb = static_cast<char*>(base) + kNoAllocFaultBytes;
  float* d_scores = reinterpret_cast<float*>(mb + align_up(m.total));
  // the tables (and the cleared fault words) go to the array in kernel parameters
  if ((st = noalloc_upload(pack(p, m), reinterpret_cast<unsigned char*>(mb), err, stream)) != DSA_OK) return st;

  CUtensorMap tk, tq;
  if ((st = encode_rows(&tk, kc->k, fp8, kc->capacity_rows, D, kKeyTile)) != DSA_OK) return st;
  if ((st = encode_rows(&tq, q->data, fp8, v.total_q * H, D, tpa * H)) != DSA_OK) return st;
  LogitsArgs la{};
  la.items = reinterpret_cast<const LogitsItem*>(mb + m.items);
  la.cta_items = reinterpret_cast<const int32_t*>(mb + m.cta);
  la.row_off = reinterpret_cast<const int64_t*>(mb + m.row_off);
  la.w = w;
  la.q_scale = fp8 ? q->scale : nullptr;
  la.k_scale = fp8 ? kc->k_scale : nullptr;
  la.k_capacity = kc->capacity_rows;
  la.scores = d_scores;
  la.inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  la.err = err;
  LogitsLaunch L{H, D, fp8, tpa, 1, static_cast<int>(p.cta_items.size()) - 1, stream, false};
  DSA_CUDA_TRY(launch_logits(L, tk, tq, la), "logits kernel launch");
  g_launches += L.grid > 0;
  TopkArgs ta{};
  ta.scores = d_scores;
  ta.row_off = la.row_off;
  ta.row_pos = reinterpret_cast<const int32_t*>(mb + m.row_pos);
  ta.top_k = top_k;
  ta.out_idx = out_idx;
  ta.out_score = out_score;
  ta.err = err;
  const int32_t* rows = reinterpret_cast<const int32_t*>(mb + m.topk_rows);
  if (p.short_count) {
    TopkArgs s = ta;
    s.rows = rows + p.short_first;
    s.n_rows = static_cast<int32_t>(p.short_count);
    DSA_CUDA_TRY(launch_topk_short(s, stream), "top-k (short rows) launch");
    ++g_launches;
  }
  for (const auto& cl : p.classes) {
    TopkArgs s = ta;
    s.rows = rows + cl.first;
    s.n_rows = static_cast<int32_t>(cl.count);
    DSA_CUDA_TRY(launch_topk(s, cl.ept, cl.cluster, stream), "top-k launch");
    ++g_launches;
  }
  return DSA_OK;
}
