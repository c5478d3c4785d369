// Internal types shared by the host planner (host_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dsa {

// Device fault codes (the first one wins; reported by dsa_check_device_errors).
enum : int {
  DSA_DEVERR_NONE = 0,
  DSA_DEVERR_TIMEOUT = 1,     // a bounded wait ran out
  DSA_DEVERR_BOUNDS = 2,      // a destination row outside the cache capacity
  DSA_DEVERR_TOPK = 3,        // selection invariant broken (count mismatch)
};

constexpr int kKeyTile = 128;       // keys per UMMA tile (the M dimension)
// Coarse per-row score histogram built by the decode logits epilogue for the top-k: every
// valid key, binned by the top 12 bits of its order-preserving key (sign, exponent and three
// mantissa bits: eighth-octave bins).
constexpr int kHistShift = 20;
constexpr int kHistBins = 1 << (32 - kHistShift);

// Order-preserving map of a float to uint32 (larger float -> larger key).
__host__ __device__ __forceinline__ uint32_t order_key(uint32_t float_bits) {
  return (float_bits & 0x80000000u) ? ~float_bits : (float_bits | 0x80000000u);
}
constexpr int kTopkThreads = 512;   // threads per top-k CTA
constexpr int kTopkBins = 2048;     // histogram bins per refinement level
constexpr int kStreamChunk = 4096;  // keys per CTA of the streaming (decode) top-k

// One CTA of the streaming top-k: keys [begin, end) of query row `row`, which is split
// into `n_chunks` such chunks.
struct TopkChunk {
  int32_t row;
  int32_t begin;
  int32_t end;
  int32_t n_chunks;
};
static_assert(sizeof(TopkChunk) == 16, "TopkChunk layout");

// One unit of logits work: `n_tok` consecutive query rows of one sequence against
// key tiles [kt_begin, kt_end) of that sequence.
struct LogitsItem {
  int64_t k_row0;    // cache row holding key position 0 of the sequence
  int32_t q_row0;    // global (packed) row of the item's first query
  int32_t n_tok;     // queries in this item
  int32_t pos0;      // position of the first query inside its sequence
  int32_t kt_begin;  // first key tile
  int32_t kt_end;    // one past the last key tile
  int32_t cmp;       // 0 or 1: the cache holds every key; m > 1: one key per m tokens (query at
                     // position p sees keys 0 .. (p + 1) / m - 1)
};
static_assert(sizeof(LogitsItem) == 32, "LogitsItem layout");

struct LogitsArgs {
  const LogitsItem* items;
  const int32_t* cta_items;  // [grid + 1]: items of CTA c are [cta_items[c], cta_items[c+1])
  const int64_t* row_off;    // [T_total]: score row r starts at scores + row_off[r]
  const float* w;            // [T_total, H]
  const float* q_scale;      // [T_total] (FP8) or nullptr
  const float* k_scale;      // [capacity_rows] (FP8) or nullptr
  int64_t k_capacity;        // rows in the cache (bounds for k_scale reads)
  float* scores;             // workspace
  uint32_t* row_hist;        // [T_total, kHistBins] zeroed coarse histograms, or nullptr
  float inv_sqrt_d;
  int* err;
};

struct TopkArgs {
  const float* scores;
  const int64_t* row_off;
  const int32_t* row_pos;    // [T_total]: position p of each query row (valid keys 0..p)
  const int32_t* rows;       // rows handled by this launch (cluster and short kernels)
  int32_t n_rows;
  int32_t top_k;
  int32_t* out_idx;
  float* out_score;
  int* err;
  // streaming kernel only
  const TopkChunk* chunks;   // [n_chunks], the chunks of a row consecutive
  int32_t n_chunks;
  const uint32_t* row_hist;  // [T_total, kHistBins] coarse histograms from the logits epilogue
  uint32_t* row_hist1;       // [T_total, kTopkBins] zeroed: level-1 histograms of each row's threshold bin
  uint32_t* row_ctr;         // [T_total, 4] zeroed: bin keys gathered, keys written above the bin, chunks done
  uint32_t* cand_key;        // gathered bin keys of row r at cand_key + row_off[r]
  int32_t* cand_idx;         // their positions, same layout
};

// ----------------------------------------------------------------------------- launchers

// Logits kernel configuration chosen by the host.
struct LogitsLaunch {
  int H, D;
  bool fp8;
  int tpa;     // queries per accumulator (N = tpa * H)
  int ng;      // accumulators (query groups) per work item
  int grid;
  cudaStream_t stream;
  bool prefill;   // prefill work items (a query block over its causal range), else decode
};


cudaError_t launch_logits(const LogitsLaunch& L, const CUtensorMap& tmap_k, const CUtensorMap& tmap_q,
                          const LogitsArgs& a);
bool logits_config_supported(int H, int D, bool fp8, int tpa, int ng, bool prefill);
// Whether that configuration's epilogue counts every stored score in its row's coarse
// histogram (the decode top-k then needs no pass of its own to build them).
bool logits_bins_rows(int H, int D, bool fp8, int tpa, int ng, bool prefill);

// Top-k over rows longer than top_k: one cluster of `cluster` CTAs per row,
// `ept` keys per thread held in registers.
cudaError_t launch_topk(const TopkArgs& a, int ept, int cluster, cudaStream_t stream);
// Rows longer than top_k, one CTA per row streaming it in passes (prefill: many rows).
cudaError_t launch_topk_rows(const TopkArgs& a, cudaStream_t stream);
// Rows whose coarse histogram the logits epilogue built: one CTA per chunk of kStreamChunk
// keys, the last CTA of a row finishing the selection inside the threshold bin.
cudaError_t launch_topk_stream(const TopkArgs& a, cudaStream_t stream);
// Coarse row histograms from the score rows (decode configurations whose logits epilogue
// does not count them), one CTA per streaming chunk; row_hist must start zeroed.
cudaError_t launch_row_hist(const TopkArgs& a, cudaStream_t stream);
// Rows with at most top_k candidates: every causal position, then padding.
cudaError_t launch_topk_short(const TopkArgs& a, cudaStream_t stream);

// Rotary embedding fused into the key append and the query quantisation.
constexpr int kRopeMaxPairs = 64;      // rope_dim <= 128
struct RopeParams {
  int32_t rope_dim;      // leading values of each vector that rotate (even)
  int32_t interleaved;   // 1: pairs (2i, 2i+1); 0: pairs (i, i + rope_dim / 2)
  double base;           // theta_i = position * base^(-2 i / rope_dim)
  double inv_freq[kRopeMaxPairs];   // base^(-2 i / rope_dim), filled by the host
};
bool rope_shape_supported(int32_t d, int32_t H, const RopeParams& r);
cudaError_t launch_rope_append(const void* src, int src_is_f32, int64_t rows, int32_t d, const int64_t* dst_rows,
                               const int32_t* positions, int64_t capacity, const RopeParams& r, int fp8, void* cache,
                               float* scale, int* err, cudaStream_t stream);
cudaError_t launch_rope_queries(const void* src, int src_is_f32, int64_t T, int32_t H, int32_t d,
                                const int32_t* positions, const RopeParams& r, int fp8, void* dst, float* scale,
                                int* err, int sms, cudaStream_t stream);

cudaError_t launch_fill_f32(float* p, int64_t n, float v, cudaStream_t stream);
cudaError_t launch_wait_expiry(long long limit_cycles, int* err, cudaStream_t stream);

// After the selection: latent-row gather, int64 cache rows, sorted order.
bool gather_row_bytes_supported(int32_t row_bytes);
int sort_selection_max();
cudaError_t launch_gather_rows(const void* src, int64_t src_rows, int32_t row_bytes, const int32_t* idx,
                               const int64_t* row_base, int64_t rows, int32_t top_k, void* dst, int* err, int sms,
                               cudaStream_t stream);
cudaError_t launch_selection_rows(const int32_t* idx, const int64_t* row_base, int64_t rows, int32_t top_k,
                                  int64_t* out, int sms, cudaStream_t stream);
cudaError_t launch_sort_selection(int32_t* idx, float* score, int64_t rows, int32_t top_k, cudaStream_t stream);

cudaError_t launch_quantize_rows_fp8(const void* src, int src_is_f32, int64_t rows, int32_t row_len,
                                     uint8_t* dst, float* scale, const int64_t* dst_rows, int64_t dst_capacity,
                                     int* err, cudaStream_t stream);
cudaError_t launch_append_bf16(const void* src, int src_is_f32, int64_t rows, int32_t row_len, uint16_t* dst,
                               const int64_t* dst_rows, int64_t dst_capacity, int* err, cudaStream_t stream);

int num_sms(int device);

}  // namespace dsa
