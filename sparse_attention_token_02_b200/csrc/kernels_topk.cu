// Per-row top-k selection over fp32 indexer scores (page "从原理到代码：手把手教你理解
// DeepSeek-V3.2的闪电索引器设计" §3 step 5, top-k per query; "Lightning Indexer 详解" §2.3:
// at most min(k, L) positions exist).
//
// Threshold select, exact, with the keys held in registers:
//   * one cluster of `cs` CTAs per row (distributed shared memory joins them); each
//     thread loads EPT scores of its CTA's slice with 16-byte loads and maps each to
//     an order-preserving uint32 key (larger float -> larger key);
//   * the cluster reduces min and max key -> candidate key interval [lo, hi]; when the
//     logits epilogue has binned the row (decode), its coarse histogram gives the
//     threshold bin directly and this level and the next are skipped;
//   * refinement level: bin = (key - lo) >> shift, with shift chosen so the interval
//     spans at most 2048 bins.  Histograms are built with shared atomics and summed
//     into rank 0 over DSMEM; rank 0 finds the bin holding the k-th largest key,
//     everything in higher bins is selected, and the interval shrinks to that bin
//     (by at least 2^10 per level, so at most four levels).  It stops when the bin
//     holds exactly the keys still needed, or when the interval is a single key
//     value (ties: any `need` of them are taken, the order of equal scores being
//     unspecified);
//   * output pass: every thread counts its selected keys, a block scan plus one
//     DSMEM atomic per CTA gives each thread its output slots.
// Output order inside a row is unspecified (the selection is a set).
#include <cooperative_groups.h>
#include <type_traits>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace dsa {

namespace {

constexpr int kThreads = kTopkThreads;
constexpr int kBins = kTopkBins;
constexpr int kBinsPerThread = kBins / kThreads;
static_assert(kBins % kThreads == 0, "bins per thread");

__device__ __forceinline__ uint32_t float_to_key(float f) { return order_key(__float_as_uint(f)); }

__device__ __forceinline__ float key_to_float(uint32_t k) {
  const uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

// Exclusive prefix sum over the CTA's threads (in threadIdx order); also returns the total.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_sums, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n_warps = blockDim.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t s = lane < n_warps ? warp_sums[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < n_warps) warp_sums[lane] = s;   // inclusive warp prefix
  }
  __syncthreads();
  total = warp_sums[n_warps - 1];
  const uint32_t before = warp == 0 ? 0u : warp_sums[warp - 1];
  __syncthreads();                            // warp_sums may be reused right after
  return before + x - v;
}

constexpr uint32_t kNotFound = 0xFFFFFFFFu;

struct SelectState {
  uint32_t lo, hi;      // candidate key interval
  uint32_t need;        // keys still to take from the interval
  uint32_t done;        // 1: take every key in [lo, hi];  2: [lo, hi] is one tied value
};

static_assert(kBinsPerThread == 4, "the histogram pull reads 4 bins as one uint4");
constexpr int kMaxCluster = 8;              // CTAs per row (the host never asks for more)

// Keys of the threshold bin gathered into rank 0 for the rest of the selection.
constexpr int kCandCap = 8192;
constexpr size_t kTopkSmemBytes = (kBins + 2 * kCandCap) * sizeof(uint32_t);

// Block-wide search of a histogram held as `cnt[j]` for the bins this thread owns (bins in
// descending order across threads): the bin whose suffix count crosses `need`.
// Exactly one thread sets *found_* (if the total reaches need).
template <int PER>
__device__ __forceinline__ void find_threshold_bin(const uint32_t (&cnt)[PER], uint32_t first_bin_desc,
                                                   uint32_t need, uint32_t* warp_sums, uint32_t* found_bin,
                                                   uint32_t* found_above, uint32_t* found_cnt) {
  uint32_t sum = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) sum += cnt[j];
  uint32_t total;
  uint32_t above = block_exclusive_scan(sum, warp_sums, total);
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    if (above < need && above + cnt[j] >= need) {
      *found_bin = first_bin_desc - j;
      *found_above = above;
      *found_cnt = cnt[j];
    }
    above += cnt[j];
  }
}

// PER consecutive bins starting at h, returned in descending bin order.
template <int PER>
__device__ __forceinline__ void load_bins_desc(const uint32_t* h, uint32_t (&c)[PER]) {
#pragma unroll
  for (int q = 0; q < PER / 4; ++q) {
    const uint4 v = __ldcg(reinterpret_cast<const uint4*>(h + 4 * q));
    c[PER - 1 - 4 * q] = v.x;
    c[PER - 2 - 4 * q] = v.y;
    c[PER - 3 - 4 * q] = v.z;
    c[PER - 4 - 4 * q] = v.w;
  }
}

// Zeroes part `part` of `parts` of a row's coarse histogram (16-byte stores) once every
// reader of it is done, so the next call's logits epilogue counts into a clear histogram
// without a memset between the launches.
__device__ __forceinline__ void clear_row_hist(uint32_t* h, int part, int parts) {
  constexpr int kVecs = kHistBins / 4;
  uint4* v = reinterpret_cast<uint4*>(h);
  const int per = (kVecs + parts - 1) / parts;
  for (int i = part * per + static_cast<int>(threadIdx.x); i < min(kVecs, (part + 1) * per); i += blockDim.x)
    v[i] = make_uint4(0u, 0u, 0u, 0u);
}

// Calls f(key, index, valid) for candidates [0, m), each thread taking every NT-th one
// (valid is false past m).  Reads
// go in batches of CPT per thread, all loads of a batch issued before any is used: global
// candidates cost an L2 round trip each, which a one-at-a-time loop would serialise.
template <bool kGlobal, bool kWithIdx, int NT, int CPT, class F>
__device__ __forceinline__ void for_candidates(const uint32_t* ck, const int32_t* ci, uint32_t m, F&& f) {
  for (uint32_t b0 = 0; b0 < m; b0 += NT * CPT) {
    uint32_t kk[CPT];
    int32_t ix[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const uint32_t i = b0 + j * NT + threadIdx.x;
      kk[j] = 0u;
      ix[j] = 0;
      if (i < m) {
        kk[j] = kGlobal ? __ldcg(ck + i) : ck[i];
        if (kWithIdx) ix[j] = kGlobal ? __ldcg(ci + i) : ci[i];
      }
    }
#pragma unroll
    for (int j = 0; j < CPT; ++j) f(kk[j], ix[j], b0 + j * NT + threadIdx.x < m);
  }
}

// Sorts one key per lane of a warp in descending order across the lanes (bitonic network).
__device__ __forceinline__ uint32_t warp_sort_desc(uint32_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const uint32_t o = __shfl_xor_sync(0xffffffffu, v, j);
      const bool asc = (lane & k) == 0, low = (lane & j) == 0;
      v = low == asc ? max(v, o) : min(v, o);
    }
  }
  return v;
}

// One CTA, all its threads: the m gathered keys (in this CTA's shared memory, or with
// kGlobalCand in global memory, read through the L2 since other CTAs wrote them) are
// n_up keys above hi, all selected, and m - n_up keys in [lo, hi] of which the `need`
// largest are selected; all n_up + need go to slots [base, base + n_up + need) of the row.
// Exact: CTA-local histogram levels narrow [lo, hi] by >= 2^10 per level; once the interval
// holds at most 32 keys one warp sorts them and the need-th largest value v becomes the
// interval [v, v] (the keys above v join the selected ones); keys above the final interval are
// taken, then `need` of its keys (a single tied value if not resolved).
// Returns false if the counts turn out inconsistent (nothing is written past the row).
template <bool kGlobalCand, int NT>
__device__ bool rank0_select(const uint32_t* cand_key, const int32_t* cand_idx, uint32_t m, uint32_t n_up,
                             uint32_t lo, uint32_t hi, uint32_t need, uint32_t base, int32_t* oi, float* os, uint32_t* hist,
                             uint32_t* warp_sums, uint32_t* lvl_bin, uint32_t* lvl_above, uint32_t* lvl_cnt,
                             uint32_t* ctr_a, uint32_t* ctr_b) {
  constexpr int PER = kBins / NT;
  constexpr int CPT = kGlobalCand ? 8 : 1;
  const int tid = threadIdx.x;
  SelectState ls;
  ls.lo = lo;
  ls.hi = hi;
  ls.need = need;
  ls.done = need == m - n_up ? 1u : 0u;
  uint32_t cnt = m - n_up;                    // keys inside [lo, hi]
  for (int level = 0; level < 5 && !ls.done; ++level) {
    if (ls.lo == ls.hi) { ls.done = 2; break; }
    if (cnt <= 32u) {
      // few keys left: gather them (key, position) into the histogram's first 64 words, sort
      // them in one warp, and keep the need-th largest value as a one-value interval
      if (tid == 0) *ctr_a = 0u;
      __syncthreads();
      for_candidates<kGlobalCand, true, NT, CPT>(cand_key, cand_idx, m, [&](uint32_t kk, int32_t ix, bool valid) {
        if (valid && kk >= ls.lo && kk <= ls.hi) {
          const uint32_t slot = atomicAdd(ctr_a, 1u);
          if (slot < 32u) {
            hist[slot] = kk;
            hist[32 + slot] = static_cast<uint32_t>(ix);
          }
        }
      });
      __syncthreads();
      if (*ctr_a != cnt) return false;        // inconsistent counts (uniform: read after the barrier)
      if (tid < 32) {
        const uint32_t v = warp_sort_desc(tid < static_cast<int>(cnt) ? hist[tid] : 0u);
        const uint32_t vk = __shfl_sync(0xffffffffu, v, static_cast<int>(ls.need) - 1);
        const uint32_t gt = __popc(__ballot_sync(0xffffffffu, v > vk));
        if (tid == 0) {
          *lvl_bin = vk;
          *lvl_above = gt;
        }
      }
      __syncthreads();
      ls.lo = *lvl_bin;
      ls.hi = ls.lo;
      ls.need -= *lvl_above;
      ls.done = 2;
      __syncthreads();                        // lvl_* and ctr_a are reused below
      break;
    }
    const int bits = 32 - __clz(ls.hi - ls.lo);
    const int shift = bits > 11 ? bits - 11 : 0;
    for (int b = tid; b < kBins; b += NT) hist[b] = 0u;
    __syncthreads();
    for_candidates<kGlobalCand, false, NT, CPT>(cand_key, cand_idx, m, [&](uint32_t kk, int32_t, bool valid) {
      if (valid && kk >= ls.lo && kk <= ls.hi) atomicAdd(&hist[(kk - ls.lo) >> shift], 1u);
    });
    __syncthreads();
    uint32_t c[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) c[j] = hist[kBins - 1 - (tid * PER + j)];
    if (tid == 0) *lvl_bin = kNotFound;
    find_threshold_bin<PER>(c, kBins - 1 - tid * PER, ls.need, warp_sums, lvl_bin, lvl_above, lvl_cnt);
    __syncthreads();
    if (*lvl_bin == kNotFound) return false;
    SelectState ns;
    ns.lo = ls.lo + (*lvl_bin << shift);
    const uint32_t width_m1 = (1u << shift) - 1u;
    ns.hi = (ls.hi - ns.lo) > width_m1 ? ns.lo + width_m1 : ls.hi;
    ns.need = ls.need - *lvl_above;
    ns.done = *lvl_cnt == ns.need ? 1u : 0u;
    cnt = *lvl_cnt;
    ls = ns;
    __syncthreads();
  }
  if (!ls.done) ls.done = 2;                  // unreachable: >= 10 bits resolved per level
  if (tid == 0) {
    *ctr_a = 0u;
    *ctr_b = 0u;
  }
  __syncthreads();
  const uint32_t n_sel_up = n_up + (need - ls.need);     // keys above the final interval
  const uint32_t first_in = base + n_sel_up;             // slots of interval keys start here
  // slots per warp: one atomic per counter and warp (every thread calls f the same number of
  // times, so the ballots see the whole warp)
  const uint32_t lane_lt = (1u << (threadIdx.x & 31)) - 1u;
  for_candidates<kGlobalCand, true, NT, CPT>(cand_key, cand_idx, m, [&](uint32_t kk, int32_t ix, bool valid) {
    const bool up = valid && kk > ls.hi;
    const bool in = valid && !up && kk >= ls.lo;
    const uint32_t bu = __ballot_sync(0xffffffffu, up), bi = __ballot_sync(0xffffffffu, in);
    uint32_t su = 0u, si = 0u;
    if ((threadIdx.x & 31) == 0) {
      if (bu) su = atomicAdd(ctr_a, static_cast<uint32_t>(__popc(bu)));
      if (bi) si = atomicAdd(ctr_b, static_cast<uint32_t>(__popc(bi)));
    }
    su = __shfl_sync(0xffffffffu, su, 0) + __popc(bu & lane_lt);
    si = __shfl_sync(0xffffffffu, si, 0) + __popc(bi & lane_lt);
    if (up) {
      const uint32_t slot = base + su;
      if (slot < first_in) {
        oi[slot] = ix;
        os[slot] = key_to_float(kk);
      }
    } else if (in && si < ls.need) {
      oi[first_in + si] = ix;
      os[first_in + si] = key_to_float(kk);
    }
  });
  __syncthreads();
  return *ctr_a == n_sel_up && *ctr_b >= ls.need && !(ls.done == 1 && *ctr_b != ls.need);
}

template <int EPT>
__global__ void __launch_bounds__(kThreads, EPT <= 8 ? 2 : 1)
topk_kernel(const TopkArgs a) {
  static_assert(EPT % 4 == 0, "EPT is a multiple of 4");
  static_assert(EPT * kThreads < 65536, "per-CTA counts are packed in 16 bits");
  extern __shared__ __align__(16) uint32_t dsm[];
  uint32_t* hist = dsm;                                             // kBins
  uint32_t* cand_key = dsm + kBins;                                 // kCandCap
  int32_t* cand_idx = reinterpret_cast<int32_t*>(cand_key + kCandCap);   // kCandCap
  __shared__ uint32_t warp_sums[32];
  __shared__ SelectState st;
  __shared__ uint32_t cnt_above, cnt_cand, base_above, base_cand;
  __shared__ uint32_t lvl_bin, lvl_above, lvl_cnt;
  __shared__ uint32_t loc_min, loc_max;

  cg::cluster_group cluster = cg::this_cluster();
  const uint32_t cs = cluster.num_blocks();
  const uint32_t crank = cluster.block_rank();
  const int tid = threadIdx.x, lane = tid & 31;
  const int row_slot = blockIdx.x / cs;
  if (row_slot >= a.n_rows) return;           // whole clusters exit together (grid = n_rows * cs)
  const int row = a.rows[row_slot];
  const int n = a.row_pos[row] + 1;           // candidate positions 0..n-1 (n > top_k here)
  const float* src = a.scores + a.row_off[row];
  const uint32_t k = static_cast<uint32_t>(a.top_k);
  int32_t* oi = a.out_idx + static_cast<int64_t>(row) * a.top_k;
  float* os = a.out_score + static_cast<int64_t>(row) * a.top_k;

  const int per = ((n + cs - 1) / cs + 3) & ~3;
  const int beg = crank * per;
  const int end = min(n, beg + per);

  uint32_t* cnt_above0 = cluster.map_shared_rank(&cnt_above, 0);
  uint32_t* cnt_cand0 = cluster.map_shared_rank(&cnt_cand, 0);
  uint32_t* ck0 = cluster.map_shared_rank(cand_key, 0);
  int32_t* ci0 = cluster.map_shared_rank(cand_idx, 0);

  for (int b = tid; b < kBins; b += kThreads) hist[b] = 0u;
  if (tid == 0) {
    cnt_above = 0u;
    cnt_cand = 0u;
    loc_min = 0xFFFFFFFFu;
    loc_max = 0u;
    lvl_bin = kNotFound;                      // stays so if a histogram cannot reach its target
    lvl_above = 0u;
    lvl_cnt = 0u;
  }
  __syncthreads();
  // rank 0's counters are zeroed before any CTA of the cluster touches them remotely: arrive
  // now, wait just before the first access to another CTA's shared memory (by then every CTA
  // has long arrived, so the wait costs nothing)
  cluster_arrive();
  grid_dependency_wait();                     // the scores come from the previous kernel

  // ---- the row's coarse histogram, when the logits epilogue built one (decode)
  constexpr int kPer0 = kHistBins / kThreads;
  uint32_t c0[kPer0];
  if (a.row_hist)
    load_bins_desc<kPer0>(a.row_hist + static_cast<int64_t>(row) * kHistBins + (kHistBins - kPer0 * (tid + 1)), c0);

  // ---- load the slice into registers as order-preserving keys (0 = absent)
  uint32_t key[EPT];
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
  for (int v = 0; v < EPT / 4; ++v) {
    const int i = beg + (v * kThreads + tid) * 4;
    float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < end) f = __ldcs(reinterpret_cast<const float4*>(src + i));
    const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t kk = (i + e < end) ? float_to_key(fv[e]) : 0u;
      key[v * 4 + e] = kk;
      if (kk) {
        kmin = min(kmin, kk);
        kmax = max(kmax, kk);
      }
    }
  }

  uint32_t bin_lo, bin_hi;
  if (a.row_hist) {
    // the histogram fixes the threshold bin B (every CTA of the cluster reads the same one)
    find_threshold_bin<kPer0>(c0, kHistBins - 1 - kPer0 * tid, k, warp_sums, &lvl_bin, &lvl_above, &lvl_cnt);
    __syncthreads();
    bin_lo = lvl_bin << kHistShift;
    bin_hi = bin_lo | ((1u << kHistShift) - 1u);
    cluster_wait();
  } else {
    // ---- data-driven first level: bins spread over the row's key range
    cluster_wait();
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
      kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    if (lane == 0) {
      atomicMin(&loc_min, kmin);
      atomicMax(&loc_max, kmax);
    }
    cluster.sync();                           // every CTA's key range is published
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    {
      uint32_t rmin[kMaxCluster], rmax[kMaxCluster];   // all remote loads in flight together
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r) {
        rmin[r] = r < static_cast<int>(cs) ? *cluster.map_shared_rank(&loc_min, r) : 0xFFFFFFFFu;
        rmax[r] = r < static_cast<int>(cs) ? *cluster.map_shared_rank(&loc_max, r) : 0u;
      }
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r) {
        lo = min(lo, rmin[r]);
        hi = max(hi, rmax[r]);
      }
    }
    const int bits0 = hi > lo ? 32 - __clz(hi - lo) : 0;
    const int shift0 = bits0 > 11 ? bits0 - 11 : 0;
#pragma unroll
    for (int e = 0; e < EPT; ++e)
      if (key[e]) atomicAdd(&hist[(key[e] - lo) >> shift0], 1u);
    cluster.sync();                           // every CTA's histogram is complete
    {
      // every CTA sums the cluster's histograms and finds the bin of the k-th key
      uint32_t c[kBinsPerThread];
#pragma unroll
      for (int j = 0; j < kBinsPerThread; ++j) c[j] = 0u;
      // this thread's kBinsPerThread consecutive bins as one 16-byte load per rank, all in flight
      const int b0 = kBins - (tid + 1) * kBinsPerThread;
      uint4 part[kMaxCluster];
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r)
        part[r] = r < static_cast<int>(cs) ? *reinterpret_cast<const uint4*>(cluster.map_shared_rank(hist, r) + b0)
                                           : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r) {
        c[0] += part[r].w;       // bins in descending order: b0+3, b0+2, b0+1, b0
        c[1] += part[r].z;
        c[2] += part[r].y;
        c[3] += part[r].x;
      }
      find_threshold_bin<kBinsPerThread>(c, kBins - 1 - tid * kBinsPerThread, k, warp_sums, &lvl_bin, &lvl_above,
                                         &lvl_cnt);
    }
    __syncthreads();
    bin_lo = lo + (lvl_bin << shift0);
    const uint32_t bin_w1 = (1u << shift0) - 1u;
    bin_hi = (hi - bin_lo) > bin_w1 ? bin_lo + bin_w1 : hi;
  }
  // the row's coarse histogram, cleared by the cluster after its first cluster-wide barrier
  // (every CTA has read it by then)
  uint32_t* my_hist = a.row_hist ? const_cast<uint32_t*>(a.row_hist) + static_cast<int64_t>(row) * kHistBins : nullptr;
  if (lvl_bin == kNotFound) {
    // The histogram holds fewer than top_k keys, which the row's data cannot produce:
    // record the fault and write nothing (every CTA of the cluster takes this branch).
    cluster.sync();                           // no CTA still reads another's shared memory
    if (my_hist) clear_row_hist(my_hist, crank, cs);
    if (crank == 0 && tid == 0) record_error(a.err, DSA_DEVERR_TOPK, row);
    return;
  }
  const uint32_t n_above_total = lvl_above, bcount = lvl_cnt;
  const uint32_t need0 = k - n_above_total;   // keys to take from the threshold bin

  if (bcount <= static_cast<uint32_t>(kCandCap)) {
    // ---- write the keys above the bin, gather the bin's keys into rank 0
    // both counts in one scan (each < 2^16 per CTA); the two slot atomics on rank 0 from two
    // warps, so that their round trips overlap
    uint32_t n_up = 0, n_in = 0;
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
      n_up += key[e] > bin_hi;
      n_in += key[e] >= bin_lo && key[e] <= bin_hi;
    }
    uint32_t tot;
    const uint32_t pre = block_exclusive_scan((n_up << 16) | n_in, warp_sums, tot);
    const uint32_t tot_up = tot >> 16, tot_in = tot & 0xFFFFu;
    if (tid == 0) base_above = tot_up ? atomicAdd(cnt_above0, tot_up) : 0u;
    if (tid == 32) base_cand = tot_in ? atomicAdd(cnt_cand0, tot_in) : 0u;
    __syncthreads();
    uint32_t iu = base_above + (pre >> 16), ic = base_cand + (pre & 0xFFFFu);
#pragma unroll
    for (int v = 0; v < EPT / 4; ++v) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t kk = key[v * 4 + e];
        const int pos = beg + (v * kThreads + tid) * 4 + e;
        if (kk > bin_hi) {
          if (iu < n_above_total) {
            oi[iu] = pos;
            os[iu] = key_to_float(kk);
          }
          ++iu;
        } else if (kk >= bin_lo && kk <= bin_hi) {
          if (ic < static_cast<uint32_t>(kCandCap)) {
            ck0[ic] = kk;
            ci0[ic] = pos;
          }
          ++ic;
        }
      }
    }
    cluster.sync();                           // rank 0 holds the whole bin; counters are final
    if (my_hist) clear_row_hist(my_hist, crank, cs);
    if (crank != 0) return;                   // nobody reads another CTA's memory after this point
    const bool above_ok = cnt_above == n_above_total && cnt_cand == bcount;
    const bool ok = rank0_select<false, kThreads>(cand_key, cand_idx, bcount, 0u, bin_lo, bin_hi, need0, n_above_total, oi, os, hist,
                                 warp_sums, &lvl_bin, &lvl_above, &lvl_cnt, &base_above, &base_cand);
    if ((!ok || !above_ok) && tid == 0) record_error(a.err, DSA_DEVERR_TOPK, row);
    return;
  }

  // ---- slow path (the threshold bin holds more keys than rank 0 can gather):
  // cluster-wide refinement over the registers, starting from the threshold bin
  uint32_t* hist0 = cluster.map_shared_rank(hist, 0);
  SelectState* st0 = cluster.map_shared_rank(&st, 0);
  SelectState s;
  s.lo = bin_lo;
  s.hi = bin_hi;
  s.need = need0;
  s.done = 0;
  cluster.sync();                             // every CTA has read the coarse histogram
  if (my_hist) clear_row_hist(my_hist, crank, cs);
  for (int level = 0; level < 8; ++level) {
    if (s.lo == s.hi) { s.done = 2; break; }
    const int bits = 32 - __clz(s.hi - s.lo);
    const int shift = bits > 11 ? bits - 11 : 0;
    cluster.sync();                           // no CTA still reads the previous histograms
    for (int b = tid; b < kBins; b += kThreads) hist[b] = 0u;
    cluster.sync();                           // every histogram (rank 0's above all) is clear
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
      const uint32_t kk = key[e];
      if (kk >= s.lo && kk <= s.hi) atomicAdd(&hist[(kk - s.lo) >> shift], 1u);
    }
    if (cs > 1) {
      __syncthreads();
      if (crank != 0)
        for (int b = tid; b < kBins; b += kThreads)
          if (hist[b]) atomicAdd(&hist0[b], hist[b]);
    }
    cluster.sync();                           // rank 0 holds the merged histogram
    if (crank == 0) {
      uint32_t c[kBinsPerThread];
#pragma unroll
      for (int j = 0; j < kBinsPerThread; ++j) c[j] = hist[kBins - 1 - (tid * kBinsPerThread + j)];
      if (tid == 0) lvl_bin = kNotFound;
      find_threshold_bin<kBinsPerThread>(c, kBins - 1 - tid * kBinsPerThread, s.need, warp_sums, &lvl_bin,
                                         &lvl_above, &lvl_cnt);
      __syncthreads();
      if (tid == 0 && lvl_bin == kNotFound) {
        SelectState bad = s;
        bad.done = 3;                         // inconsistent counts: every CTA stops below
        st = bad;
      } else if (tid == 0) {
        SelectState ns;
        ns.lo = s.lo + (lvl_bin << shift);
        const uint32_t width_m1 = (1u << shift) - 1u;
        ns.hi = (s.hi - ns.lo) > width_m1 ? ns.lo + width_m1 : s.hi;
        ns.need = s.need - lvl_above;
        ns.done = lvl_cnt == ns.need ? 1u : 0u;
        st = ns;
      }
    }
    cluster.sync();                           // rank 0 published the new state
    s = *st0;
    if (s.done) break;
  }
  if (!s.done) s.done = 2;
  if (s.done == 3) {
    cluster.sync();                           // no CTA still reads rank 0's state
    if (crank == 0 && tid == 0) record_error(a.err, DSA_DEVERR_TOPK, row);
    return;
  }

  uint32_t n_up = 0, n_in = 0;
#pragma unroll
  for (int e = 0; e < EPT; ++e) {
    n_up += key[e] > s.hi;
    n_in += (key[e] >= s.lo && key[e] <= s.hi);
  }
  uint32_t tot_up, tot_in;
  const uint32_t pre_up = block_exclusive_scan(n_up, warp_sums, tot_up);
  const uint32_t pre_in = block_exclusive_scan(n_in, warp_sums, tot_in);
  if (tid == 0) {
    base_above = tot_up ? atomicAdd(cnt_above0, tot_up) : 0u;
    base_cand = tot_in ? atomicAdd(cnt_cand0, tot_in) : 0u;
  }
  __syncthreads();
  const uint32_t n_sel_above = k - s.need;
  uint32_t iu = base_above + pre_up, ic = base_cand + pre_in;
#pragma unroll
  for (int v = 0; v < EPT / 4; ++v) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t kk = key[v * 4 + e];
      const int pos = beg + (v * kThreads + tid) * 4 + e;
      if (kk > s.hi) {
        if (iu < n_sel_above) {
          oi[iu] = pos;
          os[iu] = key_to_float(kk);
        }
        ++iu;
      } else if (kk >= s.lo && kk <= s.hi) {
        if (ic < s.need) {
          oi[n_sel_above + ic] = pos;
          os[n_sel_above + ic] = key_to_float(kk);
        }
        ++ic;
      }
    }
  }
  cluster.sync();                             // counters final; no CTA leaves while others read its smem
  if (crank == 0 && tid == 0) {
    const bool bad = cnt_above != n_sel_above || cnt_cand < s.need || (s.done == 1 && cnt_cand != s.need);
    if (bad) record_error(a.err, DSA_DEVERR_TOPK, row);
  }
}

// ---- streaming top-k for rows whose coarse histogram the logits epilogue built.
// The histogram fixes, before any score is read, the bin B that holds the k-th largest
// key and the number of keys above B, so a row's keys need not meet in one place: every
// CTA streams one chunk of kStreamChunk scores, writes the keys above B straight to the
// row's output (slots from a per-row counter), appends the keys inside B to the row's
// candidate buffer and counts them in a per-row level-1 histogram of B (2048 sub-bins).
// Only the candidates and their counts must be visible before a chunk takes its ticket; the
// keys above B are written after it.  The CTA that finishes a row's last chunk reads that
// histogram, finds the sub-bin S of the remaining keys, takes the candidates above S in one
// pass and selects inside S in shared memory.  No CTA waits for another.
constexpr int kStreamThreads = 256;
constexpr int kStreamEPT = kStreamChunk / kStreamThreads;
constexpr int kStreamPer0 = kHistBins / kStreamThreads;  // coarse histogram bins per thread
constexpr int kStreamPer1 = kBins / kStreamThreads;      // level-1 histogram bins per thread
constexpr int kSubShift = kHistShift - 11;               // level-1 sub-bin width 2^kSubShift
constexpr int kSubCap = 1024;                            // sub-bin keys held in shared memory
static_assert(kStreamEPT % 4 == 0 && kStreamPer0 % 4 == 0 && kStreamPer1 % 4 == 0, "chunk and histogram split");
static_assert((1u << (kHistShift - kSubShift)) == static_cast<uint32_t>(kBins), "one level-1 bin per sub-bin");

__global__ void __launch_bounds__(kStreamThreads) topk_stream_kernel(const TopkArgs a) {
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t sub_key[kSubCap];
  __shared__ int32_t sub_idx[kSubCap];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t lvl_bin, lvl_above, lvl_cnt, ctr_a, ctr_b;
  __shared__ unsigned long long bases;
  __shared__ int is_last;
  const int tid = threadIdx.x;
  const TopkChunk ch = a.chunks[blockIdx.x];
  const int row = ch.row;
  const int n = a.row_pos[row] + 1;
  const int64_t off = a.row_off[row];
  const float* src = a.scores + off;
  const uint32_t k = static_cast<uint32_t>(a.top_k);
  int32_t* oi = a.out_idx + static_cast<int64_t>(row) * a.top_k;
  float* os = a.out_score + static_cast<int64_t>(row) * a.top_k;
  // row counters: [0] bin keys gathered, [1] keys written above the bin (one 64-bit word), [2] chunks done
  uint32_t* ctr = a.row_ctr + 4 * static_cast<int64_t>(row);
  uint32_t* sub_hist = a.row_hist1 + static_cast<int64_t>(row) * kBins;
  // the CTA that takes the row's last ticket leaves the row's histograms and counters clear
  // for the next call (every other CTA of the row has read them before its ticket)
  auto clear_row_state = [&]() {
    clear_row_hist(const_cast<uint32_t*>(a.row_hist) + static_cast<int64_t>(row) * kHistBins, 0, 1);
    for (int b = tid; b < kBins; b += kStreamThreads) sub_hist[b] = 0u;
    if (tid < 4) ctr[tid] = 0u;
  };
  if (tid == 0) lvl_bin = kNotFound;          // published by the scan's barriers below
  grid_dependency_wait();                     // scores and histograms come from the previous kernel

  uint32_t c0[kStreamPer0];
  load_bins_desc<kStreamPer0>(a.row_hist + static_cast<int64_t>(row) * kHistBins + (kHistBins - kStreamPer0 * (tid + 1)),
                              c0);
  uint32_t key[kStreamEPT];
#pragma unroll
  for (int v = 0; v < kStreamEPT / 4; ++v) {
    const int i = ch.begin + (v * kStreamThreads + tid) * 4;
    float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < ch.end) f = __ldcs(reinterpret_cast<const float4*>(src + i));
    const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) key[v * 4 + e] = (i + e < ch.end) ? float_to_key(fv[e]) : 0u;
  }
  find_threshold_bin<kStreamPer0>(c0, kHistBins - 1 - kStreamPer0 * tid, k, warp_sums, &lvl_bin, &lvl_above,
                                  &lvl_cnt);
  __syncthreads();
  if (lvl_bin == kNotFound) {
    // fewer than top_k keys counted for a row longer than top_k: every CTA of the row
    // lands here; nothing is written, the last one clears the row's state
    if (tid == 0) {
      if (ch.begin == 0) record_error(a.err, DSA_DEVERR_TOPK, row);
      is_last = atomicAdd(ctr + 2, 1u) == static_cast<uint32_t>(ch.n_chunks - 1);
    }
    __syncthreads();
    if (is_last) {
      __threadfence();
      clear_row_state();
    }
    return;
  }
  const uint32_t bin_lo = lvl_bin << kHistShift;
  const uint32_t bin_hi = bin_lo | ((1u << kHistShift) - 1u);
  const uint32_t n_above_total = lvl_above, bcount = lvl_cnt;
  const uint32_t cap = min(bcount, static_cast<uint32_t>(n));   // the row's candidate room is >= n

  // one scan of both counts (each < 2^16 per CTA) and one 64-bit atomic for both bases
  uint32_t n_up = 0, n_in = 0;
#pragma unroll
  for (int e = 0; e < kStreamEPT; ++e) {
    n_up += key[e] > bin_hi;
    n_in += key[e] >= bin_lo && key[e] <= bin_hi;
  }
  uint32_t tot;
  const uint32_t pre = block_exclusive_scan((n_up << 16) | n_in, warp_sums, tot);
  if (tid == 0)
    bases = tot ? atomicAdd(reinterpret_cast<unsigned long long*>(ctr),
                            (static_cast<unsigned long long>(tot >> 16) << 32) | (tot & 0xFFFFu))
                : 0ull;
  __syncthreads();
  uint32_t ic = static_cast<uint32_t>(bases) + (pre & 0xFFFFu);
#pragma unroll
  for (int v = 0; v < kStreamEPT / 4; ++v) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t kk = key[v * 4 + e];
      if (kk >= bin_lo && kk <= bin_hi) {
        if (ic < cap) {
          a.cand_key[off + ic] = kk;
          a.cand_idx[off + ic] = ch.begin + (v * kStreamThreads + tid) * 4 + e;
        }
        ++ic;
        atomicAdd(sub_hist + ((kk - bin_lo) >> kSubShift), 1u);
      }
    }
  }
  __threadfence();                            // this chunk's candidates before its ticket
  __syncthreads();
  if (tid == 0) is_last = atomicAdd(ctr + 2, 1u) == static_cast<uint32_t>(ch.n_chunks - 1);
  // the keys above the bin: nobody reads them in this kernel
  uint32_t iu = static_cast<uint32_t>(bases >> 32) + (pre >> 16);
#pragma unroll
  for (int v = 0; v < kStreamEPT / 4; ++v) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t kk = key[v * 4 + e];
      if (kk > bin_hi) {
        if (iu < n_above_total) {
          oi[iu] = ch.begin + (v * kStreamThreads + tid) * 4 + e;
          os[iu] = key_to_float(kk);
        }
        ++iu;
      }
    }
  }
  __syncthreads();
  if (!is_last) return;

  // ---- the row's last chunk: every other chunk's writes are visible after this fence
  __threadfence();
  const unsigned long long got = __ldcg(reinterpret_cast<const unsigned long long*>(ctr));
  if (static_cast<uint32_t>(got >> 32) != n_above_total || static_cast<uint32_t>(got) != bcount) {
    if (tid == 0) record_error(a.err, DSA_DEVERR_TOPK, row);
    __syncthreads();                          // every thread has read the counters
    clear_row_state();
    return;
  }
  const uint32_t need0 = k - n_above_total;
  if (tid == 0) lvl_bin = kNotFound;
  uint32_t c1[kStreamPer1];
  load_bins_desc<kStreamPer1>(sub_hist + (kBins - kStreamPer1 * (tid + 1)), c1);
  find_threshold_bin<kStreamPer1>(c1, kBins - 1 - kStreamPer1 * tid, need0, warp_sums, &lvl_bin, &lvl_above,
                                  &lvl_cnt);
  __syncthreads();
  if (lvl_bin == kNotFound) {
    if (tid == 0) record_error(a.err, DSA_DEVERR_TOPK, row);
    clear_row_state();
    return;
  }
  const uint32_t above1 = lvl_above, cnt1 = lvl_cnt;
  const uint32_t sub_lo = bin_lo + (lvl_bin << kSubShift);
  const uint32_t sub_hi = sub_lo + ((1u << kSubShift) - 1u);
  bool ok;
  if (cnt1 <= static_cast<uint32_t>(kSubCap)) {
    if (tid == 0) {
      ctr_a = 0u;
      ctr_b = 0u;
    }
    __syncthreads();
    // slots per warp: one shared atomic per counter and warp instead of one per key (every
    // thread calls f the same number of times, so the ballots see the whole warp)
    const uint32_t lane_lt = (1u << (tid & 31)) - 1u;
    for_candidates<true, true, kStreamThreads, 8>(a.cand_key + off, a.cand_idx + off, bcount,
                                                   [&](uint32_t kk, int32_t ix, bool valid) {
      const bool up = valid && kk > sub_hi;
      const bool in = valid && !up && kk >= sub_lo;
      const uint32_t bu = __ballot_sync(0xffffffffu, up), bi = __ballot_sync(0xffffffffu, in);
      uint32_t tu = 0u, ti = 0u;
      if ((tid & 31) == 0) {
        if (bu) tu = atomicAdd(&ctr_a, static_cast<uint32_t>(__popc(bu)));
        if (bi) ti = atomicAdd(&ctr_b, static_cast<uint32_t>(__popc(bi)));
      }
      tu = __shfl_sync(0xffffffffu, tu, 0) + __popc(bu & lane_lt);
      ti = __shfl_sync(0xffffffffu, ti, 0) + __popc(bi & lane_lt);
      if (up && tu < above1) {
        oi[n_above_total + tu] = ix;
        os[n_above_total + tu] = key_to_float(kk);
      } else if (in && ti < static_cast<uint32_t>(kSubCap)) {
        sub_key[ti] = kk;
        sub_idx[ti] = ix;
      }
    });
    __syncthreads();
    const bool pass_ok = ctr_a == above1 && ctr_b == cnt1;
    __syncthreads();                          // every thread has read the counters
    ok = pass_ok && rank0_select<false, kStreamThreads>(sub_key, sub_idx, cnt1, 0u, sub_lo, sub_hi, need0 - above1,
                                                         n_above_total + above1, oi, os, hist, warp_sums, &lvl_bin,
                                                         &lvl_above, &lvl_cnt, &ctr_a, &ctr_b);
  } else {
    // a crowded sub-bin (many equal scores): refine over all the row's candidates
    ok = rank0_select<true, kStreamThreads>(a.cand_key + off, a.cand_idx + off, bcount, 0u, bin_lo, bin_hi, need0,
                                            n_above_total, oi, os, hist, warp_sums, &lvl_bin, &lvl_above, &lvl_cnt,
                                            &ctr_a, &ctr_b);
  }
  if (!ok && tid == 0) record_error(a.err, DSA_DEVERR_TOPK, row);
  clear_row_state();                          // the level-1 counts were read before the select
}

// ---- row-streaming top-k (prefill: many rows, no histogram from the logits kernel).
// One CTA per row, several CTAs per SM; the row is streamed from memory in passes of
// kRowIter keys with the next iteration's loads in flight, nothing held across passes.
// Sampled first try (rows longer than kRowCap): one key in 16 (a float4 per 64 keys) is
// read into shared memory; a histogram over the sample's own key range gives a threshold
// tau expected to leave about 1.25 k + 64 keys at or above it; one pass with one float
// compare per key gathers those keys into shared memory, and if there are between k and
// kRowCap of them the exact select runs on that set (the k largest keys of the row are all
// >= tau whenever at least k keys are).  Otherwise, and for rows it does not apply to:
//   pass 1: a shared-memory histogram of the top 12 key bits gives the bin B holding the
//           k-th largest key, the number of keys above it and the number inside it;
//   refinement passes (only while B holds more than kRowCap keys and several values):
//           histogram of B's keys over 2048 sub-bins, B narrows to the sub-bin;
//   final pass: when the keys above B and inside B fit in shared memory together (the
//           usual case), every key >= B's lower edge is gathered there; otherwise keys
//           above B go straight to the output and B's keys are gathered, or, when B is one
//           tied value, the first `need` of them are written directly; slots come from a
//           warp scan of the per-thread counts and one 64-bit shared atomic per warp and
//           iteration (direct writes: high word, gathered: low word);
//   the gathered keys are resolved with exact shared-memory levels.
constexpr int kRowThreads = 256;
constexpr int kRowEPT = 16;                               // keys per thread per iteration
constexpr int kRowIter = kRowThreads * kRowEPT;
constexpr int kRowCap = 4096;                             // interval keys gathered in shared memory
constexpr int kRowShift0 = 20;                            // first level: 4096 bins of the top 12 bits
constexpr int kRowBins0 = 1 << (32 - kRowShift0);
constexpr size_t kRowSmemBytes = (kRowBins0 + 2 * kRowCap) * sizeof(uint32_t);
// The row streams from HBM with only one iteration of loads in flight per thread; the L2 is
// asked for the row kRowAhead iterations ahead (one bulk prefetch per iteration, by one
// thread), so the loads find the row there instead of waiting on HBM.
constexpr int kRowAhead = 3;

// Bulk L2 prefetch of iteration `it` of a row of n keys (the row's storage is n rounded up to
// 4 floats, so the prefetch never leaves it).
__device__ __forceinline__ void row_prefetch(const float* src, int n, int it) {
  const int first = it * kRowIter;
  if (first >= n) return;
  const int last = min(n, first + kRowIter);
  const uint32_t bytes = static_cast<uint32_t>(((last - first + 3) & ~3) * sizeof(float));
  l2_prefetch_bulk(src + first, bytes);
}
static_assert(kRowBins0 % kRowThreads == 0 && kBins % kRowThreads == 0, "bins per thread");

__device__ __forceinline__ void row_load(const float* src, int n, int base, float4 (&f)[kRowEPT / 4]) {
#pragma unroll
  for (int v = 0; v < kRowEPT / 4; ++v) {
    const int i = base + (v * kRowThreads + static_cast<int>(threadIdx.x)) * 4;
    f[v] = i < n ? __ldcs(reinterpret_cast<const float4*>(src + i)) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// The sampled first try described above; returns true when it handled the row (a broken
// count invariant is recorded in *err).  All threads of the CTA call it and get the same
// answer; on false nothing has been written.
__device__ bool row_sampled_select(const float* src, int n, uint32_t k, int32_t* oi, float* os, uint32_t* hist,
                                   uint32_t* cand_key, int32_t* cand_idx, uint32_t* warp_sums, uint32_t* lvl_bin,
                                   uint32_t* lvl_above, uint32_t* lvl_cnt, uint32_t* ctr_a, uint32_t* ctr_b,
                                   uint32_t* ctr_c, int* err, int row) {
  const int tid = threadIdx.x, lane = tid & 31;
  // ---- sample: the first float4 of every `block` keys (block a multiple of 64, s <= kRowCap)
  const int block = 64 * ((n + 65535) / 65536);
  const int n_blocks = (n + block - 1) / block;
  uint32_t smin = 0xFFFFFFFFu, smax = 0u, s_local = 0u;
  constexpr int kSampleLoads = kRowCap / 4 / kRowThreads;   // n_blocks <= kRowCap / 4
  float4 sf[kSampleLoads];
#pragma unroll
  for (int j = 0; j < kSampleLoads; ++j) {                  // every load in flight before any is used
    const int b = tid + j * kRowThreads;
    sf[j] = b < n_blocks ? __ldcs(reinterpret_cast<const float4*>(src + b * block)) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int j = 0; j < kSampleLoads; ++j) {
    const int b = tid + j * kRowThreads;
    if (b >= n_blocks) break;
    const int i = b * block;
    const float fv[4] = {sf[j].x, sf[j].y, sf[j].z, sf[j].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const bool valid = i + e < n;
      const uint32_t kk = float_to_key(fv[e]);
      cand_key[4 * b + e] = valid ? kk : 0u;
      if (valid) {
        smin = min(smin, kk);
        smax = max(smax, kk);
        ++s_local;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    smin = min(smin, __shfl_xor_sync(0xffffffffu, smin, o));
    smax = max(smax, __shfl_xor_sync(0xffffffffu, smax, o));
  }
  if (tid == 0) {
    *ctr_a = 0xFFFFFFFFu;                     // sample min
    *ctr_b = 0u;                              // sample max
  }
  for (int b = tid; b < kBins; b += kRowThreads) hist[b] = 0u;
  uint32_t s_valid;
  block_exclusive_scan(s_local, warp_sums, s_valid);       // also orders the resets above
  if (lane == 0) {
    atomicMin(ctr_a, smin);
    atomicMax(ctr_b, smax);
  }
  __syncthreads();
  const uint32_t lo_s = *ctr_a, hi_s = *ctr_b;
  const int bits = hi_s > lo_s ? 32 - __clz(hi_s - lo_s) : 0;
  const int shift = bits > 11 ? bits - 11 : 0;
  for (int i = tid; i < 4 * n_blocks; i += kRowThreads) {
    const uint32_t kk = cand_key[i];
    if (i < 4 * n_blocks && ((i & 3) + (i >> 2) * block) < n) atomicAdd(&hist[(kk - lo_s) >> shift], 1u);
  }
  // sample rank of tau: about (1.25 k + 64) keys of the row expected at or above it
  const uint32_t r = static_cast<uint32_t>(
      (static_cast<unsigned long long>(k + k / 4 + 64) * s_valid + static_cast<unsigned long long>(n) - 1) /
      static_cast<unsigned long long>(n));
  if (tid == 0) *lvl_bin = kNotFound;
  {
    constexpr int PER = kBins / kRowThreads;
    uint32_t c[PER];
    __syncthreads();
#pragma unroll
    for (int j = 0; j < PER; ++j) c[j] = hist[kBins - 1 - (tid * PER + j)];
    find_threshold_bin<PER>(c, kBins - 1 - tid * PER, r, warp_sums, lvl_bin, lvl_above, lvl_cnt);
  }
  __syncthreads();
  if (*lvl_bin == kNotFound) return false;    // the sample holds fewer than r keys
  const uint32_t tau = lo_s + (*lvl_bin << shift);
  const float tau_f = key_to_float(tau);
  if (tid == 0) *ctr_a = 0u;                  // gathered keys
  __syncthreads();

  // ---- one pass: every key >= tau into shared memory (slots: warp scan + one atomic per
  // warp).  {f >= tau_f} is closed upwards in key order (key order refines float order), so it
  // holds the k largest keys as soon as it has k elements.
  float4 cur[kRowEPT / 4];
  row_load(src, n, 0, cur);
  // the histogram is idle during this pass: it stages each iteration's scores (kRowIter floats)
  float* stage = reinterpret_cast<float*>(hist);
  static_assert(kRowIter <= kRowBins0, "one iteration's scores fit the histogram buffer");
  auto gather = [&](auto tail, int base) {
    constexpr bool kTail = decltype(tail)::value;   // the last iteration: positions past n exist
#pragma unroll
    for (int v = 0; v < kRowEPT / 4; ++v)
      *reinterpret_cast<float4*>(stage + (v * kRowThreads + tid) * 4) = cur[v];
    uint32_t sel = 0u;
#pragma unroll
    for (int v = 0; v < kRowEPT / 4; ++v) {
      const float fv[4] = {cur[v].x, cur[v].y, cur[v].z, cur[v].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool hit = fv[e] >= tau_f && (!kTail || base + (v * kRowThreads + tid) * 4 + e < n);
        sel |= static_cast<uint32_t>(hit) << (v * 4 + e);
      }
    }
    const uint32_t mine = __popc(sel);
    uint32_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    uint32_t wbase = 0u;
    if (lane == 31 && incl) wbase = atomicAdd(ctr_a, incl);
    uint32_t slot = __shfl_sync(0xffffffffu, wbase, 31) + incl - mine;
    // the selected keys, bit by bit: their values come back from this thread's own staged copy
    // (written above, read by the same thread: no barrier needed)
    while (sel) {
      const int j = __ffs(sel) - 1;
      sel &= sel - 1u;
      if (slot < static_cast<uint32_t>(kRowCap)) {
        const int local = ((j >> 2) * kRowThreads + tid) * 4 + (j & 3);
        cand_key[slot] = float_to_key(stage[local]);
        cand_idx[slot] = base + local;
      }
      ++slot;
    }
  };
  int base = 0;
  for (; base + kRowIter < n; base += kRowIter) {        // every position of this iteration is < n
    if (tid == 0) row_prefetch(src, n, base / kRowIter + kRowAhead);
    float4 nxt[kRowEPT / 4];
    row_load(src, n, base + kRowIter, nxt);
    gather(std::false_type{}, base);
#pragma unroll
    for (int v = 0; v < kRowEPT / 4; ++v) cur[v] = nxt[v];
  }
  gather(std::true_type{}, base);
  __syncthreads();
  const uint32_t c = *ctr_a;
  if (c < k || c > static_cast<uint32_t>(kRowCap)) return false;   // tau missed: exact passes instead
  // the gathered keys' range
  uint32_t my_max = 0u, my_min = 0xFFFFFFFFu;
  for (uint32_t i = tid; i < c; i += kRowThreads) {
    const uint32_t kk = cand_key[i];
    my_max = max(my_max, kk);
    my_min = min(my_min, kk);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    my_max = max(my_max, __shfl_xor_sync(0xffffffffu, my_max, o));
    my_min = min(my_min, __shfl_xor_sync(0xffffffffu, my_min, o));
  }
  if (tid == 0) {
    *ctr_b = 0u;                              // largest gathered key
    *ctr_c = 0xFFFFFFFFu;                     // smallest gathered key
  }
  __syncthreads();
  if (lane == 0) {
    atomicMax(ctr_b, my_max);
    atomicMin(ctr_c, my_min);
  }
  __syncthreads();
  const uint32_t kmax = *ctr_b, kmin = *ctr_c;
  __syncthreads();                            // every thread has read the counters
  const bool ok = rank0_select<false, kRowThreads>(cand_key, cand_idx, c, 0u, kmin, kmax, k, 0u, oi, os, hist,
                                                   warp_sums, lvl_bin, lvl_above, lvl_cnt, ctr_a, ctr_b);
  if (!ok && tid == 0) record_error(err, DSA_DEVERR_TOPK, row);
  return true;
}

__global__ void __launch_bounds__(kRowThreads, 4) topk_row_kernel(const TopkArgs a) {
  extern __shared__ __align__(16) uint32_t rsm[];
  uint32_t* hist = rsm;                                   // kRowBins0 (levels >= 1 use the first kBins)
  uint32_t* cand_key = rsm + kRowBins0;                   // kRowCap
  int32_t* cand_idx = reinterpret_cast<int32_t*>(cand_key + kRowCap);
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t lvl_bin, lvl_above, lvl_cnt, ctr_a, ctr_b, ctr_c;
  __shared__ unsigned long long slot_ctr;
  const int tid = threadIdx.x, lane = tid & 31;
  const int row = a.rows[blockIdx.x];
  const int n = a.row_pos[row] + 1;                       // n > top_k
  const float* src = a.scores + a.row_off[row];
  const uint32_t k = static_cast<uint32_t>(a.top_k);
  int32_t* oi = a.out_idx + static_cast<int64_t>(row) * a.top_k;
  float* os = a.out_score + static_cast<int64_t>(row) * a.top_k;

  uint32_t lo = 0u, hi = 0xFFFFFFFFu;                     // interval holding the keys still to choose
  uint32_t need = k;                                      // keys still to take from [lo, hi]
  uint32_t cnt = static_cast<uint32_t>(n);                // keys inside [lo, hi]
  int shift = kRowShift0;
  grid_dependency_wait();                                 // the scores come from the previous kernel
  if (tid == 0)
    for (int it = 0; it < kRowAhead; ++it) row_prefetch(src, n, it);
  if (n > kRowCap && k <= static_cast<uint32_t>(kRowCap) / 2 &&
      row_sampled_select(src, n, k, oi, os, hist, cand_key, cand_idx, warp_sums, &lvl_bin, &lvl_above, &lvl_cnt,
                         &ctr_a, &ctr_b, &ctr_c, a.err, row))
    return;
  for (int level = 0;; ++level) {
    const bool final_pass = cnt <= static_cast<uint32_t>(kRowCap) || lo == hi || level >= 4;
    const int nbins = level == 0 ? kRowBins0 : kBins;
    if (!final_pass)
      for (int b = tid; b < nbins; b += kRowThreads) hist[b] = 0u;
    if (tid == 0) {
      slot_ctr = 0ull;
      lvl_bin = kNotFound;
    }
    __syncthreads();
    const uint32_t n_sel_above = k - need;                // keys above hi, all selected
    const bool gather_all = n_sel_above + cnt <= static_cast<uint32_t>(kRowCap);
    float4 cur[kRowEPT / 4];
    row_load(src, n, 0, cur);
    for (int base = 0; base < n; base += kRowIter) {
      if (tid == 0) row_prefetch(src, n, base / kRowIter + kRowAhead);
      float4 nxt[kRowEPT / 4];
      if (base + kRowIter < n) {
        row_load(src, n, base + kRowIter, nxt);
      } else {
#pragma unroll
        for (int v = 0; v < kRowEPT / 4; ++v) nxt[v] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      if (!final_pass) {
#pragma unroll
        for (int v = 0; v < kRowEPT / 4; ++v) {
          const float fv[4] = {cur[v].x, cur[v].y, cur[v].z, cur[v].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int pos = base + (v * kRowThreads + tid) * 4 + e;
            const uint32_t kk = float_to_key(fv[e]);
            if (pos < n && kk >= lo && kk <= hi) atomicAdd(&hist[(kk - lo) >> shift], 1u);
          }
        }
      } else {
        uint32_t up_mask = 0u, in_mask = 0u;              // bit j: key j is above / inside [lo, hi]
#pragma unroll
        for (int v = 0; v < kRowEPT / 4; ++v) {
          const float fv[4] = {cur[v].x, cur[v].y, cur[v].z, cur[v].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const bool valid = base + (v * kRowThreads + tid) * 4 + e < n;
            const uint32_t kk = float_to_key(fv[e]);
            up_mask |= static_cast<uint32_t>(!gather_all && valid && kk > hi) << (v * 4 + e);
            in_mask |= static_cast<uint32_t>(valid && kk >= lo && (gather_all || kk <= hi)) << (v * 4 + e);
          }
        }
        const unsigned long long mine = (static_cast<unsigned long long>(__popc(up_mask)) << 32) | __popc(in_mask);
        unsigned long long incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        unsigned long long wbase = 0ull;
        if (lane == 31 && incl) wbase = atomicAdd(&slot_ctr, incl);
        wbase = __shfl_sync(0xffffffffu, wbase, 31) + (incl - mine);
        uint32_t iu = static_cast<uint32_t>(wbase >> 32), ic = static_cast<uint32_t>(wbase);
#pragma unroll
        for (int v = 0; v < kRowEPT / 4; ++v) {
          const float fv[4] = {cur[v].x, cur[v].y, cur[v].z, cur[v].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t kk = float_to_key(fv[e]);
            const int pos = base + (v * kRowThreads + tid) * 4 + e;
            if ((up_mask >> (v * 4 + e)) & 1u) {
              if (iu < n_sel_above) {
                oi[iu] = pos;
                os[iu] = key_to_float(kk);
              }
              ++iu;
            } else if ((in_mask >> (v * 4 + e)) & 1u) {
              if (lo == hi && !gather_all) {              // one tied value: any `need` of them
                if (ic < need) {
                  oi[n_sel_above + ic] = pos;
                  os[n_sel_above + ic] = key_to_float(kk);
                }
              } else if (ic < static_cast<uint32_t>(kRowCap)) {
                cand_key[ic] = kk;
                cand_idx[ic] = pos;
              }
              ++ic;
            }
          }
        }
      }
#pragma unroll
      for (int v = 0; v < kRowEPT / 4; ++v) cur[v] = nxt[v];
    }
    __syncthreads();
    if (final_pass) {
      const uint32_t direct = gather_all ? 0u : n_sel_above, gathered = gather_all ? n_sel_above + cnt : cnt;
      bool ok = static_cast<uint32_t>(slot_ctr >> 32) == direct && static_cast<uint32_t>(slot_ctr) == gathered;
      __syncthreads();                                    // every thread has read the counters
      if (ok && (gather_all || lo != hi)) {
        if (gathered > static_cast<uint32_t>(kRowCap)) {
          ok = false;                                     // unreachable: four levels resolve 32 bits
        } else {
          ok = rank0_select<false, kRowThreads>(cand_key, cand_idx, gathered, n_sel_above - direct, lo, hi, need,
                                                direct, oi, os, hist, warp_sums, &lvl_bin, &lvl_above, &lvl_cnt,
                                                &ctr_a, &ctr_b);
        }
      }
      if (!ok && tid == 0) record_error(a.err, DSA_DEVERR_TOPK, row);
      return;
    }
    // the bin of the need-th largest key inside [lo, hi]
    if (level == 0) {
      constexpr int PER = kRowBins0 / kRowThreads;
      uint32_t c[PER];
#pragma unroll
      for (int j = 0; j < PER; ++j) c[j] = hist[kRowBins0 - 1 - (tid * PER + j)];
      find_threshold_bin<PER>(c, kRowBins0 - 1 - tid * PER, need, warp_sums, &lvl_bin, &lvl_above, &lvl_cnt);
    } else {
      constexpr int PER = kBins / kRowThreads;
      uint32_t c[PER];
#pragma unroll
      for (int j = 0; j < PER; ++j) c[j] = hist[kBins - 1 - (tid * PER + j)];
      find_threshold_bin<PER>(c, kBins - 1 - tid * PER, need, warp_sums, &lvl_bin, &lvl_above, &lvl_cnt);
    }
    __syncthreads();
    if (lvl_bin == kNotFound) {
      if (tid == 0) record_error(a.err, DSA_DEVERR_TOPK, row);
      return;
    }
    const uint32_t nlo = lo + (lvl_bin << shift);
    const uint32_t width_m1 = (1u << shift) - 1u;
    hi = (hi - nlo) > width_m1 ? nlo + width_m1 : hi;
    lo = nlo;
    need -= lvl_above;
    cnt = lvl_cnt;
    const int bits = lo == hi ? 0 : 32 - __clz(hi - lo);
    shift = bits > 11 ? bits - 11 : 0;
    __syncthreads();                                      // lvl_* read before the next level resets them
  }
}

// Coarse row histograms for decode configurations whose logits epilogue does not count
// them (FP8): one CTA per streaming chunk of kStreamChunk scores counts its keys' top bits in
// a shared histogram and adds the non-zero bins to the row's global histogram.
constexpr int kRowHistThreads = 256;
static_assert(kStreamChunk % (4 * kRowHistThreads) == 0, "whole float4 per thread and pass");

__global__ void __launch_bounds__(kRowHistThreads) row_hist_kernel(const TopkArgs a) {
  __shared__ uint32_t h[kHistBins];
  const int tid = threadIdx.x;
  for (int b = tid; b < kHistBins; b += kRowHistThreads) h[b] = 0u;
  const TopkChunk ch = a.chunks[blockIdx.x];
  const float* src = a.scores + a.row_off[ch.row];
  __syncthreads();
  grid_dependency_wait();                     // the scores come from the previous kernel
  constexpr int kPer = kStreamChunk / (4 * kRowHistThreads);
  float4 f[kPer];
#pragma unroll
  for (int v = 0; v < kPer; ++v) {            // every load in flight before any is counted
    const int i = ch.begin + (v * kRowHistThreads + tid) * 4;
    f[v] = i < ch.end ? __ldcg(reinterpret_cast<const float4*>(src + i)) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int v = 0; v < kPer; ++v) {
    const int i = ch.begin + (v * kRowHistThreads + tid) * 4;
    const float fv[4] = {f[v].x, f[v].y, f[v].z, f[v].w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (i + e < ch.end) atomicAdd(&h[float_to_key(fv[e]) >> kHistShift], 1u);
  }
  __syncthreads();
  uint32_t* row_hist = const_cast<uint32_t*>(a.row_hist) + static_cast<int64_t>(ch.row) * kHistBins;
  for (int b = tid; b < kHistBins; b += kRowHistThreads)
    if (h[b]) atomicAdd(row_hist + b, h[b]);
}

// Rows whose whole causal history fits in top_k: every position, then -1 / -inf.  Without
// out_score (the short-sequence bypass) only the positions are written and no score is read.
__global__ void __launch_bounds__(256) topk_short_kernel(const TopkArgs a) {
  grid_dependency_wait();                     // the scores come from the previous kernel
  const int row = a.rows[blockIdx.x];
  const int n = a.row_pos[row] + 1;
  int32_t* oi = a.out_idx + static_cast<int64_t>(row) * a.top_k;
  // decode: the logits epilogue counted this row too; leave its histogram clear for the next call
  if (a.row_hist) clear_row_hist(const_cast<uint32_t*>(a.row_hist) + static_cast<int64_t>(row) * kHistBins, 0, 1);
  if (!a.out_score) {
    for (int j = threadIdx.x; j < a.top_k; j += blockDim.x) oi[j] = j < n ? j : -1;
    return;
  }
  const float* src = a.scores + a.row_off[row];
  float* os = a.out_score + static_cast<int64_t>(row) * a.top_k;
  for (int j = threadIdx.x; j < a.top_k; j += blockDim.x) {
    if (j < n) {
      oi[j] = j;
      os[j] = src[j];
    } else {
      oi[j] = -1;
      os[j] = -INFINITY;
    }
  }
}

template <int EPT>
cudaError_t launch_ept(const TopkArgs& a, int cluster, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.n_rows) * cluster, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kTopkSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  static unsigned long long configured = 0;   // one bit per device ordinal
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(configured & (1ull << dev))) {
    e = cudaFuncSetAttribute(topk_kernel<EPT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kTopkSmemBytes));
    if (e != cudaSuccess) return e;
    if (dev < 64) configured |= 1ull << dev;
  }
  return cudaLaunchKernelEx(&cfg, topk_kernel<EPT>, a);
}

}  // namespace

cudaError_t launch_topk(const TopkArgs& a, int ept, int cluster, cudaStream_t stream) {
  if (a.n_rows <= 0) return cudaSuccess;
  switch (ept) {
    case 4: return launch_ept<4>(a, cluster, stream);
    case 8: return launch_ept<8>(a, cluster, stream);
    case 16: return launch_ept<16>(a, cluster, stream);
    case 32: return launch_ept<32>(a, cluster, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_topk_stream(const TopkArgs& a, cudaStream_t stream) {
  if (a.n_chunks <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.n_chunks), 1, 1);
  cfg.blockDim = dim3(kStreamThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, topk_stream_kernel, a);
}

cudaError_t launch_topk_rows(const TopkArgs& a, cudaStream_t stream) {
  if (a.n_rows <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.n_rows), 1, 1);
  cfg.blockDim = dim3(kRowThreads, 1, 1);
  cfg.dynamicSmemBytes = kRowSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static unsigned long long configured = 0;   // one bit per device ordinal
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(configured & (1ull << dev))) {
    e = cudaFuncSetAttribute(topk_row_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kRowSmemBytes));
    if (e != cudaSuccess) return e;
    if (dev < 64) configured |= 1ull << dev;
  }
  return cudaLaunchKernelEx(&cfg, topk_row_kernel, a);
}

cudaError_t launch_row_hist(const TopkArgs& a, cudaStream_t stream) {
  if (a.n_chunks <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.n_chunks), 1, 1);
  cfg.blockDim = dim3(kRowHistThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, row_hist_kernel, a);
}

cudaError_t launch_topk_short(const TopkArgs& a, cudaStream_t stream) {
  if (a.n_rows <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.n_rows), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, topk_short_kernel, a);
}

}  // namespace dsa
