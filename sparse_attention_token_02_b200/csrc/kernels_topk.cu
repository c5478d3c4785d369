// Per-row top-k selection over fp32 indexer scores (page "从原理到代码：手把手教你理解
// DeepSeek-V3.2的闪电索引器设计" §3 step 5, top-k per query; "Lightning Indexer 详解" §2.3:
// at most min(k, L) positions exist).
//
// Threshold select, exact, with the keys held in registers:
//   * one cluster of `cs` CTAs per row (distributed shared memory joins them); each
//     thread loads EPT scores of its CTA's slice with 16-byte loads and maps each to
//     an order-preserving uint32 key (larger float -> larger key);
//   * the cluster reduces min and max key -> candidate key interval [lo, hi];
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
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace dsa {

namespace {

constexpr int kThreads = kTopkThreads;
constexpr int kWarps = kThreads / 32;
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
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t s = lane < kWarps ? warp_sums[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < kWarps) warp_sums[lane] = s;   // inclusive warp prefix
  }
  __syncthreads();
  total = warp_sums[kWarps - 1];
  const uint32_t before = warp == 0 ? 0u : warp_sums[warp - 1];
  __syncthreads();                            // warp_sums may be reused right after
  return before + x - v;
}

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

template <int EPT>
__global__ void __launch_bounds__(kThreads, EPT <= 8 ? 2 : 1)
topk_kernel(const TopkArgs a) {
  static_assert(EPT % 4 == 0, "EPT is a multiple of 4");
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

  for (int b = tid; b < kBins; b += kThreads) hist[b] = 0u;
  if (tid == 0) {
    cnt_above = 0u;
    cnt_cand = 0u;
    loc_min = 0xFFFFFFFFu;
    loc_max = 0u;
  }
  __syncthreads();
  grid_dependency_wait();                     // the scores come from the previous kernel

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

  uint32_t bin_lo, bin_hi, n_above_total, bcount;
  if (a.row_hist != nullptr) {
    // ---- the logits epilogue already binned the row: the threshold bin comes straight
    // from its coarse histogram (this CTA's 8 bins: bins 4095-8t .. 4088-8t, descending)
    static_assert(kHistBins == 8 * kThreads, "the coarse histogram is read as 8 bins per thread");
    const uint32_t* h = a.row_hist + static_cast<int64_t>(row) * kHistBins + (kHistBins - 8 * (tid + 1));
    const uint4 h0 = *reinterpret_cast<const uint4*>(h);
    const uint4 h1 = *reinterpret_cast<const uint4*>(h + 4);
    const uint32_t c[8] = {h1.w, h1.z, h1.y, h1.x, h0.w, h0.z, h0.y, h0.x};
    cluster.sync();                           // #1: every CTA's counters are initialised
    find_threshold_bin<8>(c, kHistBins - 1 - 8 * tid, k, warp_sums, &lvl_bin, &lvl_above, &lvl_cnt);
    __syncthreads();
    bin_lo = lvl_bin << kHistShift;
    bin_hi = bin_lo | ((1u << kHistShift) - 1u);
    n_above_total = lvl_above;
    bcount = lvl_cnt;
  } else {
    // ---- first level from the data: bins spread over the row's key range
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
      kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    if (lane == 0) {
      atomicMin(&loc_min, kmin);
      atomicMax(&loc_max, kmax);
    }
    cluster.sync();                           // #1: every CTA's key range is published
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
    cluster.sync();                           // #2: every CTA's histogram is complete
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
    __syncthreads();
    bin_lo = lo + (lvl_bin << shift0);
    const uint32_t bin_w1 = (1u << shift0) - 1u;
    bin_hi = (hi - bin_lo) > bin_w1 ? bin_lo + bin_w1 : hi;
    n_above_total = lvl_above;
    bcount = lvl_cnt;
  }
  const uint32_t need0 = k - n_above_total;   // keys to take from the threshold bin

  if (bcount <= static_cast<uint32_t>(kCandCap)) {
    // ---- fast path: write the keys above the bin, gather the bin's keys into rank 0
    uint32_t n_up = 0, n_in = 0;
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
      n_up += key[e] > bin_hi;
      n_in += key[e] >= bin_lo && key[e] <= bin_hi;
    }
    uint32_t tot_up, tot_in;
    const uint32_t pre_up = block_exclusive_scan(n_up, warp_sums, tot_up);
    const uint32_t pre_in = block_exclusive_scan(n_in, warp_sums, tot_in);
    if (tid == 0) {
      base_above = tot_up ? atomicAdd(cnt_above0, tot_up) : 0u;
      base_cand = tot_in ? atomicAdd(cnt_cand0, tot_in) : 0u;
    }
    __syncthreads();
    uint32_t* ck0 = cluster.map_shared_rank(cand_key, 0);
    int32_t* ci0 = cluster.map_shared_rank(cand_idx, 0);
    uint32_t iu = base_above + pre_up, ic = base_cand + pre_in;
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
    if (crank != 0) return;                   // nobody reads another CTA's memory after this point

    // ---- rank 0 alone: pick need0 of the bcount gathered keys (exact, CTA-local levels)
    const uint32_t m = bcount;
    SelectState ls;
    ls.lo = bin_lo;
    ls.hi = bin_hi;
    ls.need = need0;
    ls.done = need0 == m ? 1u : 0u;
    for (int level = 0; level < 4 && !ls.done; ++level) {
      if (ls.lo == ls.hi) { ls.done = 2; break; }
      const int bits = 32 - __clz(ls.hi - ls.lo);
      const int shift = bits > 11 ? bits - 11 : 0;
      for (int b = tid; b < kBins; b += kThreads) hist[b] = 0u;
      __syncthreads();
      for (uint32_t i = tid; i < m; i += kThreads) {
        const uint32_t kk = cand_key[i];
        if (kk >= ls.lo && kk <= ls.hi) atomicAdd(&hist[(kk - ls.lo) >> shift], 1u);
      }
      __syncthreads();
      uint32_t c[kBinsPerThread];
#pragma unroll
      for (int j = 0; j < kBinsPerThread; ++j) c[j] = hist[kBins - 1 - (tid * kBinsPerThread + j)];
      find_threshold_bin<kBinsPerThread>(c, kBins - 1 - tid * kBinsPerThread, ls.need, warp_sums, &lvl_bin,
                                         &lvl_above, &lvl_cnt);
      __syncthreads();
      const uint32_t b2 = lvl_bin;
      SelectState ns;
      ns.lo = ls.lo + (b2 << shift);
      const uint32_t width_m1 = (1u << shift) - 1u;
      ns.hi = (ls.hi - ns.lo) > width_m1 ? ns.lo + width_m1 : ls.hi;
      ns.need = ls.need - lvl_above;
      ns.done = lvl_cnt == ns.need ? 1u : 0u;
      ls = ns;
      __syncthreads();
    }
    if (!ls.done) ls.done = 2;                // unreachable: >= 10 bits resolved per level
    // candidates above the final interval, then ls.need keys of the interval (ties: any)
    if (tid == 0) {
      cnt_above = 0u;                         // reused as slot counters for this CTA only
      cnt_cand = 0u;
    }
    __syncthreads();
    const uint32_t first_in = n_above_total + (need0 - ls.need);   // slots of interval keys start here
    for (uint32_t i = tid; i < m; i += kThreads) {
      const uint32_t kk = cand_key[i];
      if (kk > ls.hi) {
        const uint32_t slot = n_above_total + atomicAdd(&cnt_above, 1u);
        if (slot < first_in) {
          oi[slot] = cand_idx[i];
          os[slot] = key_to_float(kk);
        }
      } else if (kk >= ls.lo) {
        const uint32_t t = atomicAdd(&cnt_cand, 1u);
        if (t < ls.need) {
          oi[first_in + t] = cand_idx[i];
          os[first_in + t] = key_to_float(kk);
        }
      }
    }
    __syncthreads();
    if (tid == 0) {
      const bool bad = cnt_above != need0 - ls.need || cnt_cand < ls.need || (ls.done == 1 && cnt_cand != ls.need);
      if (bad) record_error(a.err, DSA_DEVERR_TOPK, row);
    }
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
      find_threshold_bin<kBinsPerThread>(c, kBins - 1 - tid * kBinsPerThread, s.need, warp_sums, &lvl_bin,
                                         &lvl_above, &lvl_cnt);
      __syncthreads();
      if (tid == 0) {
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

// Rows whose whole causal history fits in top_k: every position, then -1 / -inf.
__global__ void __launch_bounds__(256) topk_short_kernel(const TopkArgs a) {
  grid_dependency_wait();                     // the scores come from the previous kernel
  const int row = a.rows[blockIdx.x];
  const int n = a.row_pos[row] + 1;
  const float* src = a.scores + a.row_off[row];
  int32_t* oi = a.out_idx + static_cast<int64_t>(row) * a.top_k;
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
