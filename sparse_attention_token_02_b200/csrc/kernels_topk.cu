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

__device__ __forceinline__ uint32_t float_to_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

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

template <int EPT>
__global__ void __launch_bounds__(kThreads)
topk_kernel(const TopkArgs a) {
  static_assert(EPT % 4 == 0, "EPT is a multiple of 4");
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t red_min, red_max;
  __shared__ SelectState st;
  __shared__ uint32_t cnt_above, cnt_cand, base_above, base_cand;

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

  const int per = ((n + cs - 1) / cs + 3) & ~3;
  const int beg = crank * per;
  const int end = min(n, beg + per);

  uint32_t* hist0 = cluster.map_shared_rank(hist, 0);
  SelectState* st0 = cluster.map_shared_rank(&st, 0);
  uint32_t* red_min0 = cluster.map_shared_rank(&red_min, 0);
  uint32_t* red_max0 = cluster.map_shared_rank(&red_max, 0);
  uint32_t* cnt_above0 = cluster.map_shared_rank(&cnt_above, 0);
  uint32_t* cnt_cand0 = cluster.map_shared_rank(&cnt_cand, 0);

  if (tid == 0) {
    red_min = 0xFFFFFFFFu;
    red_max = 0u;
    cnt_above = 0u;
    cnt_cand = 0u;
  }

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
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  cluster.sync();                             // rank 0's reduction slots are initialised
  if (lane == 0) {
    atomicMin(red_min0, kmin);
    atomicMax(red_max0, kmax);
  }
  cluster.sync();
  SelectState s;
  s.lo = *red_min0;
  s.hi = *red_max0;
  s.need = k;
  s.done = 0;

  // ---- refinement levels
  for (int level = 0; level < 8; ++level) {
    if (s.lo == s.hi) { s.done = 2; break; }
    const uint32_t range = s.hi - s.lo;
    const int bits = 32 - __clz(range);
    const int shift = bits > 11 ? bits - 11 : 0;
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
      // thread t owns bins 2047-4t .. 2044-4t, highest first; scan gives the count above them
      uint32_t c[kBinsPerThread], sum = 0;
#pragma unroll
      for (int j = 0; j < kBinsPerThread; ++j) {
        c[j] = hist[kBins - 1 - (tid * kBinsPerThread + j)];
        sum += c[j];
      }
      uint32_t total;
      uint32_t above = block_exclusive_scan(sum, warp_sums, total);
#pragma unroll
      for (int j = 0; j < kBinsPerThread; ++j) {
        const uint32_t b = kBins - 1 - (tid * kBinsPerThread + j);
        if (above < s.need && above + c[j] >= s.need) {
          SelectState ns;
          ns.lo = s.lo + (b << shift);
          const uint32_t width_m1 = shift >= 32 ? 0xFFFFFFFFu : ((1u << shift) - 1u);
          ns.hi = (s.hi - ns.lo) > width_m1 ? ns.lo + width_m1 : s.hi;
          ns.need = s.need - above;
          ns.done = (c[j] == ns.need) ? 1u : 0u;
          st = ns;
        }
        above += c[j];
      }
    }
    cluster.sync();                           // rank 0 published the new state
    s = *st0;
    if (s.done) break;
  }
  if (!s.done) s.done = 2;                    // unreachable: each level narrows by 2^10

  // ---- output pass: keys above the interval, then `need` keys from the interval
  uint32_t n_above = 0, n_cand = 0;
#pragma unroll
  for (int e = 0; e < EPT; ++e) {
    n_above += key[e] > s.hi;
    n_cand += (key[e] >= s.lo && key[e] <= s.hi);
  }
  uint32_t tot_above, tot_cand;
  const uint32_t pre_above = block_exclusive_scan(n_above, warp_sums, tot_above);
  const uint32_t pre_cand = block_exclusive_scan(n_cand, warp_sums, tot_cand);
  if (tid == 0) {
    base_above = tot_above ? atomicAdd(cnt_above0, tot_above) : 0u;
    base_cand = tot_cand ? atomicAdd(cnt_cand0, tot_cand) : 0u;
  }
  __syncthreads();
  const uint32_t n_sel_above = k - s.need;    // slots [0, k-need) hold keys above hi
  uint32_t ia = base_above + pre_above, ic = base_cand + pre_cand;
  int32_t* oi = a.out_idx + static_cast<int64_t>(row) * a.top_k;
  float* os = a.out_score + static_cast<int64_t>(row) * a.top_k;
#pragma unroll
  for (int v = 0; v < EPT / 4; ++v) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t kk = key[v * 4 + e];
      const int pos = beg + (v * kThreads + tid) * 4 + e;
      if (kk > s.hi) {
        if (ia < n_sel_above) {
          oi[ia] = pos;
          os[ia] = key_to_float(kk);
        }
        ++ia;
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
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cluster > 8) {
    cudaError_t e = cudaFuncSetAttribute(topk_kernel<EPT>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
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
  topk_short_kernel<<<a.n_rows, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace dsa
