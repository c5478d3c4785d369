// What the consumers of a selection do with it.
//
// * Gather of the selected latent rows: the sparse MQA after the indexer reads the latent
//   c^KV only at the top-k positions (page "Study MLA Indexer", section 数学流; its 两条
//   cache 区分 table: d_c = 512 values per token; "Lightning Indexer 详解" §1: Core MLA
//   attends only over the index set).  dst[r, j, :] = src[row_base[r] + idx[r, j], :],
//   zero rows for -1.  Rows are opaque bytes (any dtype), moved as 16-byte vectors, one
//   warp per output row.  HBM-bound: row_bytes read + row_bytes written per entry.
// * Global cache rows of a selection, int64 (for consumers indexing one packed cache).
// * Sorted selection: each row by score descending, then position ascending, padding last
//   (the order torch.topk returns, the first page §3 step 5).  One CTA per row sorts
//   64-bit composite keys (order key of the score, complemented position) in shared memory
//   with a bitonic network.
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace dsa {

namespace {

constexpr int kGatherThreads = 256;
constexpr int kMaxRowVecs = 32 * 8;           // rows up to 4 KB: at most 8 vectors per lane
constexpr int kGatherInFlight = 8;            // 16-byte loads per lane issued together

constexpr int kGatherCtasPerSm = 4;           // resident CTAs per SM the grid is sized for

// Source row of output entry o: -2 none (past the end), -1 a padding entry (a zero row),
// else the row of src.  An out-of-range row is reported and written as zeros.
__device__ __forceinline__ int64_t gather_src_row(const int32_t* __restrict__ idx, const int64_t* __restrict__ row_base,
                                                  int64_t o, int64_t end, int32_t top_k, int64_t src_rows, int* err) {
  if (o >= end) return -2;
  const int32_t i = idx[o];
  if (i < 0) return -1;
  const int64_t sr = row_base[o / top_k] + i;
  if (sr < 0 || sr >= src_rows) {
    record_error(err, DSA_DEVERR_BOUNDS, static_cast<int>(o / top_k));
    return -1;
  }
  return sr;
}

// Warp w copies the contiguous output entries [n_out * w / W, n_out * (w + 1) / W) (W warps
// in the grid, so the share of every warp is the same to within one row).  It resolves the
// source rows of up to 32 entries at once (one entry per lane, so the index and row-base
// loads of a batch overlap), then copies them RPW rows at a time, VPL 16-byte vectors per
// lane per row (VPL * 32 >= the row's vectors), all RPW * VPL loads in flight before any store.
template <int VPL, int RPW>
__global__ void __launch_bounds__(kGatherThreads, kGatherCtasPerSm)
gather_rows_kernel(const uint4* __restrict__ src, int64_t src_rows, int32_t row_vecs, const int32_t* __restrict__ idx,
                   const int64_t* __restrict__ row_base, int64_t n_out, int32_t top_k, uint4* __restrict__ dst,
                   int* err) {
  static_assert(VPL * RPW == kGatherInFlight, "loads in flight per lane");
  grid_dependency_wait();                     // the selection comes from the previous kernel
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kGatherThreads + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * kGatherThreads) >> 5;
  const int64_t begin = n_out * warp / n_warps, end = n_out * (warp + 1) / n_warps;
  for (int64_t b0 = begin; b0 < end; b0 += 32) {
    const int64_t mine = gather_src_row(idx, row_base, b0 + lane, end, top_k, src_rows, err);
    const int batch = end - b0 < 32 ? static_cast<int>(end - b0) : 32;
    for (int g = 0; g < batch; g += RPW) {
      int64_t srow[RPW];
#pragma unroll
      for (int q = 0; q < RPW; ++q) srow[q] = __shfl_sync(0xffffffffu, mine, (g + q) & 31);
#pragma unroll
      for (int q = 0; q < RPW; ++q)
        if (g + q >= batch) srow[q] = -2;
      uint4 v[RPW][VPL];
#pragma unroll
      for (int q = 0; q < RPW; ++q)
#pragma unroll
        for (int u = 0; u < VPL; ++u) {
          const int c = u * 32 + lane;
          v[q][u] = make_uint4(0u, 0u, 0u, 0u);
          if (srow[q] >= 0 && c < row_vecs) v[q][u] = __ldcs(src + srow[q] * row_vecs + c);
        }
#pragma unroll
      for (int q = 0; q < RPW; ++q)
#pragma unroll
        for (int u = 0; u < VPL; ++u) {
          const int c = u * 32 + lane;
          if (srow[q] != -2 && c < row_vecs) __stcs(dst + (b0 + g + q) * row_vecs + c, v[q][u]);
        }
    }
  }
}

__global__ void __launch_bounds__(256) selection_rows_kernel(const int32_t* __restrict__ idx,
                                                             const int64_t* __restrict__ row_base, int64_t n_out,
                                                             int32_t top_k, int64_t* __restrict__ out) {
  grid_dependency_wait();
  for (int64_t o = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; o < n_out;
       o += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int32_t i = idx[o];
    out[o] = i >= 0 ? row_base[o / top_k] + i : -1;
  }
}

constexpr int kSortThreads = 512;
constexpr int kSortMax = 4096;                // entries per row the shared-memory sort takes

__global__ void __launch_bounds__(kSortThreads) sort_selection_kernel(int32_t* __restrict__ idx,
                                                                      float* __restrict__ score, int32_t top_k,
                                                                      int32_t width) {
  __shared__ unsigned long long key[kSortMax];
  grid_dependency_wait();
  int32_t* oi = idx + static_cast<int64_t>(blockIdx.x) * top_k;
  float* os = score + static_cast<int64_t>(blockIdx.x) * top_k;
  const int tid = threadIdx.x;
  // key: order key of the score (high word), ~position (low word); padding 0 sorts last
  for (int i = tid; i < width; i += kSortThreads) {
    unsigned long long kk = 0ull;
    if (i < top_k) {
      const int32_t p = oi[i];
      if (p >= 0)                             // + 0.0f: -0.0 ties with +0.0 (returned as +0.0)
        kk = (static_cast<unsigned long long>(order_key(__float_as_uint(os[i] + 0.0f))) << 32) |
             static_cast<unsigned long long>(~static_cast<uint32_t>(p));
    }
    key[i] = kk;
  }
  __syncthreads();
  // bitonic network, descending overall.  A stage of stride <= 16 touches, for each t, only
  // the 64-element block of its warp's t range, so only a stage of stride >= 32 (or the end)
  // needs the whole CTA to have finished the stage before it.
  for (int size = 2; size <= width; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = tid; t < width / 2; t += kSortThreads) {
        const int pos = 2 * t - (t & (stride - 1));
        const int partner = pos + stride;
        const bool desc = (pos & size) == 0;
        const unsigned long long a = key[pos], b = key[partner];
        if ((a < b) == desc) {
          key[pos] = b;
          key[partner] = a;
        }
      }
      const int next_stride = stride > 1 ? stride >> 1 : size;   // the next stage's stride
      if (next_stride >= 32 || (stride == 1 && size == width))
        __syncthreads();
      else
        __syncwarp();
    }
  }
  for (int i = tid; i < top_k; i += kSortThreads) {
    const unsigned long long kk = key[i];
    if (kk == 0ull) {
      oi[i] = -1;
      os[i] = -INFINITY;
    } else {
      oi[i] = static_cast<int32_t>(~static_cast<uint32_t>(kk & 0xFFFFFFFFull));
      const uint32_t u = static_cast<uint32_t>(kk >> 32);
      os[i] = __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
    }
  }
}

__global__ void __launch_bounds__(256) fill_f32_kernel(float* __restrict__ p, int64_t n, float v) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = v;
}

// Self-test of the bounded wait every kernel of the library uses: one CTA waits on an
// mbarrier that nothing arrives at, with a short limit; the wait must expire, raise the CTA's
// abort flag and let the kernel record DSA_DEVERR_TIMEOUT and return.
__global__ void wait_expiry_kernel(long long limit_cycles, int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const bool done = mbar_wait(&bar, 0, &abort_flag, limit_cycles);   // no arrival ever comes
  __syncthreads();
  if (threadIdx.x == 0 && !done && abort_flag) record_error(err, DSA_DEVERR_TIMEOUT, static_cast<int>(blockIdx.x));
}

cudaLaunchConfig_t pdl_config(dim3 grid, dim3 block, cudaStream_t stream, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

}  // namespace

cudaError_t launch_fill_f32(float* p, int64_t n, float v, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const int64_t blocks = (n + 255) / 256;
  fill_f32_kernel<<<static_cast<unsigned>(blocks < 1024 ? blocks : 1024), 256, 0, stream>>>(p, n, v);
  return cudaGetLastError();
}

bool gather_row_bytes_supported(int32_t row_bytes) {
  return row_bytes > 0 && row_bytes % 16 == 0 && row_bytes / 16 <= kMaxRowVecs;
}

int sort_selection_max() { return kSortMax; }

cudaError_t launch_wait_expiry(long long limit_cycles, int* err, cudaStream_t stream) {
  wait_expiry_kernel<<<1, 64, 0, stream>>>(limit_cycles, err);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const void* src, int64_t src_rows, int32_t row_bytes, const int32_t* idx,
                               const int64_t* row_base, int64_t rows, int32_t top_k, void* dst, int* err, int sms,
                               cudaStream_t stream) {
  const int64_t n_out = rows * top_k;
  if (n_out == 0) return cudaSuccess;
  const int32_t row_vecs = row_bytes / 16;
  const int vpl = row_vecs <= 32 ? 1 : row_vecs <= 64 ? 2 : row_vecs <= 128 ? 4 : 8;
  const int rpw = kGatherInFlight / vpl;
  const int64_t want = (n_out + rpw * (kGatherThreads / 32) - 1) / (rpw * (kGatherThreads / 32));
  const int64_t cap = static_cast<int64_t>(sms) * kGatherCtasPerSm;   // one resident wave
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pdl_config(dim3(static_cast<unsigned>(want < cap ? want : cap)), dim3(kGatherThreads),
                                      stream, attr);
  const uint4* s = static_cast<const uint4*>(src);
  uint4* d = static_cast<uint4*>(dst);
  switch (vpl) {
    case 1: return cudaLaunchKernelEx(&cfg, gather_rows_kernel<1, 8>, s, src_rows, row_vecs, idx, row_base, n_out, top_k, d, err);
    case 2: return cudaLaunchKernelEx(&cfg, gather_rows_kernel<2, 4>, s, src_rows, row_vecs, idx, row_base, n_out, top_k, d, err);
    case 4: return cudaLaunchKernelEx(&cfg, gather_rows_kernel<4, 2>, s, src_rows, row_vecs, idx, row_base, n_out, top_k, d, err);
    default: return cudaLaunchKernelEx(&cfg, gather_rows_kernel<8, 1>, s, src_rows, row_vecs, idx, row_base, n_out, top_k, d, err);
  }
}

cudaError_t launch_selection_rows(const int32_t* idx, const int64_t* row_base, int64_t rows, int32_t top_k,
                                  int64_t* out, int sms, cudaStream_t stream) {
  const int64_t n_out = rows * top_k;
  if (n_out == 0) return cudaSuccess;
  const int64_t want = (n_out + 255) / 256, cap = static_cast<int64_t>(sms) * 8;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pdl_config(dim3(static_cast<unsigned>(want < cap ? want : cap)), dim3(256), stream, attr);
  return cudaLaunchKernelEx(&cfg, selection_rows_kernel, idx, row_base, n_out, top_k, out);
}

cudaError_t launch_sort_selection(int32_t* idx, float* score, int64_t rows, int32_t top_k, cudaStream_t stream) {
  if (rows == 0 || top_k <= 1) return cudaSuccess;
  int32_t width = 2;
  while (width < top_k) width <<= 1;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pdl_config(dim3(static_cast<unsigned>(rows)), dim3(kSortThreads), stream, attr);
  return cudaLaunchKernelEx(&cfg, sort_selection_kernel, idx, score, top_k, width);
}

}  // namespace dsa
