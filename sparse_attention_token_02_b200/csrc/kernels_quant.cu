// Cache append and per-row FP8 quantisation (the indexer's "K compressor -> quant(FP8)
// -> write Indexer K cache" step, page "Study MLA Indexer", section 数学流).
//
// A row is read with 16-byte vector loads, its absmax reduced, then every element
// is divided by scale = absmax / 448 in IEEE fp32 and converted with CUDA's
// round-to-nearest-even, saturating E4M3 conversion.  Key rows (d values) take one
// warp each; query rows (one scale per token over all H*d values, 8192 for the
// indexer's 64 x 128) take one CTA each, the row held in registers between the
// absmax and the conversion, so that a decode step's few long rows spread over
// many SMs.  Memory-bound: 16-byte loads and 8-byte stores per thread.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "internal.h"
#include "ptx.cuh"

namespace dsa {

namespace {

constexpr int kWarpsPerBlock = 8;
constexpr int kLongThreads = 256;          // threads of the CTA-per-row kernel
constexpr int kLongRowMin = 1024;          // rows at least this long take a CTA each

// Loads 8 consecutive source elements as fp32.
__device__ __forceinline__ void load8(const void* src, int src_is_f32, int64_t elem, float (&v)[8]) {
  if (src_is_f32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(src) + elem);
    float4 a = __ldg(p), b = __ldg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(src) + elem));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

// Eight values divided by s and encoded as E4M3 (saturating), in element order.
__device__ __forceinline__ uint2 encode8(const float (&v)[8], float s) {
  uint32_t packed[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 4; i += 2) {
      float2 pair = make_float2(__fdiv_rn(v[4 * h + i], s), __fdiv_rn(v[4 * h + i + 1], s));
      const __nv_fp8x2_storage_t two = __nv_cvt_float2_to_fp8x2(pair, __NV_SATFINITE, __NV_E4M3);
      word |= static_cast<uint32_t>(two) << (8 * i);
    }
    packed[h] = word;
  }
  return make_uint2(packed[0], packed[1]);
}

__device__ __forceinline__ float scale_of(float amax) { return amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f; }

__global__ void __launch_bounds__(kWarpsPerBlock * 32)
quantize_rows_fp8_kernel(const void* __restrict__ src, int src_is_f32, int64_t rows, int32_t row_len,
                         uint8_t* __restrict__ dst, float* __restrict__ scale, const int64_t* __restrict__ dst_rows,
                         int64_t dst_capacity, int* err) {
  launch_dependents();                        // the indexer kernel may start its prologue
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int64_t drow = dst_rows ? dst_rows[row] : row;
  if (drow < 0 || drow >= dst_capacity) {
    if (lane == 0) record_error(err, DSA_DEVERR_BOUNDS, static_cast<int>(row));
    return;
  }
  const int64_t base = row * row_len;
  float amax = 0.f;
  for (int c = lane * 8; c < row_len; c += 32 * 8) {
    float v[8];
    load8(src, src_is_f32, base + c, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = scale_of(amax);
  if (lane == 0) scale[drow] = s;
  uint8_t* out = dst + drow * row_len;
  for (int c = lane * 8; c < row_len; c += 32 * 8) {
    float v[8];
    load8(src, src_is_f32, base + c, v);
    *reinterpret_cast<uint2*>(out + c) = encode8(v, s);
  }
}

// One CTA per row of up to CH * 8 * kLongThreads values: each thread holds its CH chunks
// of 8 values in registers from the absmax to the conversion.
template <int CH>
__global__ void __launch_bounds__(kLongThreads)
quantize_long_rows_fp8_kernel(const void* __restrict__ src, int src_is_f32, int32_t row_len,
                              uint8_t* __restrict__ dst, float* __restrict__ scale,
                              const int64_t* __restrict__ dst_rows, int64_t dst_capacity, int* err) {
  __shared__ float warp_max[kLongThreads / 32];
  launch_dependents();                        // the indexer kernel may start its prologue
  const int64_t row = blockIdx.x;
  const int64_t drow = dst_rows ? dst_rows[row] : row;
  if (drow < 0 || drow >= dst_capacity) {     // uniform over the CTA
    if (threadIdx.x == 0) record_error(err, DSA_DEVERR_BOUNDS, static_cast<int>(row));
    return;
  }
  const int chunks = row_len / 8;
  const int64_t base = row * row_len;
  float v[CH][8];
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int idx = static_cast<int>(threadIdx.x) + c * kLongThreads;
    if (idx < chunks) {
      load8(src, src_is_f32, base + idx * 8, v[c]);
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[c][i]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kLongThreads / 32; ++w) amax = fmaxf(amax, warp_max[w]);
  const float s = scale_of(amax);
  if (threadIdx.x == 0) scale[drow] = s;
  uint8_t* out = dst + drow * row_len;
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int idx = static_cast<int>(threadIdx.x) + c * kLongThreads;
    if (idx < chunks) *reinterpret_cast<uint2*>(out + idx * 8) = encode8(v[c], s);
  }
}

__global__ void __launch_bounds__(kWarpsPerBlock * 32)
append_bf16_kernel(const void* __restrict__ src, int src_is_f32, int64_t rows, int32_t row_len,
                   uint16_t* __restrict__ dst, const int64_t* __restrict__ dst_rows, int64_t dst_capacity, int* err) {
  launch_dependents();                        // the indexer kernel may start its prologue
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int64_t drow = dst_rows ? dst_rows[row] : row;
  if (drow < 0 || drow >= dst_capacity) {
    if (lane == 0) record_error(err, DSA_DEVERR_BOUNDS, static_cast<int>(row));
    return;
  }
  const int64_t base = row * row_len;
  uint16_t* out = dst + drow * row_len;
  for (int c = lane * 8; c < row_len; c += 32 * 8) {
    uint4 word;
    if (src_is_f32) {
      float v[8];
      load8(src, 1, base + c, v);
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t*>(&b);
      }
      word = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
      word = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(src) + base + c));
    }
    *reinterpret_cast<uint4*>(out + c) = word;
  }
}

}  // namespace

cudaError_t launch_quantize_rows_fp8(const void* src, int src_is_f32, int64_t rows, int32_t row_len,
                                     uint8_t* dst, float* scale, const int64_t* dst_rows, int64_t dst_capacity,
                                     int* err, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int chunks_per_thread = (row_len / 8 + kLongThreads - 1) / kLongThreads;
  if (row_len >= kLongRowMin && chunks_per_thread <= 8 && rows <= 0x7FFFFFFF) {
    const unsigned grid = static_cast<unsigned>(rows);
    if (chunks_per_thread <= 1)
      quantize_long_rows_fp8_kernel<1><<<grid, kLongThreads, 0, stream>>>(src, src_is_f32, row_len, dst, scale,
                                                                           dst_rows, dst_capacity, err);
    else if (chunks_per_thread <= 2)
      quantize_long_rows_fp8_kernel<2><<<grid, kLongThreads, 0, stream>>>(src, src_is_f32, row_len, dst, scale,
                                                                           dst_rows, dst_capacity, err);
    else if (chunks_per_thread <= 4)
      quantize_long_rows_fp8_kernel<4><<<grid, kLongThreads, 0, stream>>>(src, src_is_f32, row_len, dst, scale,
                                                                           dst_rows, dst_capacity, err);
    else
      quantize_long_rows_fp8_kernel<8><<<grid, kLongThreads, 0, stream>>>(src, src_is_f32, row_len, dst, scale,
                                                                           dst_rows, dst_capacity, err);
    return cudaGetLastError();
  }
  const int64_t blocks = (rows + kWarpsPerBlock - 1) / kWarpsPerBlock;
  quantize_rows_fp8_kernel<<<static_cast<unsigned>(blocks), kWarpsPerBlock * 32, 0, stream>>>(
      src, src_is_f32, rows, row_len, dst, scale, dst_rows, dst_capacity, err);
  return cudaGetLastError();
}

cudaError_t launch_append_bf16(const void* src, int src_is_f32, int64_t rows, int32_t row_len, uint16_t* dst,
                               const int64_t* dst_rows, int64_t dst_capacity, int* err, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int64_t blocks = (rows + kWarpsPerBlock - 1) / kWarpsPerBlock;
  append_bf16_kernel<<<static_cast<unsigned>(blocks), kWarpsPerBlock * 32, 0, stream>>>(
      src, src_is_f32, rows, row_len, dst, dst_rows, dst_capacity, err);
  return cudaGetLastError();
}

}  // namespace dsa
