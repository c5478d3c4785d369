// Rotary position embedding fused into the indexer's key append and query quantisation
// (page "Study MLA Indexer", section 数学流: k_repr_t = RoPE(x_t W_kr) -> quant(FP8) -> the
// indexer K cache; q_t = RoPE(x_t W_q)).  The pages give no RoPE detail; this is the published
// rotary embedding (RoFormer): pair i of the first rope_dim values turns by
// theta_i = p * base^(-2i / rope_dim), (a, b) -> (a cos - b sin, a sin + b cos), with pair i =
// (2i, 2i+1) (interleaved) or (i, i + rope_dim/2) (half); later values pass through.
//
// Angles: theta_i = p * inv_freq_i in fp64 (inv_freq from the host in fp64), reduced modulo
// 2 pi in fp64, then fp32 sincos of the reduced angle: positions reach 1e5 and more, where an
// fp32 product would lose whole percents.  Each (position, pair) angle is computed once and
// shared through shared memory (by the lanes of a key row, by all heads of a query token).
// The rotated row is then stored as bf16 (round to nearest even) or quantised to E4M3
// exactly as the plain quantiser does
// (scale = absmax / 448 in IEEE fp32, codes from CUDA's saturating conversion of x / scale).
// One warp per key row; one CTA per query token (all its heads share one FP8 scale).
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "internal.h"
#include "ptx.cuh"

namespace dsa {

namespace {

// (cos, sin) of pair i at position p
__device__ __forceinline__ float2 pair_cos_sin(int i, int32_t p, const RopeParams& r) {
  constexpr double kTwoPi = 6.283185307179586476925286766559;
  constexpr double kInvTwoPi = 0.15915494309189533576888376337251;
  const double theta = static_cast<double>(p) * r.inv_freq[i];
  const double red = fma(-kTwoPi, rint(theta * kInvTwoPi), theta);   // |red| <= pi (+ rounding)
  float s, c;
  sincosf(static_cast<float>(red), &s, &c);
  return make_float2(c, s);
}

// The (cos, sin) each of a lane's EPL values rotates with (values lane*EPL .. lane*EPL+EPL-1
// of a d-vector), read once from cs[] into registers; (1, 0) past rope_dim.
template <int EPL>
__device__ __forceinline__ void lane_cos_sin(int lane, const float2* cs, const RopeParams& r, float2 (&t)[EPL]) {
  const int half = r.rope_dim / 2;
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    const int idx = lane * EPL + e;
    const int pair = r.interleaved ? idx / 2 : (idx < half ? idx : idx - half);
    t[e] = idx < r.rope_dim ? cs[pair] : make_float2(1.f, 0.f);
  }
}

// Rotates the EPL values v[] a lane holds with the lane's (cos, sin) t[].
template <int EPL>
__device__ __forceinline__ void rope_lane(float (&v)[EPL], int lane, const float2 (&t)[EPL], const RopeParams& r) {
  const bool rotates = lane * EPL < r.rope_dim;           // values past rope_dim pass through untouched
  if (r.interleaved) {
#pragma unroll
    for (int e = 0; e < EPL; e += 2) {                    // pairs (2i, 2i+1) lie inside the lane
      const float a = v[e], b = v[e + 1];
      if (rotates) {
        v[e] = a * t[e].x - b * t[e].y;
        v[e + 1] = a * t[e].y + b * t[e].x;
      }
    }
  } else {
    // pair (i, i + half): the partner value sits half / EPL lanes away (half % EPL == 0)
    const int half = r.rope_dim / 2;
    const int lane_off = half / EPL;
    const bool first = lane * EPL < half;                 // a lane's values all sit on one side
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const float other = __shfl_xor_sync(0xffffffffu, v[e], lane_off);   // lane_off is a power of two
      if (rotates) v[e] = first ? v[e] * t[e].x - other * t[e].y : other * t[e].y + v[e] * t[e].x;
    }
  }
}

// EPL consecutive source values (elem is a multiple of EPL, so the vector loads are aligned)
template <int EPL>
__device__ __forceinline__ void load_row(const void* src, int src_is_f32, int64_t elem, float (&v)[EPL]) {
  static_assert(EPL == 2 || EPL == 4, "two or four values per lane");
  if (src_is_f32) {
    if constexpr (EPL == 4) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(src) + elem));
      v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    } else {
      const float2 f = __ldg(reinterpret_cast<const float2*>(static_cast<const float*>(src) + elem));
      v[0] = f.x; v[1] = f.y;
    }
  } else {
    const __nv_bfloat16* b = static_cast<const __nv_bfloat16*>(src) + elem;
    uint32_t w[EPL / 2];
    if constexpr (EPL == 4) {
      const uint2 u = __ldg(reinterpret_cast<const uint2*>(b));
      w[0] = u.x; w[1] = u.y;
    } else {
      w[0] = __ldg(reinterpret_cast<const unsigned int*>(b));
    }
#pragma unroll
    for (int i = 0; i < EPL / 2; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

template <int EPL>
__device__ __forceinline__ void store_bf16(__nv_bfloat16* dst, const float (&v)[EPL]) {
  uint32_t w[EPL / 2];
#pragma unroll
  for (int i = 0; i < EPL / 2; ++i) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&b);
  }
  if constexpr (EPL == 4)
    *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
  else
    *reinterpret_cast<uint32_t*>(dst) = w[0];
}

template <int EPL>
__device__ __forceinline__ void store_fp8(uint8_t* dst, const float (&v)[EPL], float scale) {
  uint32_t word = 0;
#pragma unroll
  for (int e = 0; e < EPL; e += 2) {
    const float2 pair = make_float2(__fdiv_rn(v[e], scale), __fdiv_rn(v[e + 1], scale));
    const __nv_fp8x2_storage_t two = __nv_cvt_float2_to_fp8x2(pair, __NV_SATFINITE, __NV_E4M3);
    word |= static_cast<uint32_t>(two) << (8 * e);
  }
  if constexpr (EPL == 4)
    *reinterpret_cast<uint32_t*>(dst) = word;
  else
    *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(word);
}

constexpr int kRopeWarps = 8;

template <int EPL>
__global__ void __launch_bounds__(kRopeWarps * 32)
rope_append_kernel(const void* __restrict__ src, int src_is_f32, int64_t rows, const int64_t* __restrict__ dst_rows,
                   const int32_t* __restrict__ positions, int64_t capacity, RopeParams rp, int fp8,
                   void* __restrict__ cache, float* __restrict__ scale, int* err) {
  launch_dependents();
  constexpr int D = EPL * 32;
  __shared__ float2 cs_all[kRopeWarps][kRopeMaxPairs];
  const int lane = threadIdx.x & 31;
  float2* cs = cs_all[threadIdx.x >> 5];
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kRopeWarps + (threadIdx.x >> 5);
  if (row >= rows) return;                              // whole warps leave together
  const int64_t drow = dst_rows[row];
  if (drow < 0 || drow >= capacity) {
    if (lane == 0) record_error(err, DSA_DEVERR_BOUNDS, static_cast<int>(row));
    return;
  }
  float v[EPL];
  load_row<EPL>(src, src_is_f32, row * D + lane * EPL, v);     // in flight while the angles compute
  const int32_t p = positions[row];
  for (int i = lane; i < rp.rope_dim / 2; i += 32) cs[i] = pair_cos_sin(i, p, rp);
  __syncwarp();
  float2 t[EPL];
  lane_cos_sin<EPL>(lane, cs, rp, t);
  rope_lane<EPL>(v, lane, t, rp);
  if (fp8) {
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) amax = fmaxf(amax, fabsf(v[e]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    if (lane == 0) scale[drow] = s;
    store_fp8<EPL>(static_cast<uint8_t*>(cache) + drow * D + lane * EPL, v, s);
  } else {
    store_bf16<EPL>(static_cast<__nv_bfloat16*>(cache) + drow * D + lane * EPL, v);
  }
}

// One CTA per query token: warp w rotates heads w, w + kRopeWarps, ... (at most HPW each);
// FP8 output shares one scale over all H * d values of the token.
template <int EPL, int HPW>
__global__ void __launch_bounds__(kRopeWarps * 32, 4)
rope_queries_kernel(const void* __restrict__ src, int src_is_f32, int32_t H, const int32_t* __restrict__ positions,
                    RopeParams rp, int fp8, void* __restrict__ dst, float* __restrict__ scale) {
  launch_dependents();
  constexpr int D = EPL * 32;
  constexpr int kMaxHeadsPerWarp = HPW;
  __shared__ float warp_max[kRopeWarps];
  __shared__ float2 cs[kRopeMaxPairs];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t t = blockIdx.x;
  float v[kMaxHeadsPerWarp][EPL];
#pragma unroll
  for (int u = 0; u < kMaxHeadsPerWarp; ++u) {          // all loads in flight while the angles compute
    const int h = warp + u * kRopeWarps;
    if (h < H) load_row<EPL>(src, src_is_f32, (t * H + h) * D + lane * EPL, v[u]);
  }
  const int32_t p = positions[t];
  for (int i = threadIdx.x; i < rp.rope_dim / 2; i += kRopeWarps * 32) cs[i] = pair_cos_sin(i, p, rp);
  __syncthreads();
  float2 tcs[EPL];                                      // the same for every head of the token
  lane_cos_sin<EPL>(lane, cs, rp, tcs);
  float amax = 0.f;
#pragma unroll
  for (int u = 0; u < kMaxHeadsPerWarp; ++u) {
    const int h = warp + u * kRopeWarps;
    if (h < H) {
      rope_lane<EPL>(v[u], lane, tcs, rp);
#pragma unroll
      for (int e = 0; e < EPL; ++e) amax = fmaxf(amax, fabsf(v[u][e]));
    }
  }
  if (fp8) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) warp_max[warp] = amax;
    __syncthreads();
    float m = 0.f;
#pragma unroll
    for (int w = 0; w < kRopeWarps; ++w) m = fmaxf(m, warp_max[w]);
    const float s = m > 0.f ? __fdiv_rn(m, 448.0f) : 1.0f;
    if (threadIdx.x == 0) scale[t] = s;
#pragma unroll
    for (int u = 0; u < kMaxHeadsPerWarp; ++u) {
      const int h = warp + u * kRopeWarps;
      if (h < H) store_fp8<EPL>(static_cast<uint8_t*>(dst) + (t * H + h) * D + lane * EPL, v[u], s);
    }
  } else {
#pragma unroll
    for (int u = 0; u < kMaxHeadsPerWarp; ++u) {
      const int h = warp + u * kRopeWarps;
      if (h < H) {
        store_bf16<EPL>(static_cast<__nv_bfloat16*>(dst) + (t * H + h) * D + lane * EPL, v[u]);
      }
    }
  }
}

}  // namespace

bool rope_shape_supported(int32_t d, int32_t H, const RopeParams& r) {
  const int epl = d / 32;
  if (d != 64 && d != 128) return false;
  if (H < 1 || H > kRopeWarps * 16) return false;
  if (r.rope_dim < 0 || r.rope_dim > d || r.rope_dim % 2 || r.rope_dim / 2 > kRopeMaxPairs) return false;
  if (!(r.base > 0.0)) return false;
  // half layout: the partner lane offset (rope_dim / 2) / EPL must be a power of two
  if (!r.interleaved && r.rope_dim > 0) {
    const int half = r.rope_dim / 2;
    if (half % epl) return false;
    const int off = half / epl;
    if (off & (off - 1)) return false;
  }
  return true;
}

cudaError_t launch_rope_append(const void* src, int src_is_f32, int64_t rows, int32_t d, const int64_t* dst_rows,
                               const int32_t* positions, int64_t capacity, const RopeParams& r, int fp8, void* cache,
                               float* scale, int* err, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((rows + kRopeWarps - 1) / kRopeWarps);
  if (d == 64)
    rope_append_kernel<2><<<blocks, kRopeWarps * 32, 0, stream>>>(src, src_is_f32, rows, dst_rows, positions, capacity,
                                                                  r, fp8, cache, scale, err);
  else
    rope_append_kernel<4><<<blocks, kRopeWarps * 32, 0, stream>>>(src, src_is_f32, rows, dst_rows, positions, capacity,
                                                                  r, fp8, cache, scale, err);
  return cudaGetLastError();
}

cudaError_t launch_rope_queries(const void* src, int src_is_f32, int64_t T, int32_t H, int32_t d,
                                const int32_t* positions, const RopeParams& r, int fp8, void* dst, float* scale,
                                cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>(T), block = kRopeWarps * 32;
  const bool few = H <= kRopeWarps * 8;                   // at most 8 heads per warp
  if (d == 64) {
    if (few) rope_queries_kernel<2, 8><<<grid, block, 0, stream>>>(src, src_is_f32, H, positions, r, fp8, dst, scale);
    else rope_queries_kernel<2, 16><<<grid, block, 0, stream>>>(src, src_is_f32, H, positions, r, fp8, dst, scale);
  } else {
    if (few) rope_queries_kernel<4, 8><<<grid, block, 0, stream>>>(src, src_is_f32, H, positions, r, fp8, dst, scale);
    else rope_queries_kernel<4, 16><<<grid, block, 0, stream>>>(src, src_is_f32, H, positions, r, fp8, dst, scale);
  }
  return cudaGetLastError();
}

}  // namespace dsa
