// Rotary position embedding fused into the indexer's key append and query quantisation
// (page "Study MLA Indexer", section 数学流: k_repr_t = RoPE(x_t W_kr) -> quant(FP8) -> the
// indexer K cache; q_t = RoPE(x_t W_q)).  The pages give no RoPE detail; this is the published
// rotary embedding (RoFormer): pair i of the first rope_dim values turns by
// theta_i = p * base^(-2i / rope_dim), (a, b) -> (a cos - b sin, a sin + b cos), with pair i =
// (2i, 2i+1) (interleaved) or (i, i + rope_dim/2) (half); later values pass through.
//
// Angles: theta_i = p * inv_freq_i in fp64 (inv_freq from the host in fp64), reduced modulo
// 2 pi in fp64, then fp32 sincos of the reduced angle: positions reach 1e5 and more, where an
// fp32 product would lose whole percents.  Each (position, pair) angle is computed once, by
// one thread, and shared through shared memory (by the lanes of a key row, by all heads of a
// query token).  The rotated row is stored as bf16 (round to nearest even) or quantised to
// E4M3: scale = absmax / 448 in IEEE fp32 (as the plain quantiser), codes from CUDA's
// saturating conversion of x * (1 / scale) with a correctly rounded reciprocal, which is
// within one fp32 ulp of x / scale (the rotation itself is fp32, so the codes are compared
// with the fp64 oracle to within one E4M3 step, not bit for bit).
//
// Both kernels are instruction-bound before they are HBM-bound unless the per-value work is
// a handful of instructions: the layout (d_I, interleaved or half pairs) is a template
// argument, a thread's angles are loaded once per row or token, and the quotient is a product.
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

// FP8 scale of a vector with absolute maximum amax (.x) and its reciprocal (.y)
__device__ __forceinline__ float2 fp8_scale(float amax) {
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  return make_float2(s, __frcp_rn(s));
}

__device__ __forceinline__ uint32_t fp8x2(float a, float b, float inv) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a * inv, b * inv), __NV_SATFINITE, __NV_E4M3));
}

// E4M3 codes of a.x, a.y, b.x, b.y (saturating, round to nearest even), lowest byte first
__device__ __forceinline__ uint32_t e4m3x4(float2 a, float2 b) {
  uint32_t r;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(r)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

__device__ __forceinline__ uint32_t bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
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

// ------------------------------------------------------------------------------- keys

constexpr int kRopeWarps = 8;
constexpr int kAppendRowsPerWarp = 4;

// One warp per kAppendRowsPerWarp consecutive rows, lane l holding values l*EPL .. l*EPL+EPL-1
// of each.  Every load of the rows (values, position, destination) is issued first; the
// rows' angles are then spread over the lanes (one sincos per lane per row at rope_dim 64).
template <int D, bool INTERLEAVED>
__global__ void __launch_bounds__(kRopeWarps * 32)
rope_append_kernel(const void* __restrict__ src, int src_is_f32, int64_t rows, const int64_t* __restrict__ dst_rows,
                   const int32_t* __restrict__ positions, int64_t capacity, RopeParams rp, int fp8,
                   void* __restrict__ cache, float* __restrict__ scale, int* err) {
  constexpr int EPL = D / 32;
  constexpr int R = kAppendRowsPerWarp;
  __shared__ float2 cs_all[kRopeWarps][R][kRopeMaxPairs];
  launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float2 (*cs)[kRopeMaxPairs] = cs_all[warp];
  const int64_t row0 = (static_cast<int64_t>(blockIdx.x) * kRopeWarps + warp) * R;
  if (row0 >= rows) return;                             // whole warps leave together
  float v[R][EPL];
  int32_t pos[R];
  int64_t drow[R];
#pragma unroll
  for (int q = 0; q < R; ++q) {
    const int64_t row = row0 + q;
    drow[q] = -1;
    pos[q] = 0;
#pragma unroll
    for (int e = 0; e < EPL; ++e) v[q][e] = 0.f;
    if (row < rows) {
      load_row<EPL>(src, src_is_f32, row * D + lane * EPL, v[q]);
      pos[q] = positions[row];
      drow[q] = dst_rows[row];
    }
  }
  const int npairs = rp.rope_dim / 2;
#pragma unroll
  for (int q = 0; q < R; ++q)
    for (int i = lane; i < npairs; i += 32) cs[q][i] = pair_cos_sin(i, pos[q], rp);
  __syncwarp();
  const int idx0 = lane * EPL;
  const bool rotates = idx0 < rp.rope_dim;
  // the R rows go through each step together (independent dependency chains side by side)
  bool valid[R];
#pragma unroll
  for (int q = 0; q < R; ++q) {
    valid[q] = row0 + q < rows && drow[q] >= 0 && drow[q] < capacity;
    if (row0 + q < rows && !valid[q] && lane == 0) record_error(err, DSA_DEVERR_BOUNDS, static_cast<int>(row0 + q));
  }
  if constexpr (INTERLEAVED) {
    if (rotates) {
#pragma unroll
      for (int q = 0; q < R; ++q)
#pragma unroll
        for (int e = 0; e < EPL; e += 2) {
          if (idx0 + e < rp.rope_dim) {
            const float2 t = cs[q][(idx0 + e) >> 1];
            const float a = v[q][e], b = v[q][e + 1];
            v[q][e] = a * t.x - b * t.y;
            v[q][e + 1] = a * t.y + b * t.x;
          }
        }
    }
  } else {
    // pair (i, i + half): the partner value sits half / EPL lanes away (a power of two)
    const int lane_off = npairs / EPL;
    const bool first = idx0 < npairs;
    const int p0 = first ? idx0 : idx0 - npairs;
    float other[R][EPL];
#pragma unroll
    for (int q = 0; q < R; ++q)
#pragma unroll
      for (int e = 0; e < EPL; ++e) other[q][e] = __shfl_xor_sync(0xffffffffu, v[q][e], lane_off & 31);
    if (rotates) {
#pragma unroll
      for (int q = 0; q < R; ++q)
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          const float2 t = cs[q][p0 + e];
          v[q][e] = first ? v[q][e] * t.x - other[q][e] * t.y : other[q][e] * t.y + v[q][e] * t.x;
        }
    }
  }
  if (fp8) {
    float amax[R];
#pragma unroll
    for (int q = 0; q < R; ++q) {
      amax[q] = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) amax[q] = fmaxf(amax[q], fabsf(v[q][e]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int q = 0; q < R; ++q) amax[q] = fmaxf(amax[q], __shfl_xor_sync(0xffffffffu, amax[q], o));
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const float2 sc = fp8_scale(amax[q]);
      if (!valid[q]) continue;
      if (lane == 0) scale[drow[q]] = sc.x;
      uint8_t* out = static_cast<uint8_t*>(cache) + drow[q] * D + idx0;
      if constexpr (EPL == 4)
        *reinterpret_cast<uint32_t*>(out) = fp8x2(v[q][0], v[q][1], sc.y) | (fp8x2(v[q][2], v[q][3], sc.y) << 16);
      else
        *reinterpret_cast<uint16_t*>(out) = static_cast<uint16_t>(fp8x2(v[q][0], v[q][1], sc.y));
    }
  } else {
#pragma unroll
    for (int q = 0; q < R; ++q) {
      if (!valid[q]) continue;
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(cache) + drow[q] * D + idx0;
      if constexpr (EPL == 4)
        *reinterpret_cast<uint2*>(out) = make_uint2(bf16x2(v[q][0], v[q][1]), bf16x2(v[q][2], v[q][3]));
      else
        *reinterpret_cast<uint32_t*>(out) = bf16x2(v[q][0], v[q][1]);
    }
  }
}

// ---------------------------------------------------------------------------- queries
//
// Persistent CTAs, each over the tokens blockIdx.x, blockIdx.x + gridDim.x, ...  A token's
// H * d source values are one contiguous block, brought into a ring of shared-memory slots
// by bulk copies (cp.async.bulk, completion counted on an mbarrier per slot) issued up to
// `stages` tokens ahead, so HBM reads of later tokens overlap the rotation and quantisation
// of the current one.  Each thread takes 8-value chunks of the token (chunk c: values
// 8c .. 8c + 7); since kQThreads * 8 is a multiple of d, all chunks of a thread sit at the
// same offset of their heads and rotate with the same angles.  All heads share the token's
// angles, computed once per token (for the next token while the current one is processed).

constexpr int kQThreads = 256;
constexpr int kQMaxStages = 8;
constexpr int kQRingBytes = 200 * 1024;      // shared memory for the rings of the CTAs on one SM
constexpr int kQMaxCtasPerSm = 3;

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               :: "r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
}

// Eight consecutive values of a slot (element offset e8, a multiple of 8) as four pairs.
__device__ __forceinline__ void slot_read8(const uint8_t* slot, int src_is_f32, int e8, float2 (&x)[4]) {
  if (src_is_f32) {
    const float4 a = *reinterpret_cast<const float4*>(slot + 4 * e8);
    const float4 b = *reinterpret_cast<const float4*>(slot + 4 * e8 + 16);
    x[0] = make_float2(a.x, a.y); x[1] = make_float2(a.z, a.w);
    x[2] = make_float2(b.x, b.y); x[3] = make_float2(b.z, b.w);
  } else {
    const uint4 u = *reinterpret_cast<const uint4*>(slot + 2 * e8);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
  }
}

// The rotation of a chunk in pairs of values (sm_100 packed fp32x2 arithmetic): v' = v C + Y S,
// with, per pair of values, interleaved: Y = (v.y, v.x), C = (cos, cos), S = (-sin, sin);
// half: Y = the partner values, C = the two cosines, S = the two sines, negated on the
// first side of the split.
template <int D, bool INTERLEAVED, int CPT>
__global__ void __launch_bounds__(kQThreads, CPT <= 4 ? kQMaxCtasPerSm : 2)
rope_queries_kernel(const uint8_t* __restrict__ src, int src_is_f32, int64_t T, int32_t H,
                    const int32_t* __restrict__ positions, RopeParams rp, int fp8, void* __restrict__ dst,
                    float* __restrict__ scale, int stages, int* err) {
  static_assert((kQThreads * 8) % D == 0, "a thread's chunks share one head offset");
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t full[kQMaxStages];
  __shared__ __align__(16) float2 cs[2][kRopeMaxPairs];
  __shared__ __align__(16) float warp_max[2][kQThreads / 32];
  __shared__ int abort_flag;
  launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int vals = H * D;                               // values of one token
  const int chunks = vals / 8;
  const uint32_t token_bytes = static_cast<uint32_t>(vals) * (src_is_f32 ? 4u : 2u);
  const int64_t n_local = T > blockIdx.x ? (T - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const int npairs = rp.rope_dim / 2;
  const int o = (tid * 8) % D;                          // head offset of every chunk of this thread
  const bool rot = o < rp.rope_dim;
  const bool first = o < npairs;                        // half pairs: this side of the split
  const int partner = first ? npairs : -npairs;
  if (tid == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(&full[s], 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    for (int64_t k = 0; k < stages && k < n_local; ++k) {
      const int64_t t = blockIdx.x + k * gridDim.x;
      mbar_arrive_expect_tx(&full[k], token_bytes);
      bulk_load(ring + k * token_bytes, src + t * token_bytes, token_bytes, &full[k]);
    }
  }
  // positions are read two tokens ahead of their use, so no global load latency sits
  // between two barriers of the token loop
  int32_t p_next = 0;
  if (n_local > 0) {
    const int32_t p = positions[blockIdx.x];
    if (n_local > 1 && tid < npairs) p_next = positions[blockIdx.x + gridDim.x];
    for (int i = tid; i < npairs; i += kQThreads) cs[0][i] = pair_cos_sin(i, p, rp);
  }
  __syncthreads();
  int64_t k = 0;
  int s = 0;                                            // slot of token k, and the parity of its use
  uint32_t phase = 0;
  for (; k < n_local; ++k, s = s + 1 == stages ? 0 : s + 1, phase ^= s == 0 ? 1u : 0u) {
    const int64_t t = blockIdx.x + k * gridDim.x;
    const int cb = static_cast<int>(k & 1);
    if (k + 1 < n_local && tid < npairs) {            // the next token's angles, published by the barrier below
      const int32_t p = p_next;
      if (k + 2 < n_local) p_next = positions[t + 2 * static_cast<int64_t>(gridDim.x)];
      for (int i = tid; i < npairs; i += kQThreads) cs[cb ^ 1][i] = pair_cos_sin(i, p, rp);
    }
    float2 C[4], S[4];
    if (rot) {
      if constexpr (INTERLEAVED) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 a = o + 2 * i < rp.rope_dim ? cs[cb][(o >> 1) + i] : make_float2(1.f, 0.f);
          C[i] = make_float2(a.x, a.x);
          S[i] = make_float2(-a.y, a.y);
        }
      } else {
        const float4* a4 = reinterpret_cast<const float4*>(&cs[cb][first ? o : o - npairs]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 a = a4[i];                       // pairs p0 + 2i, p0 + 2i + 1
          C[i] = make_float2(a.x, a.z);
          S[i] = first ? make_float2(-a.y, -a.w) : make_float2(a.y, a.w);
        }
      }
    }
    const bool ok = mbar_wait<true>(&full[s], phase, &abort_flag);
    const uint8_t* slot = ring + s * token_bytes;
    float2 x[CPT][4];
    float am[4] = {0.f, 0.f, 0.f, 0.f};                 // four independent maxima (short dependency chains)
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int c = tid + j * kQThreads;
      if (ok && c < chunks) {
        slot_read8(slot, src_is_f32, c * 8, x[j]);
        if (rot) {
          float2 y[4];
          if constexpr (INTERLEAVED) {
#pragma unroll
            for (int i = 0; i < 4; ++i) y[i] = make_float2(x[j][i].y, x[j][i].x);
          } else {
            slot_read8(slot, src_is_f32, c * 8 + partner, y);
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) x[j][i] = __ffma2_rn(x[j][i], C[i], __fmul2_rn(y[i], S[i]));
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) am[i] = fmaxf(am[i], fmaxf(fabsf(x[j][i].x), fabsf(x[j][i].y)));
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) x[j][i] = make_float2(0.f, 0.f);
      }
    }
    if (fp8) {
      float amax = fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3]));
#pragma unroll
      for (int m = 16; m > 0; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
      if (lane == 0) warp_max[cb][warp] = amax;
    }
    __syncthreads();                                    // slot s read by all; maxima and next angles visible
    if (abort_flag) break;                              // the same for every thread after the barrier
    if (tid == 0 && k + stages < n_local) {
      mbar_arrive_expect_tx(&full[s], token_bytes);
      bulk_load(ring + s * token_bytes, src + (t + static_cast<int64_t>(stages) * gridDim.x) * token_bytes,
                token_bytes, &full[s]);
    }
    if (fp8) {
      const float4 m0 = *reinterpret_cast<const float4*>(&warp_max[cb][0]);
      const float4 m1 = *reinterpret_cast<const float4*>(&warp_max[cb][4]);
      const float m = fmaxf(fmaxf(fmaxf(m0.x, m0.y), fmaxf(m0.z, m0.w)), fmaxf(fmaxf(m1.x, m1.y), fmaxf(m1.z, m1.w)));
      const float2 sc = fp8_scale(m);
      const float2 inv = make_float2(sc.y, sc.y);
      if (tid == 0) scale[t] = sc.x;
      uint8_t* out = static_cast<uint8_t*>(dst) + t * vals;
#pragma unroll
      for (int j = 0; j < CPT; ++j) {
        const int c = tid + j * kQThreads;
        if (c < chunks) {
          *reinterpret_cast<uint2*>(out + c * 8) =
              make_uint2(e4m3x4(__fmul2_rn(x[j][0], inv), __fmul2_rn(x[j][1], inv)),
                         e4m3x4(__fmul2_rn(x[j][2], inv), __fmul2_rn(x[j][3], inv)));
        }
      }
    } else {
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(dst) + t * vals;
#pragma unroll
      for (int j = 0; j < CPT; ++j) {
        const int c = tid + j * kQThreads;
        if (c < chunks)
          *reinterpret_cast<uint4*>(out + c * 8) =
              make_uint4(bf16x2(x[j][0].x, x[j][0].y), bf16x2(x[j][1].x, x[j][1].y), bf16x2(x[j][2].x, x[j][2].y),
                         bf16x2(x[j][3].x, x[j][3].y));
      }
    }
  }
  if (k < n_local) {                                    // a wait ran out: report, then let the copies land
    if (tid == 0) {
      record_error(err, DSA_DEVERR_TIMEOUT, static_cast<int>(blockIdx.x));
      int drain_abort = 0;
      for (int64_t j = k; j < n_local && j < k + stages; ++j)
        mbar_wait<true>(&full[j % stages], static_cast<uint32_t>((j / stages) & 1), &drain_abort);
    }
    __syncthreads();
  }
}

// Ring geometry of the query kernel: CTAs per SM and slots per CTA for tokens of token_bytes.
void rope_queries_geometry(uint32_t token_bytes, int* ctas_per_sm, int* stages) {
  int c = kQMaxCtasPerSm;
  while (c > 1 && kQRingBytes / c < 2 * static_cast<int>(token_bytes)) --c;
  const int st = kQRingBytes / c / static_cast<int>(token_bytes);
  *ctas_per_sm = c;
  *stages = st < kQMaxStages ? st : kQMaxStages;
}

template <int D, bool INTERLEAVED, int CPT>
cudaError_t launch_queries(const uint8_t* src, int src_is_f32, int64_t T, int32_t H, const int32_t* positions,
                           const RopeParams& r, int fp8, void* dst, float* scale, int* err, int sms,
                           cudaStream_t stream) {
  auto kernel = rope_queries_kernel<D, INTERLEAVED, CPT>;
  static unsigned long long configured = 0;   // one bit per device ordinal
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(configured & (1ull << dev))) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kQRingBytes);
    if (e != cudaSuccess) return e;
    if (dev < 64) configured |= 1ull << dev;
  }
  const uint32_t token_bytes = static_cast<uint32_t>(H) * D * (src_is_f32 ? 4u : 2u);
  int ctas = 1, stages = 2;
  rope_queries_geometry(token_bytes, &ctas, &stages);
  const size_t smem = static_cast<size_t>(stages) * token_bytes;
  int resident = 0;                                     // registers may allow fewer CTAs than the rings
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, kernel, kQThreads, smem);
  if (e != cudaSuccess) return e;
  if (resident >= 1 && resident < ctas) {
    ctas = resident;
    const int st = kQRingBytes / ctas / static_cast<int>(token_bytes);
    stages = st < kQMaxStages ? st : kQMaxStages;
  }
  const size_t smem_used = static_cast<size_t>(stages) * token_bytes;
  const int64_t cap = static_cast<int64_t>(sms) * ctas;
  const unsigned grid = static_cast<unsigned>(T < cap ? T : cap);
  kernel<<<grid, kQThreads, smem_used, stream>>>(src, src_is_f32, T, H, positions, r, fp8, dst, scale, stages, err);
  return cudaGetLastError();
}

template <int D, bool INTERLEAVED>
cudaError_t launch_queries_cpt(const uint8_t* src, int src_is_f32, int64_t T, int32_t H, const int32_t* positions,
                               const RopeParams& r, int fp8, void* dst, float* scale, int* err, int sms,
                               cudaStream_t stream) {
  const int cpt = (H * D / 8 + kQThreads - 1) / kQThreads;
  if (cpt <= 1) return launch_queries<D, INTERLEAVED, 1>(src, src_is_f32, T, H, positions, r, fp8, dst, scale, err, sms, stream);
  if (cpt <= 2) return launch_queries<D, INTERLEAVED, 2>(src, src_is_f32, T, H, positions, r, fp8, dst, scale, err, sms, stream);
  if (cpt <= 4) return launch_queries<D, INTERLEAVED, 4>(src, src_is_f32, T, H, positions, r, fp8, dst, scale, err, sms, stream);
  return launch_queries<D, INTERLEAVED, 8>(src, src_is_f32, T, H, positions, r, fp8, dst, scale, err, sms, stream);
}

}  // namespace

bool rope_shape_supported(int32_t d, int32_t H, const RopeParams& r) {
  if (d != 64 && d != 128) return false;
  const int epl = d / 32;
  if (H < 1 || H > 128) return false;
  if (r.rope_dim < 0 || r.rope_dim > d || r.rope_dim % 2 || r.rope_dim / 2 > kRopeMaxPairs) return false;
  if (!(r.base > 0.0)) return false;
  // half layout: the partner lane offset (rope_dim / 2) / EPL of the key kernel must be a
  // power of two, and the query kernel's 8-value chunks must not straddle rope_dim / 2
  if (!r.interleaved && r.rope_dim > 0) {
    const int half = r.rope_dim / 2;
    if (half % epl || half % 8) return false;
    const int off = half / epl;
    if (off & (off - 1)) return false;
  }
  return true;
}

cudaError_t launch_rope_append(const void* src, int src_is_f32, int64_t rows, int32_t d, const int64_t* dst_rows,
                               const int32_t* positions, int64_t capacity, const RopeParams& r, int fp8, void* cache,
                               float* scale, int* err, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int64_t per_cta = static_cast<int64_t>(kRopeWarps) * kAppendRowsPerWarp;
  const unsigned blocks = static_cast<unsigned>((rows + per_cta - 1) / per_cta);
  const unsigned threads = kRopeWarps * 32;
  if (d == 64) {
    if (r.interleaved)
      rope_append_kernel<64, true><<<blocks, threads, 0, stream>>>(src, src_is_f32, rows, dst_rows, positions,
                                                                   capacity, r, fp8, cache, scale, err);
    else
      rope_append_kernel<64, false><<<blocks, threads, 0, stream>>>(src, src_is_f32, rows, dst_rows, positions,
                                                                    capacity, r, fp8, cache, scale, err);
  } else {
    if (r.interleaved)
      rope_append_kernel<128, true><<<blocks, threads, 0, stream>>>(src, src_is_f32, rows, dst_rows, positions,
                                                                    capacity, r, fp8, cache, scale, err);
    else
      rope_append_kernel<128, false><<<blocks, threads, 0, stream>>>(src, src_is_f32, rows, dst_rows, positions,
                                                                     capacity, r, fp8, cache, scale, err);
  }
  return cudaGetLastError();
}

cudaError_t launch_rope_queries(const void* src, int src_is_f32, int64_t T, int32_t H, int32_t d,
                                const int32_t* positions, const RopeParams& r, int fp8, void* dst, float* scale,
                                int* err, int sms, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const uint8_t* s = static_cast<const uint8_t*>(src);
  if (d == 64) {
    if (r.interleaved) return launch_queries_cpt<64, true>(s, src_is_f32, T, H, positions, r, fp8, dst, scale, err, sms, stream);
    return launch_queries_cpt<64, false>(s, src_is_f32, T, H, positions, r, fp8, dst, scale, err, sms, stream);
  }
  if (r.interleaved) return launch_queries_cpt<128, true>(s, src_is_f32, T, H, positions, r, fp8, dst, scale, err, sms, stream);
  return launch_queries_cpt<128, false>(s, src_is_f32, T, H, positions, r, fp8, dst, scale, err, sms, stream);
}

}  // namespace dsa
