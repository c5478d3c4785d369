// Indexer logits on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Computes, for every query row t of a work item and every key s of a 128-key
// tile,
//     I[t, s] = k_scale[s] * sum_h w'[t, h] * ReLU( q[t, h, :] . k[s, :] )
//     w'[t, h] = w[t, h] * q_scale[t] / sqrt(d)
// which is the score of page "从原理到代码：手把手教你理解DeepSeek-V3.2的闪电索引器设计"
// §2.1 (and "Lightning Indexer 详解" §4) with one key per token shared by every head;
// positive scales move through the ReLU unchanged.  Only keys at or before the
// query's position are stored (the causal mask of the first page, §3 step 5); the
// rest of a score row is never written and never read.
//
// Mapping ("swap AB"): the key tile is the UMMA A operand (M = 128 keys), the
// item's queries x heads are the B operand (N = queries_per_acc * H), both
// K-major in 128-byte-swizzled shared memory written by TMA.  The fp32
// accumulator sits in TMEM with TMEM lane = key, so each epilogue thread owns
// one key and reduces over heads in registers: no cross-thread reduction, and
// score stores are coalesced along s.  The [T, H, S] logits never leave TMEM.
//
// Warp roles (one CTA per SM, persistent over a host-built list of work items):
//   warp 0      TMA producer: Q block once per item, then a ring of K tiles
//   warp 1      TMEM allocator and single-thread UMMA issuer
//   warps 2..   epilogue: tcgen05.ld -> ReLU / weighted head sum / scale / mask -> store
// Accumulators form a ring of TMEM buffers so the epilogue of one tile overlaps
// the MMAs of the next.  Every wait is bounded (see ptx.cuh).
#include <cuda_runtime.h>

#include <type_traits>

#include "internal.h"
#include "ptx.cuh"

namespace dsa {

namespace {

#ifndef DSA_SCALE_PREFETCH
#define DSA_SCALE_PREFETCH 4
#endif
constexpr int kScalePrefetch = DSA_SCALE_PREFETCH;   // tiles of FP8 key scales in flight ahead of the epilogue
#ifndef DSA_TMEM_X64
#define DSA_TMEM_X64 0                  // one 64-column TMEM load per query instead of two
#endif

template <int H_, int D_, bool FP8_, int TPA_, int NG_, int NE_, int STAGES_, int EG_ = 1, bool PF_ = false>
struct Cfg {
  static constexpr bool PF = PF_;                   // a prefill configuration (else decode)
  static constexpr int H = H_, D = D_, TPA = TPA_, NG = NG_, NE = NE_, STAGES = STAGES_;
  // Epilogue warps form EG groups; group g drains accumulators g, g+EG, ... so EG
  // accumulators are drained at once.  Inside a group, the SPLIT warps that share a TMEM
  // subpartition split the accumulator's queries.
  static constexpr int EG = EG_;
  static constexpr int NEG = NE / EG;
  static constexpr int SPLIT = NEG / 4;
  static_assert(NEG % 4 == 0 && NE % EG == 0, "epilogue groups cover the 4 TMEM subpartitions");
  static constexpr bool FP8 = FP8_;
  static constexpr int ESZ = FP8 ? 1 : 2;
  static constexpr int ROW_BYTES = D * ESZ;
  static_assert(ROW_BYTES % 128 == 0, "rows must be whole 128-byte swizzle spans");
  static constexpr int KB = ROW_BYTES / 128;         // 128-byte K blocks per row
  static constexpr int KB_ELEMS = 128 / ESZ;         // elements per K block
  static constexpr int KSTEPS = 4;                   // UMMA K steps of 32 bytes per K block
  static constexpr int BM = kKeyTile;                // keys per tile (UMMA M)
  static constexpr int N = TPA * H;                  // UMMA N per accumulator
  static_assert(N % 32 == 0 && N >= 32 && N <= 256, "accumulator width");
  static constexpr int NT = TPA * NG;                // queries per work item
  static constexpr int ACC_COLS = N;
  static constexpr int NBUF = (512 / N) < 4 ? (512 / N) : 4;
  static constexpr int TMEM_COLS_RAW = NBUF * N;
  static constexpr int TMEM_COLS = TMEM_COLS_RAW <= 32 ? 32 : TMEM_COLS_RAW <= 64 ? 64
                                 : TMEM_COLS_RAW <= 128 ? 128 : TMEM_COLS_RAW <= 256 ? 256 : 512;
  static constexpr int K_BLOCK_BYTES = BM * 128;     // one K block of a key tile
  static constexpr int K_TILE_BYTES = KB * K_BLOCK_BYTES;
  static constexpr int Q_BLOCK_BYTES = N * 128;      // one K block of one query group
  static_assert(Q_BLOCK_BYTES % 1024 == 0, "swizzle atoms must stay 1024-byte aligned");
  static constexpr int Q_BYTES = NG * KB * Q_BLOCK_BYTES;
  static constexpr int THREADS = (2 + NE) * 32;
  static_assert(EG <= NBUF, "each epilogue group needs its own accumulator buffer");
  // Register budget per thread decides how many TMEM columns stay live: 2 queries (192
  // threads, up to 255 registers), 1 query (up to 168), one 32-column chunk (fewer).
  static constexpr int QB = THREADS <= 256 ? 2 : 1;
  static constexpr bool CHUNKED = THREADS > 384;
  // every epilogue warp owns exactly one query of the work item: its head weights stay
  // in registers for the whole item
  static constexpr bool ONE_QUERY_PER_WARP = (NG == 1) && (TPA == SPLIT) && (H == 64) && !CHUNKED && !PF;
  // epilogue warps sleep inside their accumulator waits only when there are so many of
  // them that spinning would take issue slots from the ones computing
#ifdef DSA_EPI_SLEEP_MIN
  static constexpr bool EPI_SLEEP = NE >= DSA_EPI_SLEEP_MIN;
#else
  static constexpr bool EPI_SLEEP = NE >= 16;
#endif
  // the producer and MMA lanes sleep in their waits when the epilogue, not their
  // latency, sets the pace (prefill): then they leave the issue slots to the epilogue
  static constexpr bool PIPE_SLEEP = PF;
  // decode configurations can bin every row for the top-k (prefill ones compile no such code)
  // bf16 decode configurations bin every row for the top-k in the epilogue, where the HBM-bound
  // loop leaves the epilogue slack; FP8 decode (twice the keys per byte) leaves it none, so its
  // rows are binned by a separate pass over the score rows, and prefill configurations not at all
  static constexpr bool HIST = NG == 1 && !FP8 && !PF;
  // Prefill configurations (several query groups share each K tile, 64 heads) drain their
  // accumulators in a dedicated loop: every epilogue warp owns the same QPW query slots of
  // every group for a whole work item, so row pointers, weight addresses and causal limits are
  // set once per item, and the tiles whose keys precede every query of the item (all but the
  // last one or two) run without any mask or per-query test.
  static constexpr bool PREFILL_FAST = PF && H == 64 && EG == 1 && (TPA % SPLIT) == 0;
  static constexpr int QPW = PREFILL_FAST ? TPA / SPLIT : 1;   // queries per warp per group
  // shared memory carve-up (offsets from a 1024-byte aligned base)
  static constexpr int OFF_K = 0;
  static constexpr int OFF_Q = OFF_K + STAGES * K_TILE_BYTES;
  // each epilogue warp keeps its own copy of the item's w' and score-row offsets,
  // so the epilogue warps never wait on one another
  static constexpr int OFF_W = OFF_Q + Q_BYTES;
  static constexpr int W_WARP_FLOATS = NT * H;
  static constexpr int OFF_ROW = OFF_W + NE * W_WARP_FLOATS * 4;
  static constexpr int OFF_BAR = (OFF_ROW + NE * NT * 8 + 7) / 8 * 8;
  static constexpr int NUM_BARS = 2 * STAGES + 2 + 2 * NBUF + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  // + alignment slack; at least 120 KB so that one CTA holds an SM (and all its TMEM)
  static constexpr int SMEM_RAW = OFF_MISC + 16 + 1024;
  static constexpr int SMEM_BYTES = SMEM_RAW > 120 * 1024 ? SMEM_RAW : 120 * 1024;
  static constexpr uint32_t IDESC = make_idesc(FP8 ? 0u : 1u, BM, N);
};

// Counts this warp's 32 scores (one per lane, invalid lanes skipped) in the row's coarse
// histogram.  Lanes whose keys share a bin are merged first (one atomic per distinct bin
// per warp): a row's scores crowd into a few bins, and same-address atomics serialise at
// the L2.  Called by all 32 lanes together.
__device__ __forceinline__ void coarse_hist_add(uint32_t* row_hist, float v, bool valid) {
  const uint32_t bin = valid ? order_key(__float_as_uint(v)) >> kHistShift : 0xFFFFFFFFu;
  const uint32_t peers = __match_any_sync(0xffffffffu, bin);
  if (valid && static_cast<int>(threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(row_hist + bin, __popc(peers));
}

template <class C>
__device__ __forceinline__ void issue_umma(uint32_t d_tmem, uint32_t k_stage_addr, uint32_t q_group_addr) {
#pragma unroll
  for (int kb = 0; kb < C::KB; ++kb) {
#pragma unroll
    for (int ks = 0; ks < C::KSTEPS; ++ks) {
      const uint64_t a = sdesc_kmajor_sw128(k_stage_addr + kb * C::K_BLOCK_BYTES + ks * 32);
      const uint64_t b = sdesc_kmajor_sw128(q_group_addr + kb * C::Q_BLOCK_BYTES + ks * 32);
      const uint32_t acc = (kb | ks) != 0;
      if constexpr (C::FP8)
        umma_f8(d_tmem, a, b, C::IDESC, acc);
      else
        umma_f16(d_tmem, a, b, C::IDESC, acc);
    }
  }
}

// Two independent tiles (separate accumulators) issued with their K steps interleaved,
// so no UMMA waits for the one just before it to finish its read-modify-write of D.
template <class C>
__device__ __forceinline__ void issue_umma_pair(uint32_t d0, uint32_t k0, uint32_t d1, uint32_t k1, uint32_t q) {
#pragma unroll
  for (int kb = 0; kb < C::KB; ++kb) {
#pragma unroll
    for (int ks = 0; ks < C::KSTEPS; ++ks) {
      const uint64_t b = sdesc_kmajor_sw128(q + kb * C::Q_BLOCK_BYTES + ks * 32);
      const uint64_t a0 = sdesc_kmajor_sw128(k0 + kb * C::K_BLOCK_BYTES + ks * 32);
      const uint64_t a1 = sdesc_kmajor_sw128(k1 + kb * C::K_BLOCK_BYTES + ks * 32);
      const uint32_t acc = (kb | ks) != 0;
      if constexpr (C::FP8) {
        umma_f8(d0, a0, b, C::IDESC, acc);
        umma_f8(d1, a1, b, C::IDESC, acc);
      } else {
        umma_f16(d0, a0, b, C::IDESC, acc);
        umma_f16(d1, a1, b, C::IDESC, acc);
      }
    }
  }
}

// a0, a1 += w[h] * max(x[h], 0) over 32 accumulator columns already loaded into r,
// with packed fp32x2 FMAs: 1.5 issue slots per element.
__device__ __forceinline__ void relu_wsum32(const uint32_t (&r)[32], const float* __restrict__ w, float2& a0,
                                            float2& a1) {
#pragma unroll
  for (int h = 0; h < 32; h += 4) {
    const float4 wv = *reinterpret_cast<const float4*>(w + h);
    const float2 x01 = make_float2(fmaxf(__uint_as_float(r[h]), 0.f), fmaxf(__uint_as_float(r[h + 1]), 0.f));
    const float2 x23 = make_float2(fmaxf(__uint_as_float(r[h + 2]), 0.f), fmaxf(__uint_as_float(r[h + 3]), 0.f));
    a0 = __ffma2_rn(make_float2(wv.x, wv.y), x01, a0);
    a1 = __ffma2_rn(make_float2(wv.z, wv.w), x23, a1);
  }
}

// The same with the 32 weights already in registers.
__device__ __forceinline__ void relu_wsum32_reg(const uint32_t (&r)[32], const float2 (&w)[16], float2& a0,
                                                float2& a1) {
#pragma unroll
  for (int h = 0; h < 32; h += 4) {
    const float2 x01 = make_float2(fmaxf(__uint_as_float(r[h]), 0.f), fmaxf(__uint_as_float(r[h + 1]), 0.f));
    const float2 x23 = make_float2(fmaxf(__uint_as_float(r[h + 2]), 0.f), fmaxf(__uint_as_float(r[h + 3]), 0.f));
    a0 = __ffma2_rn(w[h / 2], x01, a0);
    a1 = __ffma2_rn(w[h / 2 + 1], x23, a1);
  }
}

// The same over one query's CPT*32 columns.
template <int CPT>
__device__ __forceinline__ float relu_wsum(const uint32_t (&r)[CPT][32], const float* __restrict__ w) {
  float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < CPT; ++c) relu_wsum32(r[c], w + c * 32, a0, a1);
  return (a0.x + a0.y) + (a1.x + a1.y);
}

#ifdef DSA_PIPE_STATS
// Tuning builds only: cycles each role spends waiting, summed over CTAs.
// 0 producer waits for a free K stage, 1 MMA waits for a loaded K tile, 2 MMA waits for a
// free accumulator, 3 epilogue (first warp) waits for a finished accumulator, 4 epilogue
// (first warp) compute, 5 CTA cycles, 6 producer waits for the Q buffer, 7 MMA waits for Q.
__device__ unsigned long long g_pipe_stats[12];
#define DSA_TIMED(slot, expr) ([&]() { const long long t0_ = clock64(); const bool r_ = (expr); \
                                        st_[slot] += clock64() - t0_; return r_; }())
#else
#define DSA_TIMED(slot, expr) (expr)
#endif

// Tuning knobs of the prefill epilogue (build-time; the defaults are the measured best):
// accumulator chains per query in the weighted head sum, and whether a warp with several
// query slots loads all of them before computing.
#ifndef DSA_EPI_CHAINS
#define DSA_EPI_CHAINS 2
#endif
#ifndef DSA_EPI_PAIR
#define DSA_EPI_PAIR 0
#endif
// 1: the next slot's (or half's) TMEM columns are loaded while the current ones are summed
#ifndef DSA_EPI_PIPE
#define DSA_EPI_PIPE 0
#endif

// The same with four accumulator chains: shorter dependent FFMA2 sequences.
__device__ __forceinline__ void relu_wsum32_c4(const uint32_t (&r)[32], const float* __restrict__ w, float2 (&a)[4]) {
#pragma unroll
  for (int h = 0; h < 32; h += 8) {
    const float4 w0 = *reinterpret_cast<const float4*>(w + h);
    const float4 w1 = *reinterpret_cast<const float4*>(w + h + 4);
    const float2 x0 = make_float2(fmaxf(__uint_as_float(r[h]), 0.f), fmaxf(__uint_as_float(r[h + 1]), 0.f));
    const float2 x1 = make_float2(fmaxf(__uint_as_float(r[h + 2]), 0.f), fmaxf(__uint_as_float(r[h + 3]), 0.f));
    const float2 x2 = make_float2(fmaxf(__uint_as_float(r[h + 4]), 0.f), fmaxf(__uint_as_float(r[h + 5]), 0.f));
    const float2 x3 = make_float2(fmaxf(__uint_as_float(r[h + 6]), 0.f), fmaxf(__uint_as_float(r[h + 7]), 0.f));
    a[0] = __ffma2_rn(make_float2(w0.x, w0.y), x0, a[0]);
    a[1] = __ffma2_rn(make_float2(w0.z, w0.w), x1, a[1]);
    a[2] = __ffma2_rn(make_float2(w1.x, w1.y), x2, a[2]);
    a[3] = __ffma2_rn(make_float2(w1.z, w1.w), x3, a[3]);
  }
}

__device__ __forceinline__ float chains_sum(const float2 (&a)[4]) {
  const float2 s = __fadd2_rn(__fadd2_rn(a[0], a[1]), __fadd2_rn(a[2], a[3]));
  return s.x + s.y;
}

// sum_h w[h] * max(x[h], 0) over one query's 64 accumulator columns (two 32-column halves
// already loaded), w' read from shared memory.
__device__ __forceinline__ float relu_wsum64(const uint32_t (&r0)[32], const uint32_t (&r1)[32],
                                            const float* __restrict__ w) {
  float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
  relu_wsum32(r0, w, a0, a1);
  relu_wsum32(r1, w + 32, a0, a1);
  return (a0.x + a0.y) + (a1.x + a1.y);
}

// The prefill epilogue for one work item over a plain cache (see Cfg::PREFILL_FAST): the
// warp's query slots j = g * TPA + part + u * SPLIT of every group g, tiles [kt_begin, kt_end).
// Tiles before kt_full hold only keys at or before the item's first query, so every query
// stores every key of them; the remaining (at most two) tiles mask per query and key.
template <class C>
__device__ __forceinline__ void prefill_item(const LogitsArgs& args, const LogitsItem& wi, uint32_t tmem_base, int sub,
                                             int lane, int part, const float* wq, const int64_t* rowoff,
                                             uint64_t* acc_full, uint64_t* acc_empty, volatile int* abort_flag,
                                             float (&ks_ring)[kScalePrefetch], uint32_t& acc_iter, bool& ok,
                                             long long* st_) {
  (void)st_;
  constexpr int QPW = C::QPW, SPLIT = C::SPLIT, PF = kScalePrefetch;
  const int groups = (wi.n_tok + C::TPA - 1) / C::TPA;
  float* rowp[C::NG][QPW];        // score row of each slot, advanced to this thread's key of tile 0
  const float* wp[C::NG][QPW];    // its w' in this warp's copy
  int lastk[C::NG][QPW];          // its position: the last key it sees
  bool live[C::NG][QPW];
#pragma unroll
  for (int g = 0; g < C::NG; ++g) {
#pragma unroll
    for (int u = 0; u < QPW; ++u) {
      const int j = g * C::TPA + part + u * SPLIT;
      live[g][u] = j < wi.n_tok;
      const int jj = live[g][u] ? j : 0;
      rowp[g][u] = args.scores + rowoff[jj] + sub * 32 + lane;
      wp[g][u] = wq + jj * C::H;
      lastk[g][u] = wi.pos0 + j;
    }
  }
  const int pos_last = wi.pos0 + wi.n_tok - 1;
  auto load_scale = [&](int kt) -> float {
    const int key = kt * C::BM + sub * 32 + lane;
    const int64_t krow = wi.k_row0 + key;
    return (kt < wi.kt_end && key <= pos_last && krow < args.k_capacity) ? __ldg(args.k_scale + krow) : 0.f;
  };
  const int kt_full = max(wi.kt_begin, min(wi.kt_end, (wi.pos0 + 1) / C::BM));
  auto tiles = [&](auto masked, int kt0, int kt1) {
    constexpr bool kMasked = decltype(masked)::value;
    for (int kt = kt0; kt < kt1 && ok; ++kt) {
      const int key0 = kt * C::BM;
      const int key = key0 + sub * 32 + lane;
      float kscale = 1.f;
      if constexpr (C::FP8) {
        kscale = ks_ring[0];
#pragma unroll
        for (int i = 0; i + 1 < PF; ++i) ks_ring[i] = ks_ring[i + 1];
        ks_ring[PF - 1] = load_scale(kt + PF);
      }
#pragma unroll
      for (int g = 0; g < C::NG; ++g) {
        if (g >= groups || !ok) break;
        const int b = acc_iter % C::NBUF;
        if (!DSA_TIMED(3, mbar_wait<C::EPI_SLEEP>(&acc_full[b], (acc_iter / C::NBUF) & 1, abort_flag))) {
          ok = false;
          break;
        }
        ++acc_iter;
#ifdef DSA_PIPE_STATS
        const long long tc0_ = clock64();
#endif
        tc_fence_after();
        const uint32_t tbase = tmem_base + (static_cast<uint32_t>(sub * 32) << 16) + b * C::ACC_COLS;
        if constexpr (C::CHUNKED && DSA_EPI_PIPE && QPW == 1) {
          // one slot: its second half loads while the first is summed
          if (live[g][0] && (!kMasked || key0 <= lastk[g][0])) {
            const uint32_t col = tbase + part * C::H;
            uint32_t ra[32], rb[32];
            float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
            tmem_ld_32x32b_x32(col, ra);
            tmem_ld_wait();
            tmem_ld_32x32b_x32(col + 32, rb);
            relu_wsum32(ra, wp[g][0], a0, a1);
            tmem_ld_wait();
            relu_wsum32(rb, wp[g][0] + 32, a0, a1);
            const float v = ((a0.x + a0.y) + (a1.x + a1.y)) * kscale;
            if (!kMasked || key <= lastk[g][0]) rowp[g][0][key0] = v;
          }
        } else if constexpr (!C::CHUNKED && DSA_EPI_PIPE && QPW == 2) {
          // two slots: the second slot's 64 columns load while the first slot is summed (both
          // slots' columns are read whether or not the slot holds a query: harmless, and it keeps
          // the loads unconditional)
          const uint32_t col0 = tbase + part * C::H, col1 = tbase + (part + SPLIT) * C::H;
          uint32_t ra0[32], ra1[32], rb0[32], rb1[32];
          tmem_ld_32x32b_x32(col0, ra0);
          tmem_ld_32x32b_x32(col0 + 32, ra1);
          tmem_ld_wait();
          tmem_ld_32x32b_x32(col1, rb0);
          tmem_ld_32x32b_x32(col1 + 32, rb1);
          if (live[g][0] && (!kMasked || key0 <= lastk[g][0])) {
            const float v = relu_wsum64(ra0, ra1, wp[g][0]) * kscale;
            if (!kMasked || key <= lastk[g][0]) rowp[g][0][key0] = v;
          }
          tmem_ld_wait();
          if (live[g][1] && (!kMasked || key0 <= lastk[g][1])) {
            const float v = relu_wsum64(rb0, rb1, wp[g][1]) * kscale;
            if (!kMasked || key <= lastk[g][1]) rowp[g][1][key0] = v;
          }
        } else if constexpr (C::CHUNKED) {
          // many epilogue warps, few registers each: one 32-column half at a time
#pragma unroll
          for (int u = 0; u < QPW; ++u) {
            if (live[g][u] && (!kMasked || key0 <= lastk[g][u])) {
              const uint32_t col = tbase + (part + u * SPLIT) * C::H;
              uint32_t r[32];
#if DSA_EPI_CHAINS == 4
              float2 a[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                             make_float2(0.f, 0.f)};
              tmem_ld_32x32b_x32(col, r);
              tmem_ld_wait();
              relu_wsum32_c4(r, wp[g][u], a);
              tmem_ld_32x32b_x32(col + 32, r);
              tmem_ld_wait();
              relu_wsum32_c4(r, wp[g][u] + 32, a);
              const float v = chains_sum(a) * kscale;
#else
              float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
              tmem_ld_32x32b_x32(col, r);
              tmem_ld_wait();
              relu_wsum32(r, wp[g][u], a0, a1);
              tmem_ld_32x32b_x32(col + 32, r);
              tmem_ld_wait();
              relu_wsum32(r, wp[g][u] + 32, a0, a1);
              const float v = ((a0.x + a0.y) + (a1.x + a1.y)) * kscale;
#endif
              if (!kMasked || key <= lastk[g][u]) rowp[g][u][key0] = v;
            }
          }
        } else if (DSA_EPI_PAIR && QPW == 2) {
          // both slots' 128 columns in flight behind one wait, then two independent sums
          uint32_t r[2][2][32];
          bool go[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            go[u] = live[g][u] && (!kMasked || key0 <= lastk[g][u]);
            const uint32_t col = tbase + (part + u * SPLIT) * C::H;
            if (go[u]) {
              tmem_ld_32x32b_x32(col, r[u][0]);
              tmem_ld_32x32b_x32(col + 32, r[u][1]);
            }
          }
          if (go[0] || go[1]) tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            if (go[u]) {
              const float v = relu_wsum64(r[u][0], r[u][1], wp[g][u]) * kscale;
              if (!kMasked || key <= lastk[g][u]) rowp[g][u][key0] = v;
            }
          }
        } else {
          // one slot at a time, its 64 columns in flight behind one wait
#pragma unroll
          for (int u = 0; u < QPW; ++u) {
            if (live[g][u] && (!kMasked || key0 <= lastk[g][u])) {
              const uint32_t col = tbase + (part + u * SPLIT) * C::H;
              uint32_t r0[32], r1[32];
              tmem_ld_32x32b_x32(col, r0);
              tmem_ld_32x32b_x32(col + 32, r1);
              tmem_ld_wait();
              const float v = relu_wsum64(r0, r1, wp[g][u]) * kscale;
              if (!kMasked || key <= lastk[g][u]) rowp[g][u][key0] = v;
            }
          }
        }
        tc_fence_before();
        __syncwarp();
#ifdef DSA_PIPE_STATS
        st_[4] += clock64() - tc0_;
#endif
        if (lane == 0) mbar_arrive(&acc_empty[b]);
      }
    }
  };
  tiles(std::false_type{}, wi.kt_begin, kt_full);
  tiles(std::true_type{}, kt_full, wi.kt_end);
}


template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
logits_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q,
              const LogitsArgs args) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the __shared__ array by an offset so that the
  // compiler keeps the shared address space (ld.shared / st.shared with 32-bit addresses)
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* k_full = bars;
  uint64_t* k_empty = bars + C::STAGES;
  uint64_t* q_full = bars + 2 * C::STAGES;
  uint64_t* q_empty = q_full + 1;
  uint64_t* acc_full = q_full + 2;
  uint64_t* acc_empty = acc_full + C::NBUF;
  uint64_t* drain = acc_empty + C::NBUF;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
#ifdef DSA_PIPE_STATS
  long long st_[12] = {0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0};
  const long long t_start_ = clock64();
#endif

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int b = 0; b < C::NBUF; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], C::NEG);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_q);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t smem_base = smem_addr(smem);
  // The prologue above overlaps the previous kernel; its outputs (appended keys, quantised
  // queries) are read only after this point.  The next kernel may start its own prologue.
  grid_dependency_wait();
  launch_dependents();
  const int item_begin = args.cta_items[blockIdx.x];
  const int item_end = args.cta_items[blockIdx.x + 1];

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_k = C::NG > 1 ? policy_evict_last() : policy_evict_first();
      const uint64_t pol_q = policy_evict_first();
      uint32_t k_iter = 0, item_iter = 0;
      bool ok = true;
      for (int it = item_begin; it < item_end && ok; ++it) {
        const LogitsItem wi = args.items[it];
        if (!DSA_TIMED(6, mbar_wait<C::PIPE_SLEEP>(q_empty, (item_iter & 1) ^ 1, abort_flag))) { ok = false; break; }
        mbar_arrive_expect_tx(q_full, C::Q_BYTES);
        for (int g = 0; g < C::NG; ++g)
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_2d(smem + C::OFF_Q + (g * C::KB + kb) * C::Q_BLOCK_BYTES, &tmap_q, q_full,
                        kb * C::KB_ELEMS, (wi.q_row0 + g * C::TPA) * C::H, pol_q);
        ++item_iter;
        for (int kt = wi.kt_begin; kt < wi.kt_end; ++kt, ++k_iter) {
          const int s = k_iter % C::STAGES;
          if (!DSA_TIMED(0, mbar_wait<C::PIPE_SLEEP>(&k_empty[s], ((k_iter / C::STAGES) & 1) ^ 1, abort_flag))) { ok = false; break; }
          mbar_arrive_expect_tx(&k_full[s], C::K_TILE_BYTES);
          const int32_t y = static_cast<int32_t>(wi.k_row0 + static_cast<int64_t>(kt) * C::BM);
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_2d(smem + C::OFF_K + s * C::K_TILE_BYTES + kb * C::K_BLOCK_BYTES, &tmap_k, &k_full[s],
                        kb * C::KB_ELEMS, y, pol_k);
        }
      }
      // Drain: the last load issued on each stage (and the last Q load) must land
      // before this CTA may exit.  These waits end on their own; they are bounded anyway.
      const uint32_t issued = k_iter < static_cast<uint32_t>(C::STAGES) ? k_iter : C::STAGES;
      for (uint32_t i = 0; i < issued; ++i) {
        const uint32_t n = k_iter - 1 - i;
        volatile int never = 0;
        mbar_wait(&k_full[n % C::STAGES], (n / C::STAGES) & 1, &never);
      }
      if (item_iter > 0) {
        volatile int never = 0;
        mbar_wait(q_full, (item_iter - 1) & 1, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
#ifdef DSA_PIPE_STATS
      st_[10] += clock64() - t_start_;
#endif
      uint32_t k_iter = 0, acc_iter = 0, item_iter = 0;
      bool ok = true;
      for (int it = item_begin; it < item_end && ok; ++it) {
        const LogitsItem wi = args.items[it];
        const int groups = (wi.n_tok + C::TPA - 1) / C::TPA;
        if (!DSA_TIMED(7, mbar_wait<C::PIPE_SLEEP>(q_full, item_iter & 1, abort_flag))) { ok = false; break; }
        tc_fence_after();
        if constexpr (C::NG == 1) {
          // one accumulator per tile: issue tiles in pairs, their UMMA chains interleaved
          static_assert(C::NBUF >= 2 && C::STAGES >= 2, "a pair needs two accumulators and two stages");
          for (int kt = wi.kt_begin; kt < wi.kt_end && ok;) {
            const bool two = kt + 1 < wi.kt_end;
            const int s0 = k_iter % C::STAGES, s1 = (k_iter + 1) % C::STAGES;
            const int b0 = acc_iter % C::NBUF, b1 = (acc_iter + 1) % C::NBUF;
            if (!DSA_TIMED(1, mbar_wait(&k_full[s0], (k_iter / C::STAGES) & 1, abort_flag)) ||
                (two && !DSA_TIMED(1, mbar_wait(&k_full[s1], ((k_iter + 1) / C::STAGES) & 1, abort_flag))) ||
                !DSA_TIMED(2, mbar_wait(&acc_empty[b0], ((acc_iter / C::NBUF) & 1) ^ 1, abort_flag)) ||
                (two && !DSA_TIMED(2, mbar_wait(&acc_empty[b1], (((acc_iter + 1) / C::NBUF) & 1) ^ 1, abort_flag)))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t kaddr0 = smem_base + C::OFF_K + s0 * C::K_TILE_BYTES;
            const uint32_t kaddr1 = smem_base + C::OFF_K + s1 * C::K_TILE_BYTES;
            if (two)
              issue_umma_pair<C>(tmem_base + b0 * C::ACC_COLS, kaddr0, tmem_base + b1 * C::ACC_COLS, kaddr1,
                                 smem_base + C::OFF_Q);
            else
              issue_umma<C>(tmem_base + b0 * C::ACC_COLS, kaddr0, smem_base + C::OFF_Q);
            umma_commit(&acc_full[b0]);
            if (two) umma_commit(&acc_full[b1]);
            umma_commit(&k_empty[s0]);
            if (two) umma_commit(&k_empty[s1]);
            const int adv = two ? 2 : 1;
            kt += adv;
            k_iter += adv;
            acc_iter += adv;
          }
        } else
        for (int kt = wi.kt_begin; kt < wi.kt_end && ok; ++kt, ++k_iter) {
          const int s = k_iter % C::STAGES;
          if (!DSA_TIMED(1, mbar_wait<C::PIPE_SLEEP>(&k_full[s], (k_iter / C::STAGES) & 1, abort_flag))) { ok = false; break; }
          tc_fence_after();
          for (int g = 0; g < groups; ++g, ++acc_iter) {
            const int b = acc_iter % C::NBUF;
            if (!DSA_TIMED(2, mbar_wait<C::PIPE_SLEEP>(&acc_empty[b], ((acc_iter / C::NBUF) & 1) ^ 1, abort_flag))) { ok = false; break; }
            tc_fence_after();
#ifdef DSA_PIPE_STATS
            const long long ti0_ = clock64();
#endif
            issue_umma<C>(tmem_base + b * C::ACC_COLS, smem_base + C::OFF_K + s * C::K_TILE_BYTES,
                          smem_base + C::OFF_Q + g * C::KB * C::Q_BLOCK_BYTES);
#ifdef DSA_PIPE_STATS
            const long long ti1_ = clock64();
            st_[8] += ti1_ - ti0_;
#endif
            umma_commit(&acc_full[b]);
#ifdef DSA_PIPE_STATS
            st_[9] += clock64() - ti1_;
#endif
          }
          if (ok) umma_commit(&k_empty[s]);
        }
        if (ok) umma_commit(q_empty);
        ++item_iter;
      }
#ifdef DSA_PIPE_STATS
      const long long tl_end_ = clock64();
#endif
      // Let every issued UMMA finish before TMEM is released.
      umma_commit(drain);
      volatile int never = 0;
      mbar_wait(drain, 0, &never);
#ifdef DSA_PIPE_STATS
      st_[11] = tl_end_;                      // exit time minus this = drain + final barrier
#endif
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int ew = warp - 2;                  // 0 .. NE-1
    const int sub = warp & 3;                 // TMEM subpartition this warp may access
    constexpr int SPLIT = C::SPLIT;           // warps of a group sharing one subpartition
    const int grp = ew / C::NEG;              // accumulators grp, grp+EG, ... are this warp's
    const int part = (ew % C::NEG) / 4;       // which share of an accumulator's queries
    float* wq = reinterpret_cast<float*>(smem + C::OFF_W) + ew * C::W_WARP_FLOATS;
    int64_t* rowoff = reinterpret_cast<int64_t*>(smem + C::OFF_ROW) + ew * C::NT;
    uint32_t acc_iter = 0;
    bool ok = true;
    for (int it = item_begin; it < item_end && ok; ++it) {
      const LogitsItem wi = args.items[it];
      // counts score v of the item's query j in its row's coarse histogram; all lanes together
      auto hist_count = [&](int j, float v, bool valid) {
        coarse_hist_add(args.row_hist + static_cast<int64_t>(wi.q_row0 + j) * kHistBins, v, valid);
      };
      __syncwarp();                           // this warp is done with the previous item's copies
      for (int i = lane; i < wi.n_tok * C::H; i += 32) {
        const int j = i / C::H;
        float v = args.w[static_cast<int64_t>(wi.q_row0 + j) * C::H + (i - j * C::H)] * args.inv_sqrt_d;
        if constexpr (C::FP8) v *= args.q_scale[wi.q_row0 + j];
        wq[i] = v;
      }
      for (int j = lane; j < wi.n_tok; j += 32) rowoff[j] = args.row_off[wi.q_row0 + j];
      __syncwarp();
      float2 wr_lo[16], wr_hi[16];                // this warp's query's w' (ONE_QUERY_PER_WARP)
      if constexpr (C::ONE_QUERY_PER_WARP) {
        const int j = part < wi.n_tok ? part : 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          wr_lo[i] = *reinterpret_cast<const float2*>(wq + j * 64 + 2 * i);
          wr_hi[i] = *reinterpret_cast<const float2*>(wq + j * 64 + 32 + 2 * i);
        }
      }
      const int groups = (wi.n_tok + C::TPA - 1) / C::TPA;
      // last key query j sees: its position, or over a cache of one key per `cmp` tokens the
      // last block its position completes
      const int cmp = wi.cmp > 1 ? wi.cmp : 1;
      const int pos_last = cmp == 1 ? wi.pos0 + wi.n_tok - 1 : (wi.pos0 + wi.n_tok) / cmp - 1;
      // FP8 key scales are loaded kScalePrefetch tiles ahead of use, so the per-tile
      // global-memory latency overlaps the epilogues of the tiles in between.
      constexpr int PF = kScalePrefetch;
      float ks_ring[PF];
      auto load_scale = [&](int kt) -> float {
        const int key = kt * C::BM + sub * 32 + lane;
        const int64_t krow = wi.k_row0 + key;
        return (kt < wi.kt_end && key <= pos_last && krow < args.k_capacity) ? __ldg(args.k_scale + krow) : 0.f;
      };
      if constexpr (C::FP8) {
#pragma unroll
        for (int i = 0; i < PF; ++i) ks_ring[i] = load_scale(wi.kt_begin + i);
      }
      if constexpr (C::PREFILL_FAST) {
        if (cmp == 1) {
#ifdef DSA_PIPE_STATS
          prefill_item<C>(args, wi, tmem_base, sub, lane, part, wq, rowoff, acc_full, acc_empty, abort_flag,
                          ks_ring, acc_iter, ok, st_);
#else
          prefill_item<C>(args, wi, tmem_base, sub, lane, part, wq, rowoff, acc_full, acc_empty, abort_flag,
                          ks_ring, acc_iter, ok, nullptr);
#endif
          continue;
        }
      }
      // the tile loop, compiled twice: plain causal limits (one add per query) and limits
      // over a compressed cache (a division), so the plain loop carries no compression test
      auto tile_loop = [&](auto compressed) {
        constexpr bool kCompressed = decltype(compressed)::value;
        auto last_key = [&](int j) -> int {
          if constexpr (kCompressed) return (wi.pos0 + j + 1) / cmp - 1;
          else return wi.pos0 + j;
        };
        for (int kt = wi.kt_begin; kt < wi.kt_end && ok; ++kt) {
          const int key0 = kt * C::BM;                      // first key of the tile
          const int key = key0 + sub * 32 + lane;           // this thread's key (its TMEM lane)
          float kscale = 1.f;
          if constexpr (C::FP8) {
            kscale = ks_ring[0];
  #pragma unroll
            for (int i = 0; i + 1 < PF; ++i) ks_ring[i] = ks_ring[i + 1];
            ks_ring[PF - 1] = load_scale(kt + PF);
          }
          for (int g = 0; g < groups; ++g, ++acc_iter) {
            if (C::EG > 1 && static_cast<int>(acc_iter % C::EG) != grp) continue;   // another group's
            const int b = acc_iter % C::NBUF;
            if (!DSA_TIMED(3, mbar_wait<C::EPI_SLEEP>(&acc_full[b], (acc_iter / C::NBUF) & 1, abort_flag))) { ok = false; break; }
  #ifdef DSA_PIPE_STATS
            const long long tc0_ = clock64();
  #endif
            tc_fence_after();
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(sub * 32) << 16) + b * C::ACC_COLS;
            const int j_lo = g * C::TPA;
            const int j_hi = min(j_lo + C::TPA, wi.n_tok);
            if constexpr (C::ONE_QUERY_PER_WARP) {
              const int j = part;                                        // this warp's query
              if (j < wi.n_tok && key0 <= last_key(j)) {                 // warp-uniform
                float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
  #if DSA_TMEM_X64
                uint32_t r[64];
                tmem_ld_32x32b_x64(tbase + j * 64, r);
                tmem_ld_wait();
                relu_wsum32_reg(*reinterpret_cast<uint32_t(*)[32]>(r), wr_lo, a0, a1);
                relu_wsum32_reg(*reinterpret_cast<uint32_t(*)[32]>(r + 32), wr_hi, a0, a1);
  #else
                uint32_t r0[32], r1[32];
                tmem_ld_32x32b_x32(tbase + j * 64, r0);
                tmem_ld_32x32b_x32(tbase + j * 64 + 32, r1);
                tmem_ld_wait();
                relu_wsum32_reg(r0, wr_lo, a0, a1);
                relu_wsum32_reg(r1, wr_hi, a0, a1);
  #endif
                const float v = ((a0.x + a0.y) + (a1.x + a1.y)) * kscale;
                const bool valid = key <= last_key(j);
                if (valid) args.scores[rowoff[j] + key] = v;
                if (C::HIST && args.row_hist) hist_count(j, v, valid);
              }
            } else if constexpr (C::H >= 32 && C::CHUNKED) {
              // many epilogue warps: one 32-column chunk in registers at a time
              constexpr int CPT = C::H / 32;
              for (int j = j_lo + part; j < j_hi; j += SPLIT) {
                if (key0 > last_key(j)) continue;                        // the tile is after this query
                float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
  #pragma unroll
                for (int c = 0; c < CPT; ++c) {
                  uint32_t r[32];
                  tmem_ld_32x32b_x32(tbase + (j - j_lo) * C::H + c * 32, r);
                  tmem_ld_wait();
                  relu_wsum32(r, wq + j * C::H + c * 32, a0, a1);
                }
                const float v = ((a0.x + a0.y) + (a1.x + a1.y)) * kscale;
                const bool valid = key <= last_key(j);
                if (valid) args.scores[rowoff[j] + key] = v;
                if (C::HIST && args.row_hist) hist_count(j, v, valid);
              }
            } else if constexpr (C::H >= 32) {
              // QB queries per pass: their loads are in flight behind one tcgen05.wait::ld
              constexpr int CPT = C::H / 32;
              for (int j0 = j_lo + part; j0 < j_hi; j0 += C::QB * SPLIT) {
                uint32_t r[C::QB][CPT][32];
                bool live[C::QB];
                bool any = false;
  #pragma unroll
                for (int u = 0; u < C::QB; ++u) {
                  const int j = j0 + u * SPLIT;
                  live[u] = j < j_hi && key0 <= last_key(j);             // warp-uniform
                  any |= live[u];
                  if (live[u]) {
  #pragma unroll
                    for (int c = 0; c < CPT; ++c) tmem_ld_32x32b_x32(tbase + (j - j_lo) * C::H + c * 32, r[u][c]);
                  }
                }
                if (!any) continue;                                      // the tile is after these queries
                tmem_ld_wait();
  #pragma unroll
                for (int u = 0; u < C::QB; ++u) {
                  const int j = j0 + u * SPLIT;
                  if (live[u]) {
                    const float v = relu_wsum<CPT>(r[u], wq + j * C::H) * kscale;
                    const bool valid = key <= last_key(j);
                    if (valid) args.scores[rowoff[j] + key] = v;
                    if (C::HIST && args.row_hist) hist_count(j, v, valid);
                  }
                }
              }
            } else {
              // H < 32: one 32-column load holds 32/H queries
              constexpr int QPC = 32 / C::H;
              for (int c = part; c < C::N / 32; c += SPLIT) {
                const int jc = j_lo + c * QPC;
                if (jc >= j_hi) break;
                uint32_t r[32];
                tmem_ld_32x32b_x32(tbase + c * 32, r);
                tmem_ld_wait();
  #pragma unroll
                for (int u = 0; u < QPC; ++u) {
                  const int j = jc + u;
                  if (j < j_hi) {
                    float acc = 0.f;
  #pragma unroll
                    for (int h = 0; h < C::H; ++h)
                      acc = fmaf(wq[j * C::H + h], fmaxf(__uint_as_float(r[u * C::H + h]), 0.f), acc);
                    const float v = acc * kscale;
                    const bool valid = key <= last_key(j);
                    if (valid) args.scores[rowoff[j] + key] = v;
                    if (C::HIST && args.row_hist) hist_count(j, v, valid);
                  }
                }
              }
            }
            tc_fence_before();
            __syncwarp();
  #ifdef DSA_PIPE_STATS
            st_[4] += clock64() - tc0_;
  #endif
            if (lane == 0) mbar_arrive(&acc_empty[b]);
          }
        }
      };
      if (cmp == 1)
        tile_loop(std::false_type{});
      else
        tile_loop(std::true_type{});
    }
  }

  __syncwarp();                              // the single-lane roles rejoin their warps
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort_flag) record_error(args.err, DSA_DEVERR_TIMEOUT, blockIdx.x);
#ifdef DSA_PIPE_STATS
  if (threadIdx.x == 0) {                     // producer lane
    atomicAdd(&g_pipe_stats[0], st_[0]);
    atomicAdd(&g_pipe_stats[6], st_[6]);
    atomicAdd(&g_pipe_stats[5], clock64() - t_start_);
  }
  if (threadIdx.x == 32) {                    // MMA lane
    atomicAdd(&g_pipe_stats[10], st_[10]);
    atomicAdd(&g_pipe_stats[11], clock64() - st_[11]);
    atomicAdd(&g_pipe_stats[1], st_[1]);
    atomicAdd(&g_pipe_stats[2], st_[2]);
    atomicAdd(&g_pipe_stats[7], st_[7]);
    atomicAdd(&g_pipe_stats[8], st_[8]);
    atomicAdd(&g_pipe_stats[9], st_[9]);
  }
  if (threadIdx.x == 64) {                    // first epilogue warp
    atomicAdd(&g_pipe_stats[3], st_[3]);
    atomicAdd(&g_pipe_stats[4], st_[4]);
  }
#endif
}

template <class C>
cudaError_t launch_cfg(const LogitsLaunch& L, const CUtensorMap& tk, const CUtensorMap& tq, const LogitsArgs& a) {
  static unsigned long long configured = 0;   // one bit per device ordinal
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(configured & (1ull << dev))) {
    e = cudaFuncSetAttribute(logits_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev < 64) configured |= 1ull << dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.grid, 1, 1);
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = L.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, logits_kernel<C>, tk, tq, a);
}

// The configurations this library is built with.  H=64/d=128 is the DeepSeek-V3.2
// indexer shape ("Study MLA Indexer", 关键参数); H=4/d=64 serves small models.  Epilogue
// warps (NE), pipeline depth (STAGES) and epilogue groups (EG) of each configuration can be
// overridden at build time, e.g. -DDSA_PF8_STAGES=7, for tuning; the host chooses TPA/NG.
#ifndef DSA_PB16_NE
#define DSA_PB16_NE 8
#endif
#ifndef DSA_PB16_STAGES
#define DSA_PB16_STAGES 2
#endif
#ifndef DSA_PB16_EG
#define DSA_PB16_EG 1
#endif
#ifndef DSA_PF8_NE
#define DSA_PF8_NE 8
#endif
#ifndef DSA_PF8_STAGES
#define DSA_PF8_STAGES 4
#endif
#ifndef DSA_PF8_EG
#define DSA_PF8_EG 1
#endif
#ifndef DSA_D1B16_NE
#define DSA_D1B16_NE 4
#endif
#ifndef DSA_D1B16_STAGES
#define DSA_D1B16_STAGES 6
#endif
#ifndef DSA_D2F8_NE
#define DSA_D2F8_NE 8
#endif
#ifndef DSA_D2F8_STAGES
#define DSA_D2F8_STAGES 8
#endif
#ifndef DSA_D2F8_EG
#define DSA_D2F8_EG 1
#endif
//                                  H   D   FP8   TPA NG NE               STAGES               EG
using CfgPrefillBf16   = Cfg<64, 128, false, 4, 2, DSA_PB16_NE,  DSA_PB16_STAGES,  DSA_PB16_EG, true>;
using CfgPrefillFp8    = Cfg<64, 128, true,  4, 2, DSA_PF8_NE,   DSA_PF8_STAGES,   DSA_PF8_EG, true>;
using CfgDecode1Bf16   = Cfg<64, 128, false, 1, 1, DSA_D1B16_NE, DSA_D1B16_STAGES>;
using CfgDecode2Bf16   = Cfg<64, 128, false, 2, 1, 8, 5>;
using CfgDecode4Bf16   = Cfg<64, 128, false, 4, 1, 8, 4>;
using CfgDecode1Fp8    = Cfg<64, 128, true,  1, 1, 4, 10>;
using CfgDecode2Fp8    = Cfg<64, 128, true,  2, 1, DSA_D2F8_NE,  DSA_D2F8_STAGES,  DSA_D2F8_EG>;
using CfgDecode4Fp8    = Cfg<64, 128, true,  4, 1, 8, 10>;
using CfgPrefillSmallH = Cfg<4,  64,  false, 64, 1, 4, 4>;

template <class... Cs>
constexpr bool all_fit() { return ((Cs::SMEM_BYTES <= 232448) && ...); }
static_assert(all_fit<CfgPrefillBf16, CfgPrefillFp8, CfgDecode1Bf16, CfgDecode2Bf16, CfgDecode4Bf16, CfgDecode1Fp8,
                      CfgDecode2Fp8, CfgDecode4Fp8, CfgPrefillSmallH>(),
              "shared memory of a configuration exceeds 227 KB");

}  // namespace

#ifdef DSA_PIPE_STATS
extern "C" __attribute__((visibility("default"))) int dsa_debug_pipe_stats(unsigned long long* out, int reset) {
  if (cudaMemcpyFromSymbol(out, g_pipe_stats, sizeof(g_pipe_stats)) != cudaSuccess) return 1;
  if (reset) {
    unsigned long long z[12] = {0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0};
    if (cudaMemcpyToSymbol(g_pipe_stats, z, sizeof(z)) != cudaSuccess) return 1;
  }
  return 0;
}
#endif

bool logits_config_supported(int H, int D, bool fp8, int tpa, int ng, bool prefill) {
  if (H == 64 && D == 128) {
    if (prefill) return tpa == 4 && ng == 2;
    if (ng == 1 && (tpa == 1 || tpa == 2 || tpa == 4)) return true;
  }
  if (H == 4 && D == 64 && !fp8 && tpa == 64 && ng == 1) return true;
  return false;
}

cudaError_t launch_logits(const LogitsLaunch& L, const CUtensorMap& tk, const CUtensorMap& tq,
                          const LogitsArgs& a) {
  if (L.grid <= 0) return cudaSuccess;
  if (L.H == 64 && L.D == 128) {
    if (L.prefill) {
      if (L.tpa != 4 || L.ng != 2) return cudaErrorInvalidValue;
      return L.fp8 ? launch_cfg<CfgPrefillFp8>(L, tk, tq, a) : launch_cfg<CfgPrefillBf16>(L, tk, tq, a);
    }
    if (L.ng == 1) {
      switch (L.tpa) {
        case 1: return L.fp8 ? launch_cfg<CfgDecode1Fp8>(L, tk, tq, a) : launch_cfg<CfgDecode1Bf16>(L, tk, tq, a);
        case 2: return L.fp8 ? launch_cfg<CfgDecode2Fp8>(L, tk, tq, a) : launch_cfg<CfgDecode2Bf16>(L, tk, tq, a);
        case 4: return L.fp8 ? launch_cfg<CfgDecode4Fp8>(L, tk, tq, a) : launch_cfg<CfgDecode4Bf16>(L, tk, tq, a);
        default: break;
      }
    }
  }
  if (L.H == 4 && L.D == 64 && !L.fp8 && L.tpa == 64 && L.ng == 1)
    return launch_cfg<CfgPrefillSmallH>(L, tk, tq, a);
  return cudaErrorInvalidValue;
}

bool logits_bins_rows(int H, int D, bool fp8, int tpa, int ng, bool prefill) {
  if (H != 64 || D != 128 || prefill || ng != 1) return false;
  switch (tpa) {
    case 1: return fp8 ? CfgDecode1Fp8::HIST : CfgDecode1Bf16::HIST;
    case 2: return fp8 ? CfgDecode2Fp8::HIST : CfgDecode2Bf16::HIST;
    case 4: return fp8 ? CfgDecode4Fp8::HIST : CfgDecode4Bf16::HIST;
    default: return false;
  }
}

int logits_queries_per_item(int H, int D, bool prefill, int max_q_len) {
  (void)D;
  if (H == 4) return 64;
  if (prefill) return 8;
  return max_q_len <= 1 ? 1 : max_q_len <= 2 ? 2 : 4;
}

}  // namespace dsa
