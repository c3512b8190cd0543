// select.cu -- Top-K block selection of the sparse branch.
//
// "视频扩散模型中的稀疏注意力机制解析 (ijyty.com)" 1.2: partition tokens into
// blocks, take each block's mean vector, score the query side against every
// key-block mean, keep the Top-K blocks.  Readings: the query side is pooled
// per query block too (all rows of a block share one kept set); means cover
// valid rows only; scores are unscaled dot products; ties keep the lower
// block index.
//
// Precision: block sums of bf16 values are formed in float64 (exact for bf16
// inputs in any realistic range) and divided by the row count; the kept set
// is the one float64 dot products of these means decide.  The scores are
// formed on the tensor cores from a two-term bf16 split of each mean with a
// certified error bound, and only the blocks the bound leaves undecided are
// scored again in float64 (select_rows_kernel).
//
// Kernels: pool (HBM-bound: reads Q and K once; writes the float64 means,
// their bf16 hi/lo split and squared norms), score (tcgen05: S = Qbar Kbar^T
// per head, 128 query blocks x 128 key blocks per accumulator, written to the
// workspace in float32), select_rows (per 16 query blocks of a head: the
// k-th largest score, the float64 recheck, the ascending kept lists and the
// union of each pair of query blocks' lists for the attention kernel),
// pair_union (the same union for caller-supplied lists).
#include "common.cuh"
#include "internal.h"

namespace salad {
namespace {

constexpr int kBlock = 64;

// ------------------------------------------------------------------ pool --
// CTA (i, bh, z): the mean of block i of head bh of Q (z = 0) or K (z = 1),
// summed in float64 over the valid rows and written in float64 [bh][i][c];
// its two-term bf16 split for the score MMAs, hi = bf16(f), lo = bf16(f - hi)
// with f the float32 rounding of the mean (hi and lo [bh][i][c], row-major);
// and its squared norm (float64 sum, stored as float32).
template <int D>
__global__ void __launch_bounds__(128) pool_kernel(const uint4* __restrict__ q,
                                                   const uint4* __restrict__ k, int N, int nb,
                                                   double* __restrict__ qbar,
                                                   double* __restrict__ kbar,
                                                   __nv_bfloat16* __restrict__ qhi,
                                                   __nv_bfloat16* __restrict__ qlo,
                                                   __nv_bfloat16* __restrict__ khi,
                                                   __nv_bfloat16* __restrict__ klo,
                                                   float* __restrict__ qn2,
                                                   float* __restrict__ kn2) {
  constexpr int CPR = D / 8;     // 16-byte chunks per row
  constexpr int RPI = 128 / CPR; // rows per iteration
  __shared__ double red[RPI][D];
  __shared__ double nred[4];
  const int i = blockIdx.x;
  const long long bh = blockIdx.y;
  const bool is_k = blockIdx.z != 0;
  const uint4* src = is_k ? k : q;
  double* dst = is_k ? kbar : qbar;
  __nv_bfloat16* hi = is_k ? khi : qhi;
  __nv_bfloat16* lo = is_k ? klo : qlo;
  float* n2 = is_k ? kn2 : qn2;
  const int row0 = i * kBlock;
  const int rows = min(kBlock, N - row0);
  const int chunk = threadIdx.x % CPR;
  const int rsub = threadIdx.x / CPR;
  double acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0;
  const uint4* base = src + (bh * N + row0) * CPR + chunk;
  auto add = [&](const uint4& v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack_bf16x2(w[e]);
      acc[2 * e] += static_cast<double>(f.x);
      acc[2 * e + 1] += static_cast<double>(f.y);
    }
  };
  if (rows == kBlock) {
    // A full block: every load of the thread in flight before the first add.
    constexpr int kIt = kBlock / RPI;
    uint4 v[kIt];
#pragma unroll
    for (int t = 0; t < kIt; ++t) v[t] = __ldcs(base + static_cast<long long>(rsub + t * RPI) * CPR);
#pragma unroll
    for (int t = 0; t < kIt; ++t) add(v[t]);
  } else {
    for (int r = rsub; r < rows; r += RPI) add(__ldcs(base + static_cast<long long>(r) * CPR));
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[rsub][chunk * 8 + e] = acc[e];
  __syncthreads();
  double part = 0.0;
  for (int c = threadIdx.x; c < D; c += 128) {
    double s = 0.0;
#pragma unroll
    for (int r = 0; r < RPI; ++r) s += red[r][c];
    const double m = s / static_cast<double>(rows);
    const long long at = (bh * nb + i) * D + c;
    dst[at] = m;
    const float f = static_cast<float>(m);
    const __nv_bfloat16 h = __float2bfloat16_rn(f);
    hi[at] = h;
    lo[at] = __float2bfloat16_rn(f - __bfloat162float(h));   // f - h is exact in float32
    part = fma(m, m, part);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if ((threadIdx.x & 31) == 0) nred[threadIdx.x >> 5] = part;
  __syncthreads();
  if (threadIdx.x == 0) n2[bh * nb + i] = static_cast<float>((nred[0] + nred[1]) + (nred[2] + nred[3]));
}

// ----------------------------------------------------------------- score --
// S[bh][i][j] = Qbar_i . Kbar_j for 128 query blocks (one CTA, M = 128) and
// its share of the key blocks, 64 at a time (N = 64; four chunks of key
// means in flight, accumulators in eight 64-column TMEM buffers), as three
// bf16 products of the split means:
//   S~ = qhi khi + qhi klo + qlo khi   (float32 accumulation).
// The error bound (used by select_rows_kernel), with u = 2^-8 the unit
// roundoff of bf16 (8-bit significand): f = fl32(m) is within 2^-24 |m| of
// m; hi = bf16(f) within u |f| of f; r = f - hi is exact and lo = bf16(r)
// within u |r| <= u^2 |f| of r.  So a mean is hi + lo + e with |e| <=
// 1.004 2^-16 |m|, and the dropped qlo klo and the e terms give at most
// 3.1 2^-16 |q_c||k_c| per channel.  The 3d products are exact in float32
// (8-bit by 8-bit significands) and their float32 sum, in any order and
// rounding to nearest or toward zero, is off by at most 3d 2^-23 times the
// sum of their moduli (<= 1.016 sum_c |q_c||k_c|).  With Cauchy-Schwarz:
//   |S~ - S| <= (3.1 2^-16 + 3.09 d 2^-23) |qbar_i| |kbar_j|
// plus an absolute term for values below float32's normal range.  (Reading:
// the tensor core's float32 accumulation is taken to be no worse than
// float32 additions; bf16 products are exact.)
//
// Warp roles (192 threads): warp 0 lane 0 issues the TMA loads and the MMAs;
// warp 1 holds the TMEM allocation; warps 2..5 read the accumulators (TMEM
// lane quarter w % 4) and write the scores.
template <int D>
struct SC {
  static constexpr int kN = 64;                     // key blocks per chunk (MMA N)
  static constexpr int kStages = 4;                 // key-mean chunks in flight
  static constexpr int kBufs = 512 / kN;            // TMEM accumulator buffers
  static constexpr int kSlabA = 128 * 128;          // 128 rows of one 64-channel slab
  static constexpr int kSlabB = kN * 128;           // kN rows of one 64-channel slab
  static constexpr int kA = (D / 64) * kSlabA;      // one operand (hi or lo) of 128 rows
  static constexpr int kB = (D / 64) * kSlabB;      // one operand of kN key rows
  static constexpr int kSmemUsed = 1024 + 2 * kA + kStages * 2 * kB + 512;   // A hi/lo, B hi/lo stages
  // Over half of the SM's shared memory, so one CTA (and its 512 TMEM
  // columns) occupies each SM.
  static constexpr int kSmem = kSmemUsed > 120 * 1024 ? kSmemUsed : 120 * 1024;
};

template <int D>
__global__ void __launch_bounds__(192, 1) score_kernel(const __grid_constant__ CUtensorMap mqh,
                                                       const __grid_constant__ CUtensorMap mql,
                                                       const __grid_constant__ CUtensorMap mkh,
                                                       const __grid_constant__ CUtensorMap mkl,
                                                       int nb, int nbs, int splits,
                                                       float* __restrict__ S, unsigned* err,
                                                       unsigned long long wait_ns) {
  using C = SC<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* a_hi = sm;
  unsigned char* a_lo = a_hi + C::kA;
  unsigned char* b_st = a_lo + C::kA;                    // [kStages][hi, lo]
  uint64_t* bars = reinterpret_cast<uint64_t*>(b_st + C::kStages * 2 * C::kB);
  // bars: a_full, b_full[kStages], b_empty[kStages], acc_full[kBufs],
  // acc_empty[kBufs], drain
  constexpr int NS = C::kStages, NB = C::kBufs;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 + 2 * NS + 2 * NB);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  static_assert((2 + 2 * NS + 2 * NB) * 8 + 8 <= 512, "barrier region");
  const uint32_t a_full = smem_u32(bars);
  auto b_full = [&](int s) { return smem_u32(bars + 1 + s); };
  auto b_empty = [&](int s) { return smem_u32(bars + 1 + NS + s); };
  auto acc_full = [&](int b) { return smem_u32(bars + 1 + 2 * NS + b); };
  auto acc_empty = [&](int b) { return smem_u32(bars + 1 + 2 * NS + NB + b); };
  const uint32_t drain = smem_u32(bars + 1 + 2 * NS + 2 * NB);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int i0 = blockIdx.x * 128;
  const int bh = blockIdx.z;
  // This CTA's key chunks: [cbeg, cbeg + nch) of the row's kN-column chunks
  // (the chunks are split over gridDim.y = splits CTAs).
  const int nchunks = (nb + C::kN - 1) / C::kN;
  const int cbeg = static_cast<int>(static_cast<long long>(nchunks) * blockIdx.y / splits);
  const int nch = static_cast<int>(static_cast<long long>(nchunks) * (blockIdx.y + 1) / splits) - cbeg;

  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(b_full(s), 1);
      mbar_init(b_empty(s), 1);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(acc_full(b), 1);
      mbar_init(acc_empty(b), 4);   // the four epilogue warps
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&mqh);
    tma_prefetch_map(&mql);
    tma_prefetch_map(&mkh);
    tma_prefetch_map(&mkl);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      int loaded = 0, consumed = 0;   // chunks whose K means were requested / have landed
      auto load_b = [&](int c) {
        const int s = c % NS;
        unsigned char* bh_ = b_st + s * 2 * C::kB;
        mbar_arrive_expect_tx(b_full(s), 2 * C::kB);
#pragma unroll
        for (int hh = 0; hh < D / 64; ++hh) {
          tma_load_3d(smem_u32(bh_ + hh * C::kSlabB), &mkh, b_full(s), hh * 64, (cbeg + c) * C::kN,
                      bh);
          tma_load_3d(smem_u32(bh_ + C::kB + hh * C::kSlabB), &mkl, b_full(s), hh * 64,
                      (cbeg + c) * C::kN, bh);
        }
        loaded = c + 1;
      };
      mbar_arrive_expect_tx(a_full, 2 * C::kA);
#pragma unroll
      for (int hh = 0; hh < D / 64; ++hh) {
        tma_load_3d(smem_u32(a_hi + hh * C::kSlabA), &mqh, a_full, hh * 64, i0, bh);
        tma_load_3d(smem_u32(a_lo + hh * C::kSlabA), &mql, a_full, hh * 64, i0, bh);
      }
      for (int c = 0; c < NS && c < nch; ++c) load_b(c);
      constexpr uint32_t idesc = idesc_bf16(128, C::kN, false, false);
      ok = mbar_wait(a_full, 0, wait_ns, abort_flag);
      const uint64_t dah = sdesc_sw128(smem_u32(a_hi), 16, 1024);
      const uint64_t dal = sdesc_sw128(smem_u32(a_lo), 16, 1024);
      for (int c = 0; c < nch && ok; ++c) {
        const int s = c % NS, buf = c % NB;
        if (!mbar_wait(b_full(s), (c / NS) & 1, wait_ns, abort_flag)) { ok = false; break; }
        consumed = c + 1;
        if (c >= NB && !mbar_wait(acc_empty(buf), ((c - NB) / NB) & 1, wait_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const unsigned char* bs = b_st + s * 2 * C::kB;
        const uint64_t dbh = sdesc_sw128(smem_u32(bs), 16, 1024);
        const uint64_t dbl = sdesc_sw128(smem_u32(bs + C::kB), 16, 1024);
        const uint32_t acc = tmem + C::kN * buf;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t oa = static_cast<uint64_t>(((ks / 4) * C::kSlabA + (ks % 4) * 32) >> 4);
          const uint64_t ob = static_cast<uint64_t>(((ks / 4) * C::kSlabB + (ks % 4) * 32) >> 4);
          mma_ss(acc, dah + oa, dbh + ob, idesc, ks > 0 ? 1u : 0u);
          mma_ss(acc, dah + oa, dbl + ob, idesc, 1u);
          mma_ss(acc, dal + oa, dbh + ob, idesc, 1u);
        }
        mma_commit(b_empty(s));
        mma_commit(acc_full(buf));
        // The previous chunk's stage is free once its MMAs have read it
        // (they run ahead of the ones just issued): refill it with chunk
        // c - 1 + NS.
        if (c >= 1 && c - 1 + NS < nch) {
          if (!mbar_wait(b_empty((c - 1) % NS), ((c - 1) / NS) & 1, wait_ns, abort_flag)) {
            ok = false;
            break;
          }
          load_b(c - 1 + NS);
        }
      }
      if (!ok) raise_timeout(err, abort_flag);
      // Leave nothing in flight: requested loads landed, issued MMAs done.
      for (int c = consumed; c < loaded; ++c)
        if (!mbar_wait(b_full(c % NS), (c / NS) & 1, wait_ns, nullptr)) atomicOr(err, kErrTimeout);
      mma_commit(drain);
      if (!mbar_wait(drain, 0, wait_ns, nullptr)) atomicOr(err, kErrTimeout);
    }
  } else if (warp >= 2) {
    const int quarter = warp % 4;
    const int r = quarter * 32 + lane;                 // query block i0 + r
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const bool row_ok = i0 + r < nb;
    float* srow = S + (static_cast<long long>(bh) * nb + (row_ok ? i0 + r : 0)) * nbs;
    bool ok = true;
    for (int c = 0; c < nch && ok; ++c) {
      const int buf = c % NB;
      if (!__all_sync(0xffffffffu, mbar_wait(acc_full(buf), (c / NB) & 1, wait_ns, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < C::kN; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(lane_base + C::kN * buf + c0, v);
        if (row_ok) {
          float4* dst = reinterpret_cast<float4*>(srow + (cbeg + c) * C::kN + c0);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                 __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty(buf));
    }
    if (!ok) raise_timeout(err, abort_flag);
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------ selection --
// One CTA takes RB query blocks of one head: per block (one warp) the kept
// set from the float32 scores S~ and the bound E above, then the union of
// each pair of query blocks' kept sets for the attention kernel.
//
// Exact float64 decision.  With T the k-th largest score of the row in S~,
// bracketed as blo <= T <= bhi, the float64 k-th largest lies in
// [blo - E, bhi + E]: a block scoring above bhi + 2E is among the float64
// Top-K for certain, one below blo - 2E is not; only the blocks in between
// (the candidates, typically none or a few) are scored again in float64
// (ascending c, the same sum as the float64 definition) and ranked by
// (score desc, index asc).  The kept set is therefore the float64 selection.
//
// Per row: the row's scores in registers (column lane + 32 u); a bisection
// on the value brackets T until the bracket is narrower than the bound or
// holds at most 8 scores -- those are then gathered one per lane and T is
// taken exactly; then the band, the float64 recheck (candidates ranked
// directly, or by a radix select over float64 keys when there are many), the
// kept bitmap and the ascending index list.  Per pair of query blocks (one
// warp): the union of the two kept bitmaps as an ascending list of entries
// j | mask << 16.
// Threads per CTA: 256, or 192 for many scores per lane (their registers
// then allow two CTAs, 12 warps, per SM).
template <int VPL> constexpr int sel_threads() { return VPL <= 16 ? 256 : (VPL <= 64 ? 192 : 256); }
template <int VPL> constexpr int sel_min_blocks() { return VPL <= 16 ? 3 : (VPL <= 64 ? 2 : 1); }
constexpr int kCandMax = 64;              // float64 candidates buffered per warp

__device__ __forceinline__ unsigned long long dkey(double x) {
  x = x + 0.0;
  const unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(x));
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// float64 score of (query block row qrow, key block j): ascending-c fma chain.
template <int D>
__device__ __forceinline__ double score64(const double* __restrict__ qrow,
                                          const double* __restrict__ kb, int j) {
  const double* kr = kb + static_cast<long long>(j) * D;
  double acc = 0.0;
#pragma unroll 8
  for (int c = 0; c < D; ++c) acc = fma(__ldg(qrow + c), __ldg(kr + c), acc);
  return acc;
}

// Radix select over 64-bit keys of the items j in [0, n) for which key_of
// reports ok: finds, 8 bits per pass from the top, the digits of the
// `want`-th largest key; stops early once every key sharing the prefix is
// wanted.  On return `want` is the number still wanted among keys equal to
// the (masked) prefix.  Warp-collective; hist: 256 words of this warp.
template <typename KeyOf>
__device__ __forceinline__ void radix_select64(int n, int& want, unsigned long long& prefix,
                                               unsigned long long& pmask, unsigned* hist, int lane,
                                               KeyOf key_of) {
  prefix = 0;
  pmask = 0;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int j = lane; j < n; j += 32) {
      bool ok;
      const unsigned long long key = key_of(j, ok);
      if (ok && (key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncwarp();
    unsigned mine = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) mine += hist[lane * 8 + e];
    unsigned suffix = mine;  // inclusive suffix sum: bins >= 8 lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned t = __shfl_down_sync(0xffffffffu, suffix, o);
      if (lane + o < 32) suffix += t;
    }
    const unsigned above_lane = suffix - mine;
    const bool here = above_lane < static_cast<unsigned>(want) && suffix >= static_cast<unsigned>(want);
    const int owner = __ffs(__ballot_sync(0xffffffffu, here)) - 1;
    int digit = 0;
    unsigned above = 0;
    if (lane == owner) {
      unsigned acc = above_lane;
      for (int e = 7; e >= 0; --e) {
        const unsigned h = hist[lane * 8 + e];
        if (acc + h >= static_cast<unsigned>(want)) {
          digit = lane * 8 + e;
          above = acc;
          break;
        }
        acc += h;
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, owner);
    above = __shfl_sync(0xffffffffu, above, owner);
    want -= static_cast<int>(above);
    prefix |= static_cast<unsigned long long>(digit) << shift;
    pmask |= 0xFFull << shift;
    const bool settled = hist[digit] == static_cast<unsigned>(want);
    __syncwarp();
    if (settled) return;
  }
}


// VPL: scores of a row each lane keeps in registers (column j = lane + 32 u).
template <int D, int RB, int VPL>
__global__ void __launch_bounds__(sel_threads<VPL>(), sel_min_blocks<VPL>()) select_rows_kernel(
    const float* __restrict__ S, int nbs, const float* __restrict__ qn2,
    const float* __restrict__ kn2, const double* __restrict__ qbar64,
    const double* __restrict__ kbar64, int nb, int topk, int32_t* __restrict__ idx,
    int32_t* __restrict__ lists, int32_t* __restrict__ counts) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int nw = (nb + 31) / 32;
  unsigned* scratch = reinterpret_cast<unsigned*>(smem_raw);              // [warps][256 + 3 kCandMax]
  constexpr int kSelThreads = sel_threads<VPL>(), kWarps = kSelThreads / 32;
  unsigned* bits = scratch + kWarps * (256 + kCandMax * 3);               // [RB][nw]
  float* red = reinterpret_cast<float*>(bits + RB * nw);                  // [threads]
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const long long bh = blockIdx.y;
  const int i0 = blockIdx.x * RB;
  const int rows = min(RB, nb - i0);

  // Largest key-mean norm of the head.
  float kmax2 = 0.0f;
  for (int j = tid; j < nb; j += kSelThreads) kmax2 = fmaxf(kmax2, __ldg(kn2 + bh * nb + j));
  red[tid] = kmax2;
  __syncthreads();
  if (warp == 0) {
    float m = 0.0f;
    for (int t = lane; t < kSelThreads; t += 32) m = fmaxf(m, red[t]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[0] = m;
  }
  __syncthreads();
  const double kmax = sqrtf(red[0]);

  // ---- per row (warp): the k-th largest float32 score, the band and, where
  // needed, the float64 decision; each warp's radix histogram and candidate
  // buffer.
  unsigned* hist = scratch + warp * (256 + kCandMax * 3);
  double* cs = reinterpret_cast<double*>(hist + 256);
  int* cj = reinterpret_cast<int*>(cs + kCandMax);
  for (int r = warp; r < RB; r += kWarps) {
    unsigned* kept = bits + r * nw;
    for (int w = lane; w < nw; w += 32) kept[w] = 0u;
    __syncwarp();
    if (r >= rows) continue;
    // The row's scores in registers: column j = lane + 32 u (-inf past nb).
    const float* srow = S + (bh * nb + i0 + r) * static_cast<long long>(nbs);
    float vals[VPL];
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      const int j = lane + 32 * u;
      vals[u] = j < nb ? __ldg(srow + j) : -INFINITY;
    }
    // Bracket the k-th largest float32 score T: cnt(>= lo) >= topk > cnt(>= hi),
    // so lo <= T < hi, by bisection on the value until the bracket is
    // narrower than the bound E allows.
    const double qnr = sqrtf(__ldg(qn2 + bh * nb + i0 + r));
    const bool wide = !(qnr < 1e18 && kmax < 1e18);
    const double E = (3.1 * 1.52587890625e-5 + 3.09 * D * 1.1920928955078125e-7) * 1.05 * qnr * kmax +
                     D * 1.0e-36 * (1.0 + qnr + kmax);
    auto count_ge = [&](float t) -> int {
      unsigned cnt = 0;
#pragma unroll
      for (int u = 0; u < VPL; ++u) cnt += vals[u] >= t ? 1u : 0u;
      return static_cast<int>(__reduce_add_sync(0xffffffffu, cnt));
    };
    float mn = INFINITY, mx = -INFINITY;
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      if (lane + 32 * u < nb) mn = fminf(mn, vals[u]);
      mx = fmaxf(mx, vals[u]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    double blo = mx, bhi = mx;   // T = mx when at least topk scores tie at the maximum
    int c_hi = 0;
    if (!wide && (c_hi = count_ge(mx)) < topk) {
      float lo = mn, hi = mx;
      int c_lo = nb;               // cnt(>= lo) >= topk > cnt(>= hi) = c_hi
      // The stopping width in float32 (any bracket is sound: it only sets how
      // many candidates the band holds).
      const float half_e = static_cast<float>(0.5 * E);
      for (int it = 0; it < 64 && hi - lo > half_e && c_lo - c_hi > 8; ++it) {
        const float mid = lo + 0.5f * (hi - lo);
        if (!(mid > lo && mid < hi)) break;   // adjacent floats
        const int cm = count_ge(mid);
        if (cm >= topk) { lo = mid; c_lo = cm; } else { hi = mid; c_hi = cm; }
      }
      blo = lo;
      bhi = hi;
      if (c_lo - c_hi <= 8) {
        // At most 8 scores lie in [lo, hi): gather them, one per lane, and
        // take T exactly: the largest x with cnt(>= x) >= topk - c_hi among
        // them (every score >= hi is counted in c_hi).
        float* gbuf = reinterpret_cast<float*>(hist);
        int ng = 0;
#pragma unroll
        for (int u = 0; u < VPL; ++u) {
          const bool g = vals[u] >= lo && vals[u] < hi;
          const unsigned b = __ballot_sync(0xffffffffu, g);
          if (g) gbuf[ng + __popc(b & ((1u << lane) - 1u))] = vals[u];
          ng += __popc(b);
        }
        __syncwarp();
        const float x = lane < ng ? gbuf[lane] : -INFINITY;
        int cge = 0;
        for (int u = 0; u < ng; ++u) cge += __shfl_sync(0xffffffffu, x, u) >= x ? 1 : 0;
        float t = (lane < ng && cge >= topk - c_hi) ? x : -INFINITY;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, o));
        __syncwarp();
        blo = t;
        bhi = t;
      }
    }
    // The float64 k-th largest lies within [blo - E, bhi + E]: above
    // bhi + 2E a block is kept for certain, below blo - 2E dropped.
    const double lo = wide ? -INFINITY : blo - 2.0 * E, hi = wide ? INFINITY : bhi + 2.0 * E;
    // The same tests in float32 against the band's ends rounded outward
    // (hi up, lo down): a score above hi_f is above hi, and every score in
    // the band is a candidate (a few just outside it may be too).
    const float hi_f = wide ? INFINITY : __double2float_ru(hi);
    const float lo_f = wide ? -INFINITY : __double2float_rd(lo);
    auto is_cand_v = [&](float v) { return !(v > hi_f) && v >= lo_f; };
    // Certain members (word u of the kept bitmap is the ballot over u) and
    // the candidates.
    int n_in = 0, n_cand = 0;
    unsigned cand_w[VPL];
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      const bool valid = lane + 32 * u < nb;
      const bool in = valid && vals[u] > hi_f;
      const bool cand = valid && is_cand_v(vals[u]);
      const unsigned bin = __ballot_sync(0xffffffffu, in);
      cand_w[u] = __ballot_sync(0xffffffffu, cand);
      if (lane == 0 && u < nw) kept[u] = bin;
      n_in += __popc(bin);
      n_cand += __popc(cand_w[u]);
    }
    __syncwarp();
    const int need = topk - n_in;   // 0 <= need <= n_cand
    if (need == n_cand) {
      // Every candidate is kept: no float64 needed.
      if (lane == 0) {
#pragma unroll
        for (int u = 0; u < VPL; ++u)
          if (u < nw) kept[u] |= cand_w[u];
      }
    } else if (need > 0) {
      const double* qrow = qbar64 + (bh * nb + i0 + r) * D;
      const double* kb64 = kbar64 + bh * nb * D;
      if (n_cand <= kCandMax) {
        // Buffer the candidates (ascending j) with their float64 scores and
        // keep the `need` best by (score desc, j asc).
        int nc = 0;
#pragma unroll
        for (int u = 0; u < VPL; ++u) {
          const unsigned b = cand_w[u];
          if ((b >> lane) & 1u) cj[nc + __popc(b & ((1u << lane) - 1u))] = lane + 32 * u;
          nc += __popc(b);
        }
        __syncwarp();
        for (int t = lane; t < nc; t += 32) cs[t] = score64<D>(qrow, kb64, cj[t]);
        __syncwarp();
        for (int t = lane; t < nc; t += 32) {
          // Ranked on the order-preserving keys: a total order, so exactly
          // `need` candidates are kept whatever the values.
          const unsigned long long st = dkey(cs[t]);
          int rank = 0;
          for (int u = 0; u < nc; ++u) {
            const unsigned long long su = dkey(cs[u]);
            rank += (su > st || (su == st && u < t)) ? 1 : 0;
          }
          if (rank < need) atomicOr(&kept[cj[t] / 32], 1u << (cj[t] % 32));
        }
        __syncwarp();
      } else {
        // Many candidates (near-degenerate rows, e.g. exact ties): a radix
        // select over their float64 keys, each key recomputed when read.
        auto is_cand = [&](int j) { return is_cand_v(srow[j]); };
        int want64 = need;
        unsigned long long pfx = 0, pm = 0;
        radix_select64(nb, want64, pfx, pm, hist, lane, [&](int j, bool& ok) {
          ok = is_cand(j);
          return ok ? dkey(score64<D>(qrow, kb64, j)) : 0ull;
        });
        int eq_seen = 0;
        for (int j0 = 0; j0 < nb; j0 += 32) {
          const int j = j0 + lane;
          const bool cand = j < nb && is_cand(j);
          const unsigned long long key = cand ? (dkey(score64<D>(qrow, kb64, j)) & pm) : 0ull;
          const bool gt = cand && key > pfx;
          const bool eq = cand && key == pfx;
          const unsigned eqb = __ballot_sync(0xffffffffu, eq);
          const int eq_rank = eq_seen + __popc(eqb & ((1u << lane) - 1u));
          const unsigned kb2 = __ballot_sync(0xffffffffu, gt || (eq && eq_rank < want64));
          if (lane == 0) kept[j0 / 32] |= kb2;
          eq_seen += __popc(eqb);
        }
        __syncwarp();
      }
    }
    __syncwarp();
    // The kept list, ascending.
    if (idx != nullptr) {
      int32_t* out = idx + (bh * nb + i0 + r) * static_cast<long long>(topk);
      // Lane w writes the blocks of word w after those of the words before it.
      int written = 0;
      for (int w0 = 0; w0 < nw; w0 += 32) {
        const int w = w0 + lane;
        unsigned word = w < nw ? kept[w] : 0u;
        const int cnt = __popc(word);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        int pos = written + incl - cnt;
        while (word) {
          const int bit = __ffs(word) - 1;
          word &= word - 1;
          if (pos < topk) out[pos] = 32 * w + bit;
          ++pos;
        }
        written += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
  }
  if (lists == nullptr) return;
  __syncthreads();

  // ---- phase 3: union of the kept sets of each pair (2p, 2p+1) of the chunk
  const int npairs_all = (nb + 1) / 2;
  for (int pr = warp; pr < (rows + 1) / 2; pr += kWarps) {
    const int p = i0 / 2 + pr;
    const unsigned* A = bits + (2 * pr) * nw;
    const bool has_b = 2 * pr + 1 < rows;
    const unsigned* Bm = bits + (2 * pr + 1) * nw;
    const long long item = bh * npairs_all + p;
    int32_t* out = lists + item * (2 * topk);
    int base = 0;
    for (int w0 = 0; w0 < nw; w0 += 32) {
      const int w = w0 + lane;
      const unsigned a = w < nw ? A[w] : 0u;
      const unsigned b = (w < nw && has_b) ? Bm[w] : 0u;
      unsigned u = a | b;
      const int c = __popc(u);
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      int pos = base + incl - c;
      while (u) {
        const int bit = __ffs(u) - 1;
        u &= u - 1;
        const int mask = static_cast<int>((a >> bit) & 1u) | (static_cast<int>((b >> bit) & 1u) << 1);
        if (pos < 2 * topk) out[pos] = (w * 32 + bit) | (mask << 16);
        ++pos;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) counts[item] = min(base, 2 * topk);
  }
}

// ------------------------------------------------------------ pair union --
// One warp per (bh, p).  Kept lists of query blocks 2p and 2p+1 -> one
// ascending list of entries j | mask << 16.
__global__ void pair_union_kernel(const int32_t* __restrict__ idx, int BH, int nb, int topk,
                                  int32_t* __restrict__ lists, int32_t* __restrict__ counts) {
  extern __shared__ unsigned bits_raw[];
  const int warps = blockDim.x / 32;
  const int wid = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nwords = (nb + 31) / 32;
  unsigned* A = bits_raw + wid * 2 * nwords;
  unsigned* Bm = A + nwords;
  const int npairs = (nb + 1) / 2;
  const long long item = static_cast<long long>(blockIdx.x) * warps + wid;
  if (item >= static_cast<long long>(BH) * npairs) return;
  const long long bh = item / npairs;
  const int p = static_cast<int>(item % npairs);
  for (int w = lane; w < nwords; w += 32) { A[w] = 0; Bm[w] = 0; }
  __syncwarp();
  const int32_t* ia = idx + (bh * nb + 2 * p) * topk;
  const bool has_b = 2 * p + 1 < nb;
  // Entries outside [0, nb) (possible only in caller-supplied lists) are dropped.
  for (int t = lane; t < topk; t += 32) {
    const int j = ia[t];
    if (j >= 0 && j < nb) atomicOr(&A[j >> 5], 1u << (j & 31));
    if (has_b) {
      const int j2 = ia[topk + t];
      if (j2 >= 0 && j2 < nb) atomicOr(&Bm[j2 >> 5], 1u << (j2 & 31));
    }
  }
  __syncwarp();
  int32_t* out = lists + item * (2 * topk);
  int base = 0;
  for (int w0 = 0; w0 < nwords; w0 += 32) {
    const int w = w0 + lane;
    const unsigned a = w < nwords ? A[w] : 0u;
    const unsigned b = w < nwords ? Bm[w] : 0u;
    unsigned u = a | b;
    const int c = __popc(u);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int pos = base + incl - c;
    while (u) {
      const int bit = __ffs(u) - 1;
      u &= u - 1;
      const int mask = static_cast<int>((a >> bit) & 1u) | (static_cast<int>((b >> bit) & 1u) << 1);
      if (pos < 2 * topk) out[pos] = (w * 32 + bit) | (mask << 16);
      ++pos;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) counts[item] = min(base, 2 * topk);
}


size_t sel_smem_bytes(int threads, int RB, int nb) {
  const size_t nw = (static_cast<size_t>(nb) + 31) / 32;
  return static_cast<size_t>(threads / 32) * (256 + kCandMax * 3) * 4 + RB * nw * 4 + threads * 4;
}

struct SelectLayout {
  size_t qbar, kbar, qhi, qlo, khi, klo, qn2, kn2, S, total;
  int nbs;   // row length of the score matrix (whole 128-column chunks)
};
SelectLayout select_layout(int B, int H, int N, int d, int block) {
  const size_t nb = (static_cast<size_t>(N) + block - 1) / block;
  const size_t BH = static_cast<size_t>(B) * H;
  SelectLayout L;
  L.nbs = static_cast<int>((nb + 127) / 128 * 128);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  L.qbar = take(BH * nb * d * sizeof(double));
  L.kbar = take(BH * nb * d * sizeof(double));
  L.qhi = take(BH * nb * d * 2);
  L.qlo = take(BH * nb * d * 2);
  L.khi = take(BH * nb * d * 2);
  L.klo = take(BH * nb * d * 2);
  L.qn2 = take(BH * nb * sizeof(float));
  L.kn2 = take(BH * nb * sizeof(float));
  L.S = take(BH * nb * L.nbs * sizeof(float));
  L.total = off;
  return L;
}

template <int D, int RB, int VPL>
cudaError_t launch_select_rows(const Ctx& c, const float* S, int nbs, const float* qn2,
                               const float* kn2, const double* q64, const double* k64, int BH,
                               int nb, int topk, int32_t* idx, int32_t* lists, int32_t* counts) {
  const size_t smem = sel_smem_bytes(sel_threads<VPL>(), RB, nb);
  cudaError_t e = cudaFuncSetAttribute(select_rows_kernel<D, RB, VPL>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((nb + RB - 1) / RB, BH);
  select_rows_kernel<D, RB, VPL><<<grid, sel_threads<VPL>(), smem, c.stream>>>(
      S, nbs, qn2, kn2, q64, k64, nb, topk, idx, lists, counts);
  return cudaGetLastError();
}

// The row's scores per lane kept in registers (nb <= 32 VPL); one query
// block per warp: 8 per CTA (256 threads), or 6 (192 threads, two CTAs per
// SM) for 512 < nb <= 2048.
template <int D>
cudaError_t dispatch_select(const Ctx& c, const float* S, int nbs, const float* qn2,
                            const float* kn2, const double* q64, const double* k64, int BH,
                            int nb, int topk, int32_t* idx, int32_t* lists, int32_t* counts) {
  if (nb <= 512)
    return launch_select_rows<D, 8, 16>(c, S, nbs, qn2, kn2, q64, k64, BH, nb, topk, idx, lists,
                                         counts);
  if (nb <= 2048)
    return launch_select_rows<D, 6, 64>(c, S, nbs, qn2, kn2, q64, k64, BH, nb, topk, idx, lists,
                                         counts);
  return launch_select_rows<D, 8, 128>(c, S, nbs, qn2, kn2, q64, k64, BH, nb, topk, idx, lists,
                                        counts);
}

template <int D>
cudaError_t launch_score(const Ctx& c, const SelectLayout& L, char* base, int BH, int nb) {
  CUtensorMap mqh, mql, mkh, mkl;
  if (!make_tmap_bf16_3d_rows(&mqh, base + L.qhi, BH, nb, D, 128) ||
      !make_tmap_bf16_3d_rows(&mql, base + L.qlo, BH, nb, D, 128) ||
      !make_tmap_bf16_3d_rows(&mkh, base + L.khi, BH, nb, D, SC<D>::kN) ||
      !make_tmap_bf16_3d_rows(&mkl, base + L.klo, BH, nb, D, SC<D>::kN))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(score_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       SC<D>::kSmem);
  if (e != cudaSuccess) return e;
  // Split each row tile's key chunks over CTAs while the grid is under one
  // CTA per SM.
  const int tiles = (nb + 127) / 128, nchunks = (nb + SC<D>::kN - 1) / SC<D>::kN;
  int splits = c.num_sms / (tiles * BH);
  if (splits > nchunks) splits = nchunks;
  if (splits < 1) splits = 1;
  dim3 grid(tiles, splits, BH);
  score_kernel<D><<<grid, 192, SC<D>::kSmem, c.stream>>>(
      mqh, mql, mkh, mkl, nb, L.nbs, splits, reinterpret_cast<float*>(base + L.S), c.err,
      c.wait_ns);
  return cudaGetLastError();
}

// Pools Q (z = 0) and K (z = 1), scores, then selects.
cudaError_t pool_and_select(const Ctx& c, const void* q, const void* k, int B, int H, int N, int d,
                            int topk, int32_t* idx, void* ws, int32_t* lists, int32_t* counts,
                            cudaEvent_t pooled) {
  const SelectLayout L = select_layout(B, H, N, d, kBlock);
  char* base = static_cast<char*>(ws);
  double* qbar = reinterpret_cast<double*>(base + L.qbar);
  double* kbar = reinterpret_cast<double*>(base + L.kbar);
  auto bf = [&](size_t o) { return reinterpret_cast<__nv_bfloat16*>(base + o); };
  float* qn2 = reinterpret_cast<float*>(base + L.qn2);
  float* kn2 = reinterpret_cast<float*>(base + L.kn2);
  const float* S = reinterpret_cast<const float*>(base + L.S);
  const int nb = (N + kBlock - 1) / kBlock;
  const int BH = B * H;
  dim3 pg(nb, BH, 2);
  if (d == 128)
    pool_kernel<128><<<pg, 128, 0, c.stream>>>(static_cast<const uint4*>(q),
                                                static_cast<const uint4*>(k), N, nb, qbar, kbar,
                                                bf(L.qhi), bf(L.qlo), bf(L.khi), bf(L.klo), qn2,
                                                kn2);
  else
    pool_kernel<64><<<pg, 128, 0, c.stream>>>(static_cast<const uint4*>(q),
                                               static_cast<const uint4*>(k), N, nb, qbar, kbar,
                                               bf(L.qhi), bf(L.qlo), bf(L.khi), bf(L.klo), qn2,
                                               kn2);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (pooled != nullptr && (e = cudaEventRecord(pooled, c.stream)) != cudaSuccess) return e;
  e = d == 128 ? launch_score<128>(c, L, base, BH, nb) : launch_score<64>(c, L, base, BH, nb);
  if (e != cudaSuccess) return e;
  if (d == 128)
    return dispatch_select<128>(c, S, L.nbs, qn2, kn2, qbar, kbar, BH, nb, topk, idx, lists,
                                counts);
  return dispatch_select<64>(c, S, L.nbs, qn2, kn2, qbar, kbar, BH, nb, topk, idx, lists, counts);
}

}  // namespace

size_t select_ws_bytes(int B, int H, int N, int d, int block) {
  return select_layout(B, H, N, d, block).total;
}

cudaError_t launch_select(const Ctx& c, const void* q, const void* k, int B, int H, int N, int d,
                          int topk, int32_t* idx, void* ws, int32_t* lists, int32_t* counts,
                          cudaEvent_t pooled) {
  return pool_and_select(c, q, k, B, H, N, d, topk, idx, ws, lists, counts, pooled);
}

size_t pairs_ws_bytes(int B, int H, int N, int topk) {
  const size_t nb = (static_cast<size_t>(N) + kBlock - 1) / kBlock;
  const size_t items = static_cast<size_t>(B) * H * ((nb + 1) / 2);
  return align256(items * 2 * topk * sizeof(int32_t)) + align256(items * sizeof(int32_t));
}

cudaError_t launch_pair_union(const Ctx& c, const int32_t* idx, int BH, int nb, int topk,
                              int32_t* lists, int32_t* counts) {
  const int warps = 8;
  const int nwords = (nb + 31) / 32;
  const size_t smem = static_cast<size_t>(warps) * 2 * nwords * sizeof(unsigned);
  const long long items = static_cast<long long>(BH) * ((nb + 1) / 2);
  pair_union_kernel<<<static_cast<unsigned>((items + warps - 1) / warps), warps * 32, smem,
                      c.stream>>>(idx, BH, nb, topk, lists, counts);
  return cudaGetLastError();
}

}  // namespace salad
