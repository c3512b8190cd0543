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
// formed in float32 with a certified error bound, and only the blocks the
// bound leaves undecided are scored again in float64 (select_fused_kernel).
//
// Kernels: pool (HBM-bound: reads Q and K once), select_fused (per chunk of
// query blocks of a head: float32 scores in shared memory, a radix select,
// the float64 recheck, the ascending kept lists and the union of each pair
// of query blocks' lists for the attention kernel), pair_union (the same
// union for caller-supplied lists).
#include "common.cuh"
#include "internal.h"

namespace salad {
namespace {

constexpr int kBlock = 64;

// ------------------------------------------------------------------ pool --
// CTA (i, bh, z): the mean of block i of head bh of Q (z = 0) or K (z = 1),
// summed in float64 over the valid rows and written in float64; rounded once
// to float32 for the selection's float32 pass: Q row-major [bh][i][c], K
// channel-major [bh][c][i] (row length nbs, so a chunk of channels is a run
// of contiguous rows), with the squared norm of each rounded K mean.
template <int D>
__global__ void __launch_bounds__(128) pool_kernel(const uint4* __restrict__ q,
                                                   const uint4* __restrict__ k, int N, int nb,
                                                   int nbs, double* __restrict__ qbar,
                                                   double* __restrict__ kbar,
                                                   float* __restrict__ qbar32,
                                                   float* __restrict__ kbar32t,
                                                   float* __restrict__ kn2) {
  constexpr int CPR = D / 8;     // 16-byte chunks per row
  constexpr int RPI = 128 / CPR; // rows per iteration
  __shared__ double red[RPI][D];
  __shared__ float nred[4];
  const int i = blockIdx.x;
  const long long bh = blockIdx.y;
  const bool is_k = blockIdx.z != 0;
  const uint4* src = is_k ? k : q;
  double* dst = is_k ? kbar : qbar;
  const int row0 = i * kBlock;
  const int rows = min(kBlock, N - row0);
  const int chunk = threadIdx.x % CPR;
  const int rsub = threadIdx.x / CPR;
  double acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0;
  const uint4* base = src + (bh * N + row0) * CPR + chunk;
#pragma unroll 4
  for (int r = rsub; r < rows; r += RPI) {
    const uint4 v = __ldcs(base + static_cast<long long>(r) * CPR);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack_bf16x2(w[e]);
      acc[2 * e] += static_cast<double>(f.x);
      acc[2 * e + 1] += static_cast<double>(f.y);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[rsub][chunk * 8 + e] = acc[e];
  __syncthreads();
  float part = 0.0f;
  for (int c = threadIdx.x; c < D; c += 128) {
    double s = 0.0;
#pragma unroll
    for (int r = 0; r < RPI; ++r) s += red[r][c];
    const double m = s / static_cast<double>(rows);
    dst[(bh * nb + i) * D + c] = m;
    const float m32 = static_cast<float>(m);
    if (is_k) {
      kbar32t[(bh * D + c) * static_cast<long long>(nbs) + i] = m32;
      part = fmaf(m32, m32, part);
    } else {
      qbar32[(bh * nb + i) * D + c] = m32;
    }
  }
  if (is_k) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if ((threadIdx.x & 31) == 0) nred[threadIdx.x >> 5] = part;
    __syncthreads();
    if (threadIdx.x == 0) kn2[bh * nb + i] = (nred[0] + nred[1]) + (nred[2] + nred[3]);
  }
}

// ------------------------------------------------------ fused selection --
// One CTA scores a chunk of RB query blocks of one head against all nb key
// blocks, selects the topk largest per query block, and merges the kept
// lists of the chunk's pairs of query blocks for the attention kernel.
//
// Exact float64 decision at float32 cost.  Scores are formed in float32 from
// the float32-rounded means (a sequential fma chain over c, staged through
// shared memory), so each differs from the float64 score by at most
//   E_i = (d + 8) 2^-24 * 1.05 * |qbar_i|_2 * max_j |kbar_j|_2
// (rounding of the means to float32 and of the d-term fma chain, with a 5%
// margin that also covers the float32 norms).  With T the k-th largest
// float32 score of the row, bracketed as blo <= T <= bhi, the float64 k-th
// largest lies in [blo - E, bhi + E]: a block scoring above bhi + 2E is among
// the float64 Top-K for certain, one below blo - 2E is not; only the blocks in between (the
// candidates, typically none or a few) are scored again in float64 (ascending
// c, the same sum as the float64 definition) and ranked by (score desc,
// index asc).  The kept set is therefore the float64 selection.
//
// Phases (256 threads):
//  1. scores: thread (ty, tx) accumulates RPT rows (RPT ty ..) x 4 columns
//     (4 tx ..) of a column tile; the channel-major key means stream through
//     a ring of cp.async chunks.  RPT = 8 where a 512-column tile covers the
//     row (nb <= 512): each 16-byte key load then feeds 32 fma, not 16.
//  2. one warp per row: a bisection on the value brackets the k-th largest
//     float32 score T, until the bracket is narrower than the bound or holds
//     at most 32 scores -- those are then gathered one per lane and T is
//     taken exactly; then the band, the float64 recheck (candidates ranked
//     directly, or by a radix select over float64 keys when there are many),
//     the kept bitmap and the ascending index list.
//  3. one warp per pair of query blocks: the union of the two kept bitmaps
//     as an ascending list of entries j | mask << 16.
template <int D, int RB, int RPT>
struct SelCfg {
  static constexpr int kThreads = 256;
  static constexpr int kWarps = kThreads / 32;
  static constexpr int kRPT = RPT;                 // query rows per thread
  static constexpr int kRG = RB / kRPT;            // row groups
  static constexpr int kCG = kThreads / kRG;       // 4-column groups
  static constexpr int kCT = 4 * kCG;              // columns per tile
  static constexpr int kKC = kRPT == 8 ? 4 : 8;    // channels per staged chunk
  static constexpr int kRing = 4;                  // chunks in flight (cp.async stages)
  static constexpr int kCandMax = 64;              // float64 candidates buffered per warp
  // The staging ring, reused after the scores by the float64 recheck.
  static constexpr int kStageFloats = kRing * kKC * kCT;
  static_assert(kCG >= 32 && kCG % 32 == 0, "a warp spans one row group");
  static_assert(D % kKC == 0, "chunking");
  static_assert(kStageFloats * 4 >= kWarps * (256 * 4 + kCandMax * 12), "recheck scratch");
};

template <int D, int RB, int RPT>
size_t sel_smem_bytes(int nb) {
  using C = SelCfg<D, RB, RPT>;
  const size_t nbp = (static_cast<size_t>(nb) + 3) & ~static_cast<size_t>(3);
  const size_t nw = (static_cast<size_t>(nb) + 31) / 32;
  return static_cast<size_t>(D) * RB * 4            // qs [D][RB]
         + static_cast<size_t>(C::kStageFloats) * 4 // ks [ring][KC][CT], later the recheck scratch
         + RB * nbp * 4                             // scores [RB][nbp]
         + RB * nw * 4                              // kept bitmaps [RB][nw]
         + (C::kThreads + RB + 8) * 4;              // norm reduction, row norms
}

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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// VPL: scores of a row each lane keeps in registers (column j = lane + 32 u).
template <int D, int RB, int VPL, int RPT>
__global__ void __launch_bounds__(256, VPL <= 16 ? 3 : 1) select_fused_kernel(
    const float* __restrict__ qbar32, const float* __restrict__ kbar32t,
    const float* __restrict__ kn2, const double* __restrict__ qbar64,
    const double* __restrict__ kbar64, int nb, int nbs, int topk, int32_t* __restrict__ idx,
    int32_t* __restrict__ lists, int32_t* __restrict__ counts) {
  using C = SelCfg<D, RB, RPT>;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int nbp = (nb + 3) & ~3;
  const int nw = (nb + 31) / 32;
  float* qs = reinterpret_cast<float*>(smem_raw);                        // [D][RB]
  float* ks = qs + D * RB;                                                // [ring][KC][CT]
  float* sc = ks + C::kStageFloats;                                       // [RB][nbp]
  unsigned* bits = reinterpret_cast<unsigned*>(sc + RB * nbp);            // [RB][nw]
  float* red = reinterpret_cast<float*>(bits + RB * nw);                  // [threads]
  float* qn = red + C::kThreads;                                          // [RB] row norms
  float* kmax_s = qn + RB;                                                // [1]

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const long long bh = blockIdx.y;
  const int i0 = blockIdx.x * RB;
  const int rows = min(RB, nb - i0);
  const float* qb = qbar32 + (bh * nb + i0) * D;
  const float* kt = kbar32t + bh * D * static_cast<long long>(nbs);

  // ---- phase 1: float32 scores.  Chunk ch = (column tile, KC channels): KC
  // rows of CT key means from the channel-major copy, streamed by cp.async
  // through a ring of kRing chunks, kRing - 1 in flight ahead of the one
  // being multiplied.
  const int ty = tid / C::kCG, tx = tid % C::kCG;
  const int ntile = (nb + C::kCT - 1) / C::kCT;
  constexpr int kChunks = D / C::kKC;
  constexpr int kCopies = C::kKC * C::kCT / 4;   // 16-byte copies per chunk
  const int nch = ntile * kChunks;
  auto issue = [&](int ch) {
    float* dst = ks + (ch % C::kRing) * C::kKC * C::kCT;
    const int j0 = (ch / kChunks) * C::kCT, c0 = (ch % kChunks) * C::kKC;
    for (int e = tid; e < kCopies; e += C::kThreads) {
      const int row = e / (C::kCT / 4), col = 4 * (e % (C::kCT / 4));
      cp_async16(smem_u32(dst + row * C::kCT + col),
                 kt + static_cast<long long>(c0 + row) * nbs + j0 + col);
    }
  };
#pragma unroll
  for (int s0 = 0; s0 < C::kRing - 1; ++s0) {
    if (s0 < nch) issue(s0);
    cp_async_commit();
  }
  // The chunk's query means, transposed (invalid rows are 0), meanwhile.
  for (int e = tid; e < D * RB; e += C::kThreads) {
    const int r = e / D, c = e % D;
    qs[c * RB + r] = r < rows ? __ldg(qb + static_cast<long long>(r) * D + c) : 0.0f;
  }
  float acc[C::kRPT][4];
#pragma unroll
  for (int a2 = 0; a2 < C::kRPT; ++a2)
#pragma unroll
    for (int b2 = 0; b2 < 4; ++b2) acc[a2][b2] = 0.0f;
  for (int ch = 0; ch < nch; ++ch) {
    cp_async_wait<C::kRing - 2>();   // this thread's copies of chunk ch have landed
    __syncthreads();                 // everyone's have; chunk ch - 1 is no longer read
    if (ch + C::kRing - 1 < nch) issue(ch + C::kRing - 1);
    cp_async_commit();
    const float* kbuf = ks + (ch % C::kRing) * C::kKC * C::kCT;
    const int c0 = (ch % kChunks) * C::kKC;
    float4 qv[C::kKC][C::kRPT / 4], kv[C::kKC];
#pragma unroll
    for (int c = 0; c < C::kKC; ++c) {
#pragma unroll
      for (int g = 0; g < C::kRPT / 4; ++g)
        qv[c][g] = *reinterpret_cast<const float4*>(qs + (c0 + c) * RB + C::kRPT * ty + 4 * g);
      kv[c] = *reinterpret_cast<const float4*>(kbuf + c * C::kCT + 4 * tx);
    }
#pragma unroll
    for (int c = 0; c < C::kKC; ++c) {
      const float k4[4] = {kv[c].x, kv[c].y, kv[c].z, kv[c].w};
#pragma unroll
      for (int g = 0; g < C::kRPT / 4; ++g) {
        const float q4[4] = {qv[c][g].x, qv[c][g].y, qv[c][g].z, qv[c][g].w};
#pragma unroll
        for (int a2 = 0; a2 < 4; ++a2)
#pragma unroll
          for (int b2 = 0; b2 < 4; ++b2)
            acc[4 * g + a2][b2] = fmaf(q4[a2], k4[b2], acc[4 * g + a2][b2]);
      }
    }
    if (ch % kChunks == kChunks - 1) {
      const int j = (ch / kChunks) * C::kCT + 4 * tx;
#pragma unroll
      for (int a2 = 0; a2 < C::kRPT; ++a2) {
#pragma unroll
        for (int b2 = 0; b2 < 4; ++b2) {
          if (j + b2 < nb) sc[(C::kRPT * ty + a2) * nbp + j + b2] = acc[a2][b2];
          acc[a2][b2] = 0.0f;
        }
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();   // the ring is free for the recheck scratch
  // Largest key-mean norm of the head (from the pooling pass) and each row's
  // query-mean norm.
  float kmax2 = 0.0f;
  for (int j = tid; j < nb; j += C::kThreads) kmax2 = fmaxf(kmax2, __ldg(kn2 + bh * nb + j));
  red[tid] = kmax2;
  if (tid < RB) {
    float n2 = 0.0f;
    for (int c = 0; c < D; ++c) n2 = fmaf(qs[c * RB + tid], qs[c * RB + tid], n2);
    qn[tid] = sqrtf(n2);
  }
  __syncthreads();
  if (warp == 0) {
    float m = 0.0f;
    for (int t = lane; t < C::kThreads; t += 32) m = fmaxf(m, red[t]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) kmax_s[0] = sqrtf(m);
  }
  __syncthreads();
  const double kmax = kmax_s[0];

  // ---- phase 2: per row (warp), the k-th largest float32 score, the band
  // and, where needed, the float64 decision.  The staging buffers now hold
  // each warp's radix histogram and candidate buffer.
  unsigned* hist = reinterpret_cast<unsigned*>(ks) + warp * (256 + C::kCandMax * 3);
  double* cs = reinterpret_cast<double*>(hist + 256);
  int* cj = reinterpret_cast<int*>(cs + C::kCandMax);
  for (int r = warp; r < RB; r += C::kWarps) {
    unsigned* kept = bits + r * nw;
    for (int w = lane; w < nw; w += 32) kept[w] = 0u;
    __syncwarp();
    if (r >= rows) continue;
    const float* srow = sc + r * nbp;
    // The row's scores in registers: column j = lane + 32 u (-inf past nb).
    float vals[VPL];
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      const int j = lane + 32 * u;
      vals[u] = j < nb ? srow[j] : -INFINITY;
    }
    // Bracket the k-th largest float32 score T: cnt(>= lo) >= topk > cnt(>= hi),
    // so lo <= T < hi, by bisection on the value until the bracket is
    // narrower than the bound E allows.
    const double qnr = static_cast<double>(qn[r]);
    const bool wide = !(qnr < 1e18 && kmax < 1e18);
    const double E = (D + 8) * 5.9604644775390625e-8 * 1.05 * qnr * kmax + D * 2.4e-38;
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
      for (int it = 0; it < 64 && static_cast<double>(hi) - lo > 0.5 * E && c_lo - c_hi > 32;
           ++it) {
        const float mid = lo + 0.5f * (hi - lo);
        if (!(mid > lo && mid < hi)) break;   // adjacent floats
        const int cm = count_ge(mid);
        if (cm >= topk) { lo = mid; c_lo = cm; } else { hi = mid; c_hi = cm; }
      }
      blo = lo;
      bhi = hi;
      if (c_lo - c_hi <= 32) {
        // At most 32 scores lie in [lo, hi): gather them, one per lane, and
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
    auto is_cand_v = [&](float v) {
      const double dv = static_cast<double>(v);
      return !(dv > hi) && (wide || dv >= lo);
    };
    // Certain members (word u of the kept bitmap is the ballot over u) and
    // the candidates.
    int n_in = 0, n_cand = 0;
    unsigned cand_w[VPL];
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      const bool valid = lane + 32 * u < nb;
      const bool in = valid && static_cast<double>(vals[u]) > hi;
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
      if (n_cand <= C::kCandMax) {
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
      int written = 0;
      for (int w = 0; w < nw; ++w) {
        const unsigned word = kept[w];
        const int pos = written + __popc(word & ((1u << lane) - 1u));
        if (((word >> lane) & 1u) && pos < topk) out[pos] = 32 * w + lane;
        written += __popc(word);
      }
    }
  }
  if (lists == nullptr) return;
  __syncthreads();

  // ---- phase 3: union of the kept sets of each pair (2p, 2p+1) of the chunk
  const int npairs_all = (nb + 1) / 2;
  for (int pr = warp; pr < (rows + 1) / 2; pr += C::kWarps) {
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

struct SelectLayout {
  size_t qbar, kbar, qbar32, kbar32t, kn2, total;
  int nbs;   // row length of the channel-major float32 K means
};
SelectLayout select_layout(int B, int H, int N, int d, int block) {
  const size_t nb = (static_cast<size_t>(N) + block - 1) / block;
  const size_t BH = static_cast<size_t>(B) * H;
  SelectLayout L;
  // Whole 512-column tiles, so a chunk's copies never leave their row.
  L.nbs = static_cast<int>((nb + 511) / 512 * 512);
  L.qbar = 0;
  L.kbar = L.qbar + align256(BH * nb * d * sizeof(double));
  L.qbar32 = L.kbar + align256(BH * nb * d * sizeof(double));
  L.kbar32t = L.qbar32 + align256(BH * nb * d * sizeof(float));
  L.kn2 = L.kbar32t + align256(BH * d * L.nbs * sizeof(float));
  L.total = L.kn2 + align256(BH * nb * sizeof(float));
  return L;
}

template <int D, int RB, int VPL, int RPT = 4>
cudaError_t launch_select_fused(const Ctx& c, const float* q32, const float* k32t,
                                const float* kn2, const double* q64, const double* k64, int BH,
                                int nb, int nbs, int topk, int32_t* idx, int32_t* lists,
                                int32_t* counts) {
  const size_t smem = sel_smem_bytes<D, RB, RPT>(nb);
  cudaError_t e = cudaFuncSetAttribute(select_fused_kernel<D, RB, VPL, RPT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((nb + RB - 1) / RB, BH);
  select_fused_kernel<D, RB, VPL, RPT><<<grid, SelCfg<D, RB, RPT>::kThreads, smem, c.stream>>>(
      q32, k32t, kn2, q64, k64, nb, nbs, topk, idx, lists, counts);
  return cudaGetLastError();
}

// The chunk size (16 query blocks per CTA while their scores fit next to the
// staging ring, else 8; every nb up to 4096 fits) and the row's scores per
// lane kept in registers (nb <= 32 VPL).
template <int D>
cudaError_t dispatch_select(const Ctx& c, const float* q32, const float* k32t, const float* kn2,
                            const double* q64, const double* k64, int BH, int nb, int nbs,
                            int topk, int32_t* idx, int32_t* lists, int32_t* counts) {
  const bool rb16 = sel_smem_bytes<D, 16, 4>(nb) <= 200 * 1024;
  if (nb <= 512)
    return launch_select_fused<D, 16, 16, 8>(c, q32, k32t, kn2, q64, k64, BH, nb, nbs, topk, idx,
                                          lists, counts);
  if (nb <= 2048)
    return rb16 ? launch_select_fused<D, 16, 64>(c, q32, k32t, kn2, q64, k64, BH, nb, nbs, topk,
                                                 idx, lists, counts)
                : launch_select_fused<D, 8, 64>(c, q32, k32t, kn2, q64, k64, BH, nb, nbs, topk,
                                                idx, lists, counts);
  return launch_select_fused<D, 8, 128>(c, q32, k32t, kn2, q64, k64, BH, nb, nbs, topk, idx,
                                        lists, counts);
}

// Pools Q (z = 0) and K (z = 1), then selects.
cudaError_t pool_and_select(const Ctx& c, const void* q, const void* k, int B, int H, int N, int d,
                            int topk, int32_t* idx, void* ws, int32_t* lists, int32_t* counts) {
  const SelectLayout L = select_layout(B, H, N, d, kBlock);
  char* base = static_cast<char*>(ws);
  double* qbar = reinterpret_cast<double*>(base + L.qbar);
  double* kbar = reinterpret_cast<double*>(base + L.kbar);
  float* qbar32 = reinterpret_cast<float*>(base + L.qbar32);
  float* kbar32t = reinterpret_cast<float*>(base + L.kbar32t);
  float* kn2 = reinterpret_cast<float*>(base + L.kn2);
  const int nb = (N + kBlock - 1) / kBlock;
  const int BH = B * H;
  dim3 pg(nb, BH, 2);
  if (d == 128)
    pool_kernel<128><<<pg, 128, 0, c.stream>>>(static_cast<const uint4*>(q),
                                                static_cast<const uint4*>(k), N, nb, L.nbs, qbar,
                                                kbar, qbar32, kbar32t, kn2);
  else
    pool_kernel<64><<<pg, 128, 0, c.stream>>>(static_cast<const uint4*>(q),
                                               static_cast<const uint4*>(k), N, nb, L.nbs, qbar,
                                               kbar, qbar32, kbar32t, kn2);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (d == 128)
    return dispatch_select<128>(c, qbar32, kbar32t, kn2, qbar, kbar, BH, nb, L.nbs, topk, idx,
                                lists, counts);
  return dispatch_select<64>(c, qbar32, kbar32t, kn2, qbar, kbar, BH, nb, L.nbs, topk, idx,
                             lists, counts);
}

}  // namespace

size_t select_ws_bytes(int B, int H, int N, int d, int block) {
  return select_layout(B, H, N, d, block).total;
}

cudaError_t launch_select(const Ctx& c, const void* q, const void* k, int B, int H, int N, int d,
                          int topk, int32_t* idx, void* ws, int32_t* lists, int32_t* counts) {
  return pool_and_select(c, q, k, B, H, N, d, topk, idx, ws, lists, counts);
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
