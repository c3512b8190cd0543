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
// inputs in any realistic range), divided by the row count, and the scores
// are float64 dot products, so the kept set is decided in float64.
//
// Kernels: pool (HBM-bound: reads Q and K once), score (small float64 GEMM
// per head, nb x nb x d), topk (one warp per query block: radix select on
// order-preserving 64-bit keys, then an ordered compaction), pair_union
// (one warp per pair of query blocks: bitmap merge of the two kept lists).
#include "common.cuh"
#include "internal.h"

namespace salad {
namespace {

constexpr int kBlock = 64;

// ------------------------------------------------------------------ pool --
template <int D>
__global__ void __launch_bounds__(128) pool_kernel(const uint4* __restrict__ q,
                                                   const uint4* __restrict__ k, int N, int nb,
                                                   double* __restrict__ qbar,
                                                   double* __restrict__ kbar) {
  constexpr int CPR = D / 8;     // 16-byte chunks per row
  constexpr int RPI = 128 / CPR; // rows per iteration
  __shared__ double red[RPI][D];
  const int i = blockIdx.x;
  const long long bh = blockIdx.y;
  const uint4* src = blockIdx.z == 0 ? q : k;
  double* dst = blockIdx.z == 0 ? qbar : kbar;
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
  for (int c = threadIdx.x; c < D; c += 128) {
    double s = 0.0;
#pragma unroll
    for (int r = 0; r < RPI; ++r) s += red[r][c];
    dst[(bh * nb + i) * D + c] = s / static_cast<double>(rows);
  }
}

// ----------------------------------------------------------------- score --
// S[bh][i][j] = sum_c qbar[bh][i][c] * kbar[bh][j][c] in float64, each sum
// taken in ascending c.  64 x 64 tile per CTA of 128 threads, 8 (rows) x 4
// (columns) outputs per thread: rows 2*ty + {0,1} + 16a, columns 2*tx +
// {0,1} + 32b, so each 16-byte shared load of a half-warp covers contiguous
// banks.  The c dimension is staged 16 at a time through two shared buffers;
// the next chunk is read from global memory into registers while the current
// one is multiplied.
constexpr int kST = 64;    // tile edge
constexpr int kSK = 16;    // c-chunk staged per step
constexpr int kSPad = 2;   // row padding (keeps 16-byte alignment, spreads banks)
__global__ void __launch_bounds__(128, 4) score_kernel(const double* __restrict__ qbar,
                                                    const double* __restrict__ kbar, int nb,
                                                    int D, double* __restrict__ S) {
  __shared__ __align__(16) double qs[2][kSK][kST + kSPad];
  __shared__ __align__(16) double ks[2][kSK][kST + kSPad];
  const long long bh = blockIdx.z;
  const int i0 = blockIdx.y * kST, j0 = blockIdx.x * kST;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const double* qb = qbar + bh * nb * D;
  const double* kb = kbar + bh * nb * D;
  // Staging: thread t moves elements (row t/8 + 16v, c-pair t%8) of each
  // operand, v = 0..3: 16-byte reads, 128 bytes per row.
  const int sr = threadIdx.x / 8, sc = 2 * (threadIdx.x % 8);
  double2 gq[4], gk[4];
  auto fetch = [&](int c0) {
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int r = sr + 16 * v;
      gq[v] = (i0 + r < nb) ? *reinterpret_cast<const double2*>(qb + static_cast<long long>(i0 + r) * D + c0 + sc)
                            : make_double2(0.0, 0.0);
      gk[v] = (j0 + r < nb) ? *reinterpret_cast<const double2*>(kb + static_cast<long long>(j0 + r) * D + c0 + sc)
                            : make_double2(0.0, 0.0);
    }
  };
  auto stash = [&](int buf) {
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int r = sr + 16 * v;
      qs[buf][sc][r] = gq[v].x;
      qs[buf][sc + 1][r] = gq[v].y;
      ks[buf][sc][r] = gk[v].x;
      ks[buf][sc + 1][r] = gk[v].y;
    }
  };
  double acc[8][4];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
  const int nchunks = D / kSK;
  fetch(0);
  stash(0);
  __syncthreads();
  for (int ch = 0; ch < nchunks; ++ch) {
    const int buf = ch & 1;
    if (ch + 1 < nchunks) fetch((ch + 1) * kSK);
#pragma unroll
    for (int cc = 0; cc < kSK; ++cc) {
      double2 qa[4], kk[2];
#pragma unroll
      for (int a = 0; a < 4; ++a)
        qa[a] = *reinterpret_cast<const double2*>(&qs[buf][cc][2 * ty + 16 * a]);
#pragma unroll
      for (int b = 0; b < 2; ++b)
        kk[b] = *reinterpret_cast<const double2*>(&ks[buf][cc][2 * tx + 32 * b]);
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          acc[2 * a][2 * b] = fma(qa[a].x, kk[b].x, acc[2 * a][2 * b]);
          acc[2 * a][2 * b + 1] = fma(qa[a].x, kk[b].y, acc[2 * a][2 * b + 1]);
          acc[2 * a + 1][2 * b] = fma(qa[a].y, kk[b].x, acc[2 * a + 1][2 * b]);
          acc[2 * a + 1][2 * b + 1] = fma(qa[a].y, kk[b].y, acc[2 * a + 1][2 * b + 1]);
        }
    }
    // The other buffer was last read before the previous barrier.
    if (ch + 1 < nchunks) stash(buf ^ 1);
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int i = i0 + 2 * ty + 16 * (a / 2) + (a % 2);
    if (i >= nb) continue;
    double* srow = S + (bh * nb + i) * nb;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = j0 + 2 * tx + 32 * (b / 2) + (b % 2);
      if (j < nb) srow[j] = acc[a][b];
    }
  }
}

// ------------------------------------------------------------------ topk --
__device__ __forceinline__ unsigned long long order_key(double x) {
  x = x + 0.0;  // -0.0 -> +0.0: equal scores must share one key
  const unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(x));
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// One warp per query block row (bh, i).  Keys staged in shared memory.
__global__ void topk_kernel(const double* __restrict__ S, int nrows, int nb, int topk,
                            int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int warps = blockDim.x / 32;
  const int wid = threadIdx.x / 32, lane = threadIdx.x % 32;
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(smem_raw) +
                             static_cast<size_t>(wid) * nb;
  unsigned* hist = reinterpret_cast<unsigned*>(reinterpret_cast<unsigned long long*>(smem_raw) +
                                               static_cast<size_t>(warps) * nb) +
                   wid * 256;
  const long long row = static_cast<long long>(blockIdx.x) * warps + wid;
  if (row >= nrows) return;
  const double* srow = S + row * nb;
  for (int j = lane; j < nb; j += 32) keys[j] = order_key(srow[j]);
  __syncwarp();

  unsigned long long prefix = 0, pmask = 0;
  int want = topk;
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int j = lane; j < nb; j += 32) {
      const unsigned long long key = keys[j];
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncwarp();
    // Lane L owns bins 8L .. 8L+7.  Suffix sums over lanes find the digit.
    unsigned mine = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) mine += hist[lane * 8 + e];
    unsigned suffix = mine;  // inclusive suffix sum: bins >= 8L
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned t = __shfl_down_sync(0xffffffffu, suffix, o);
      if (lane + o < 32) suffix += t;
    }
    const unsigned above_lane = suffix - mine;  // bins >= 8(L+1)
    const bool here = (above_lane < static_cast<unsigned>(want)) &&
                      (suffix >= static_cast<unsigned>(want));
    const unsigned ballot = __ballot_sync(0xffffffffu, here);
    const int owner = __ffs(ballot) - 1;
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
    // Every key that shares the prefix so far is kept: the set is decided
    // (no tie among kept and dropped keys is left to break).
    const bool settled = hist[digit] == static_cast<unsigned>(want);
    __syncwarp();
    if (settled) {
      want = 0x7fffffff;
      break;
    }
  }
  // Keep every key whose masked value exceeds the prefix and the first
  // `want` whose masked value equals it, in index order.  After all eight
  // passes the mask is full and `prefix` is the exact key of the topk-th
  // largest score; after an early stop every equal key is kept.
  int32_t* out = idx + row * topk;
  int written = 0, eq_seen = 0;
  for (int j0 = 0; j0 < nb; j0 += 32) {
    const int j = j0 + lane;
    const unsigned long long key = j < nb ? (keys[j] & pmask) : 0ull;
    const bool gt = j < nb && key > prefix;
    const bool eq = j < nb && key == prefix;
    const unsigned eq_ballot = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_seen + __popc(eq_ballot & ((1u << lane) - 1u));
    const bool keep = gt || (eq && eq_rank < want);
    const unsigned kb = __ballot_sync(0xffffffffu, keep);
    const int pos = written + __popc(kb & ((1u << lane) - 1u));
    if (keep && pos < topk) out[pos] = j;
    written += __popc(kb);
    eq_seen += __popc(eq_ballot);
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
  size_t qbar, kbar, scores, total;
};
SelectLayout select_layout(int B, int H, int N, int d, int block) {
  const size_t nb = (static_cast<size_t>(N) + block - 1) / block;
  const size_t BH = static_cast<size_t>(B) * H;
  SelectLayout L;
  L.qbar = 0;
  L.kbar = L.qbar + align256(BH * nb * d * sizeof(double));
  L.scores = L.kbar + align256(BH * nb * d * sizeof(double));
  L.total = L.scores + align256(BH * nb * nb * sizeof(double));
  return L;
}

}  // namespace

size_t select_ws_bytes(int B, int H, int N, int d, int block) {
  return select_layout(B, H, N, d, block).total;
}

cudaError_t launch_select(const Ctx& c, const void* q, const void* k, int B, int H, int N, int d,
                          int topk, int32_t* idx, void* ws) {
  const SelectLayout L = select_layout(B, H, N, d, kBlock);
  char* base = static_cast<char*>(ws);
  double* qbar = reinterpret_cast<double*>(base + L.qbar);
  double* kbar = reinterpret_cast<double*>(base + L.kbar);
  double* S = reinterpret_cast<double*>(base + L.scores);
  const int nb = (N + kBlock - 1) / kBlock;
  const int BH = B * H;
  dim3 pg(nb, BH, 2);
  if (d == 128)
    pool_kernel<128><<<pg, 128, 0, c.stream>>>(static_cast<const uint4*>(q),
                                                static_cast<const uint4*>(k), N, nb, qbar, kbar);
  else
    pool_kernel<64><<<pg, 128, 0, c.stream>>>(static_cast<const uint4*>(q),
                                               static_cast<const uint4*>(k), N, nb, qbar, kbar);
  dim3 sg((nb + kST - 1) / kST, (nb + kST - 1) / kST, BH);
  score_kernel<<<sg, 128, 0, c.stream>>>(qbar, kbar, nb, d, S);
  // topk: as many warps per CTA as fit 192 KB of staged keys (>= 1).
  const size_t per_warp = static_cast<size_t>(nb) * 8 + 256 * 4;
  int warps = static_cast<int>((192 * 1024) / per_warp);
  if (warps > 8) warps = 8;
  if (warps < 1) warps = 1;
  const size_t smem = per_warp * warps;
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int nrows = BH * nb;
  topk_kernel<<<(nrows + warps - 1) / warps, warps * 32, smem, c.stream>>>(S, nrows, nb, topk,
                                                                          idx);
  return cudaGetLastError();
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
