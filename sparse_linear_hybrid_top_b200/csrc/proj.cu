// proj.cu -- the full-width projections of the hybrid layer on tcgen05.
//
// "SALAD: Sparse Attention with Linear Attention Distillation"
// (paper.rainbus.top), 方法步骤详情 steps 4 and 7: the linear branch's output
// passes a linear projection before the gated sum, and the heads' combined
// output passes the layer's output projection.  Read as full-width layers,
// both are one GEMM over the heads of a token concatenated (column h*d + c):
//
//   out[b][n][:] = resid[b][n][:] + s_b * (A_cat[b][n][:] W)
//
// with A [B][H][N][d] bf16 read in place (no concatenated copy: a 4-D tensor
// map over (d, N, H, B) serves the K slab h*d + c0 .. +64 of 128 tokens), W
// row-major [H*d][n_out] bf16 (an MN-major B operand, n contiguous), fp32
// accumulation in TMEM, and the gate scale plus the residual add fused into
// the epilogue.  out is per-head [B][H][N][d] (n_out == H*d, may alias resid:
// every element is read, then written, by the same thread) or token-major
// [B][N][n_out].
//
// Tiles: 128 tokens x NT output columns (NT = 256, 128 or 64, the widest that
// divides n_out), a ring of 64-deep K stages (A: 128 x 64, B: 64 x NT, both
// 128-byte swizzled), a persistent grid of one CTA per SM walking the tiles
// with the n tile fastest so the CTAs in flight share their A rows in L2.
// Warp roles (320 threads):
//   warp 0      TMA producer
//   warp 1      TMEM allocator and the single MMA-issuing thread
//   warps 2..9  epilogue: warp w reads TMEM lane quarter w % 4 (rows) and
//               column half (w - 2) / 4 of the accumulator.
// The accumulator is double-buffered in TMEM (2 x NT columns) so a tile's
// epilogue overlaps the next tile's MMAs.  Every wait is bounded; a wait that
// runs out raises the device error word and the CTA leaves through the common
// teardown (loads drained, MMAs committed, TMEM loads completed, TMEM freed).
#include "common.cuh"
#include "internal.h"

namespace salad {
namespace {

// ------------------------------------------------ CTA pairs (cta_group::2) --
// A cluster of two CTAs on the two SMs of a TPC shares each MMA: the even
// CTA (rank 0) issues it, A comes from both CTAs' shared memory (M halves),
// B likewise (N halves), and each CTA's TMEM holds its M half of D.
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory location in cluster CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}
// Arrive on an mbarrier of another CTA of the cluster (address from mapa).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
               : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_dst),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// D[tmem, both CTAs] (+)= A[smem, both CTAs] * B[smem, both CTAs]^T
__device__ __forceinline__ void mma_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` in every CTA of `cta_mask` when this thread's
// tcgen05 ops are done (an arrive, not a load: no data crosses CTAs).
__device__ __forceinline__ void mma_commit_pair_mc(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(cta_mask)
      : "memory");
}
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
// Tiled loads of one CTA of a pair into its own shared memory, completing
// on the mbarrier `cluster_bar` (in either CTA of the pair; no multicast).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t cluster_bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(map), "r"(cluster_bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_4d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t cluster_bar, int c0, int c1, int c2,
                                                 int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(map), "r"(cluster_bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

template <int NT>
struct PJ {
  static constexpr int kA = 128 * 128;          // 128 rows x 64 k, 128 B per row
  static constexpr int kBSlab = 64 * 128;       // 64 k rows x 64 n, 128 B per row
  static constexpr int kB = (NT / 64) * kBSlab;
  static constexpr int kStage = kA + kB;
  static constexpr int kStages = NT == 256 ? 4 : (NT == 128 ? 6 : 8);
  static constexpr int kCols = 2 * NT < 32 ? 32 : 2 * NT;   // TMEM columns (power of 2)
  static constexpr int kBarBytes = 256;
  static constexpr int kSmem = kStages * kStage + kBarBytes;
  static constexpr int kHalf = NT / 2;          // columns per epilogue warp
  static constexpr int kChunks = kHalf / 32;    // 32-column TMEM loads per warp
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
  static_assert((2 * kStages + 5) * 8 + 8 <= kBarBytes, "barrier region");
};

struct ProjParams {
  int B, H, N, d;
  int n_out;
  int kblocks;          // H*d / 64
  int m_tiles;          // ceil(N / 128)
  int n_tiles;          // n_out / NT
  long long tiles;      // B * m_tiles * n_tiles
  int out_per_head;
  __nv_bfloat16* out;
  const __nv_bfloat16* resid;
  const float* s;
  float drop;
  unsigned* err;
  unsigned long long wait_ns;
};

struct Tile {
  int b, mt, nt;
};

__device__ __forceinline__ Tile make_tile(const ProjParams& P, long long t) {
  Tile x;
  x.nt = static_cast<int>(t % P.n_tiles);
  const long long r = t / P.n_tiles;
  x.mt = static_cast<int>(r % P.m_tiles);
  x.b = static_cast<int>(r / P.m_tiles);
  return x;
}

// A sample whose linear branch is dropped keeps out == resid: every role
// skips its tiles (all read the same s_b, written by an earlier kernel).
__device__ __forceinline__ bool skip_sample(const ProjParams& P, int b) {
  return P.s != nullptr && P.s[b] < P.drop;
}

template <int NT>
__global__ void __launch_bounds__(320, 1) proj_kernel(const __grid_constant__ CUtensorMap ma,
                                                      const __grid_constant__ CUtensorMap mw,
                                                      const __grid_constant__ ProjParams P) {
  using C = PJ<NT>;
  constexpr int NS = C::kStages;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  if (reinterpret_cast<uintptr_t>(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(P.err, kErrLayout);
    return;
  }
  unsigned char* ring = smem_raw;   // [NS] x {A 128 x 64 | B (NT/64) slabs of 64 x 64}
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + NS * C::kStage);
  // bars: full[NS] empty[NS] acc_full[2] acc_empty[2] drain
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * NS + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  auto full = [&](int i) { return smem_u32(bars + i); };
  auto empty = [&](int i) { return smem_u32(bars + NS + i); };
  auto acc_full = [&](int i) { return smem_u32(bars + 2 * NS + i); };
  auto acc_empty = [&](int i) { return smem_u32(bars + 2 * NS + 2 + i); };
  const uint32_t drain = smem_u32(bars + 2 * NS + 4);
  auto st_addr = [&](long long c) { return smem_u32(ring + static_cast<int>(c % NS) * C::kStage); };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const unsigned long long wait_ns = P.wait_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(full(i), 1);
      mbar_init(empty(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full(i), 1);
      mbar_init(acc_empty(i), 8);   // the eight epilogue warps
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&ma);
    tma_prefetch_map(&mw);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), C::kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      // ================================================= TMA producer
      long long sc = 0;   // ring stages filled so far
      bool ok = true;
      for (long long t = blockIdx.x; t < P.tiles && ok; t += gridDim.x) {
        const Tile x = make_tile(P, t);
        if (skip_sample(P, x.b)) continue;
        for (int kb = 0; kb < P.kblocks; ++kb) {
          const int si = static_cast<int>(sc % NS);
          const long long n = sc / NS;
          if (n > 0 &&
              !mbar_wait(empty(si), static_cast<uint32_t>((n - 1) & 1), wait_ns, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t dst = st_addr(sc);
          ++sc;
          mbar_arrive_expect_tx(full(si), C::kStage);
          // K columns k0 .. k0+63 of the concatenated heads: head k0 / d,
          // channels k0 % d ..; token rows past N read 0.
          const int k0 = kb * 64;
          tma_load_4d(dst, &ma, full(si), k0 % P.d, x.mt * 128, k0 / P.d, x.b);
#pragma unroll
          for (int j = 0; j < NT / 64; ++j)
            tma_load_2d(dst + C::kA + j * C::kBSlab, &mw, full(si), x.nt * NT + j * 64, k0);
        }
      }
      if (!ok) raise_timeout(P.err, abort_flag);
      // Drain every issued load before leaving.
      for (int i = 0; i < NS && i < sc; ++i) {
        const long long last = i + ((sc - 1 - i) / NS) * NS;
        if (!mbar_wait(full(i), static_cast<uint32_t>((last / NS) & 1), wait_ns, nullptr))
          atomicOr(P.err, kErrTimeout);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ================================================= MMA issue
      // D[128 x NT] (+)= A[128 x 16] B[16 x NT] four times per stage.  A is
      // K-major (16 K elements = 32 bytes further along the swizzled row), B
      // MN-major (64-wide n slabs 8 KB apart, 16 K rows = 2 KB further).
      constexpr uint32_t idesc = idesc_bf16(128, NT, false, true);
      const uint64_t a_desc0 = sdesc_sw128(st_addr(0), 16, 1024);
      const uint64_t b_desc0 = sdesc_sw128(st_addr(0) + C::kA, C::kBSlab, 1024);
      long long sc = 0;
      uint32_t tc = 0;    // tiles computed (accumulator buffer tc & 1)
      bool ok = true;
      for (long long t = blockIdx.x; t < P.tiles && ok; t += gridDim.x) {
        const Tile x = make_tile(P, t);
        if (skip_sample(P, x.b)) continue;
        const int buf = static_cast<int>(tc & 1);
        if (tc >= 2 &&
            !mbar_wait(acc_empty(buf), ((tc - 2) >> 1) & 1, wait_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(buf * NT);
        for (int kb = 0; kb < P.kblocks; ++kb) {
          const int si = static_cast<int>(sc % NS);
          if (!mbar_wait(full(si), static_cast<uint32_t>((sc / NS) & 1), wait_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t off = static_cast<uint64_t>((si * C::kStage) >> 4);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_ss(acc, a_desc0 + off + ks * 2, b_desc0 + off + ks * 128, idesc,
                   (kb | ks) != 0 ? 1u : 0u);
          mma_commit(empty(si));
          ++sc;
        }
        if (!ok) break;
        mma_commit(acc_full(buf));
        ++tc;
      }
      if (!ok) raise_timeout(P.err, abort_flag);
      mma_commit(drain);
      if (!mbar_wait(drain, 0, wait_ns, nullptr)) atomicOr(P.err, kErrTimeout);
    }
    __syncwarp();
  } else {
    // ================================================= epilogue
    const int quarter = warp % 4;
    const int half = (warp - 2) / 4;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint32_t tc = 0;
    bool ok = true;
    for (long long t = blockIdx.x; t < P.tiles; t += gridDim.x) {
      const Tile x = make_tile(P, t);
      if (skip_sample(P, x.b)) continue;
      const int buf = static_cast<int>(tc & 1);
      const int n = x.mt * 128 + row;
      const bool live = n < P.N;
      const int j0 = x.nt * NT + half * C::kHalf;
      // Element (n, j) of out / resid.
      auto elem = [&](int j) -> long long {
        if (P.out_per_head) {
          const int h = j / P.d;
          return ((static_cast<long long>(x.b) * P.H + h) * P.N + n) * P.d + (j - h * P.d);
        }
        return (static_cast<long long>(x.b) * P.N + n) * P.n_out + j;
      };
      // The residual of this thread's columns, loaded before the wait.
      uint4 res[C::kChunks * 4];
#pragma unroll
      for (int i = 0; i < C::kChunks * 4; ++i) res[i] = make_uint4(0u, 0u, 0u, 0u);
      if (P.resid != nullptr && live) {
#pragma unroll
        for (int ch = 0; ch < C::kChunks; ++ch) {
          const uint4* src = reinterpret_cast<const uint4*>(P.resid + elem(j0 + ch * 32));
#pragma unroll
          for (int i = 0; i < 4; ++i) res[ch * 4 + i] = src[i];
        }
      }
      const float scale = P.s != nullptr ? P.s[x.b] : 1.0f;
      if (!__all_sync(0xffffffffu,
                      mbar_wait(acc_full(buf), (tc >> 1) & 1, wait_ns, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < C::kChunks; ++ch) {
        uint32_t r[32];
        tmem_ld32(lane_base + static_cast<uint32_t>(buf * NT + half * C::kHalf + ch * 32), r);
        if (live) {
          uint4 o[4];
          uint32_t* ow = reinterpret_cast<uint32_t*>(o);
          const uint32_t* rw = reinterpret_cast<const uint32_t*>(&res[ch * 4]);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 rv = unpack_bf16x2(rw[i]);
            ow[i] = pack_bf16x2(fmaf(scale, __uint_as_float(r[2 * i]), rv.x),
                                fmaf(scale, __uint_as_float(r[2 * i + 1]), rv.y));
          }
          uint4* dst = reinterpret_cast<uint4*>(P.out + elem(j0 + ch * 32));
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = o[i];
        }
      }
      // This warp is done with the buffer.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty(buf));
      ++tc;
    }
    if (!ok) raise_timeout(P.err, abort_flag);
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kCols);
  }
}

// ---------------------------------------------------------------------------
// The same GEMM on a pair of CTAs (cta_group::2), for n_out a multiple of 256:
// a pair tile is 256 tokens x 256 columns.  Each CTA loads its 128 token rows
// of A and its 128-column half of W per stage (32 KB), so a stage feeds the
// tensor pipe twice as long per byte of shared memory as in the single-CTA
// kernel, six stages fit, and W crosses L2 once per pair.  The even CTA
// issues the MMAs; both CTAs' loads complete on its full barriers, its
// commits arrive on both CTAs' empty and accumulator barriers, and both
// CTAs' epilogue warps release the accumulator on its barrier.
struct PJ2 {
  static constexpr int kA = 128 * 128;          // this CTA's 128 rows x 64 k
  static constexpr int kBSlab = 64 * 128;       // 64 k rows x 64 n
  static constexpr int kB = 2 * kBSlab;         // this CTA's 128 columns of W
  static constexpr int kStage = kA + kB;        // 32 KB
  static constexpr int kStages = 6;
  static constexpr int kCols = 512;             // two 128 x 256 fp32 accumulators
  static constexpr int kBarBytes = 256;
  static constexpr int kSmem = kStages * kStage + kBarBytes;
  static constexpr int kChunks = 4;             // 128 columns per epilogue warp
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
  static_assert((2 * kStages + 5) * 8 + 8 <= kBarBytes, "barrier region");
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(320, 1)
    proj_pair_kernel(const __grid_constant__ CUtensorMap ma, const __grid_constant__ CUtensorMap mw,
                     const __grid_constant__ ProjParams P) {
  using C = PJ2;
  constexpr int NS = C::kStages;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // Both CTAs see the same layout, so both leave here or neither does.
  if (reinterpret_cast<uintptr_t>(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(P.err, kErrLayout);
    return;
  }
  unsigned char* ring = smem_raw;   // [NS] x {A 128 x 64 | W 2 slabs of 64 x 64}
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + NS * C::kStage);
  // bars: full[NS] (used in the even CTA) empty[NS] acc_full[2] acc_empty[2]
  // (used in the even CTA) drain
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * NS + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  auto full = [&](int i) { return smem_u32(bars + i); };
  auto empty = [&](int i) { return smem_u32(bars + NS + i); };
  auto acc_full = [&](int i) { return smem_u32(bars + 2 * NS + i); };
  auto acc_empty = [&](int i) { return smem_u32(bars + 2 * NS + 2 + i); };
  const uint32_t drain = smem_u32(bars + 2 * NS + 4);
  auto st_addr = [&](long long c) { return smem_u32(ring + static_cast<int>(c % NS) * C::kStage); };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const bool even = rank == 0;
  const long long pair = blockIdx.x / 2, npairs = gridDim.x / 2;
  const unsigned long long wait_ns = P.wait_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(full(i), 1);
      mbar_init(empty(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full(i), 1);
      mbar_init(acc_empty(i), 16);   // eight epilogue warps in each CTA
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&ma);
    tma_prefetch_map(&mw);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_holder), C::kCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();   // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      // ================================================= TMA producer (each CTA)
      const uint32_t full0 = mapa_shared(full(0), 0);   // the even CTA's full[0]
      long long sc = 0;
      bool ok = true;
      for (long long t = pair; t < P.tiles && ok; t += npairs) {
        const Tile x = make_tile(P, t);
        if (skip_sample(P, x.b)) continue;
        for (int kb = 0; kb < P.kblocks; ++kb) {
          const int si = static_cast<int>(sc % NS);
          const long long n = sc / NS;
          if (n > 0 &&
              !mbar_wait(empty(si), static_cast<uint32_t>((n - 1) & 1), wait_ns, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t dst = st_addr(sc);
          ++sc;
          if (even) mbar_arrive_expect_tx(full(si), 2 * C::kStage);   // both CTAs' bytes
          const uint32_t fb = full0 + static_cast<uint32_t>(si) * 8u;
          const int k0 = kb * 64;
          tma_load_4d_pair(dst, &ma, fb, k0 % P.d, x.mt * 256 + static_cast<int>(rank) * 128,
                           k0 / P.d, x.b);
#pragma unroll
          for (int j = 0; j < 2; ++j)
            tma_load_2d_pair(dst + C::kA + j * C::kBSlab, &mw, fb,
                             x.nt * 256 + static_cast<int>(rank) * 128 + j * 64, k0);
        }
      }
      if (!ok) raise_timeout(P.err, abort_flag);
      // Drain: a fill has landed once the MMAs that read it are done, which
      // its stage's empty barrier reports; wait for each stage's last fill.
      for (int i = 0; i < NS && i < sc; ++i) {
        const long long last = i + ((sc - 1 - i) / NS) * NS;
        if (!mbar_wait(empty(i), static_cast<uint32_t>((last / NS) & 1), wait_ns, nullptr))
          atomicOr(P.err, kErrTimeout);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && even) {
      // ================================================= MMA issue (even CTA)
      // D[256 x 256] (+)= A[256 x 16] W[16 x 256] four times per stage; each
      // CTA holds 128 rows of A and 128 columns of W at the same offsets.
      constexpr uint32_t idesc = idesc_bf16(256, 256, false, true);
      const uint64_t a_desc0 = sdesc_sw128(st_addr(0), 16, 1024);
      const uint64_t b_desc0 = sdesc_sw128(st_addr(0) + C::kA, C::kBSlab, 1024);
      long long sc = 0;
      uint32_t tc = 0;
      bool ok = true;
      for (long long t = pair; t < P.tiles && ok; t += npairs) {
        const Tile x = make_tile(P, t);
        if (skip_sample(P, x.b)) continue;
        const int buf = static_cast<int>(tc & 1);
        if (tc >= 2 &&
            !mbar_wait(acc_empty(buf), ((tc - 2) >> 1) & 1, wait_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(buf * 256);
        for (int kb = 0; kb < P.kblocks; ++kb) {
          const int si = static_cast<int>(sc % NS);
          if (!mbar_wait(full(si), static_cast<uint32_t>((sc / NS) & 1), wait_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t off = static_cast<uint64_t>((si * C::kStage) >> 4);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_ss_pair(acc, a_desc0 + off + ks * 2, b_desc0 + off + ks * 128, idesc,
                        (kb | ks) != 0 ? 1u : 0u);
          mma_commit_pair_mc(empty(si), 0x3);
          ++sc;
        }
        if (!ok) break;
        mma_commit_pair_mc(acc_full(buf), 0x3);
        ++tc;
      }
      if (!ok) raise_timeout(P.err, abort_flag);
      mma_commit_pair(drain);
      if (!mbar_wait(drain, 0, wait_ns, nullptr)) atomicOr(P.err, kErrTimeout);
    }
    __syncwarp();
  } else {
    // ================================================= epilogue (each CTA)
    const int quarter = warp % 4;
    const int half = (warp - 2) / 4;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t acc_empty0 = mapa_shared(acc_empty(0), 0);   // the even CTA's
    uint32_t tc = 0;
    bool ok = true;
    for (long long t = pair; t < P.tiles; t += npairs) {
      const Tile x = make_tile(P, t);
      if (skip_sample(P, x.b)) continue;
      const int buf = static_cast<int>(tc & 1);
      const int n = x.mt * 256 + static_cast<int>(rank) * 128 + row;
      const bool live = n < P.N;
      const int j0 = x.nt * 256 + half * 128;
      auto elem = [&](int j) -> long long {
        if (P.out_per_head) {
          const int h = j / P.d;
          return ((static_cast<long long>(x.b) * P.H + h) * P.N + n) * P.d + (j - h * P.d);
        }
        return (static_cast<long long>(x.b) * P.N + n) * P.n_out + j;
      };
      uint4 res[C::kChunks * 4];
#pragma unroll
      for (int i = 0; i < C::kChunks * 4; ++i) res[i] = make_uint4(0u, 0u, 0u, 0u);
      if (P.resid != nullptr && live) {
#pragma unroll
        for (int ch = 0; ch < C::kChunks; ++ch) {
          const uint4* src = reinterpret_cast<const uint4*>(P.resid + elem(j0 + ch * 32));
#pragma unroll
          for (int i = 0; i < 4; ++i) res[ch * 4 + i] = src[i];
        }
      }
      const float scale = P.s != nullptr ? P.s[x.b] : 1.0f;
      if (!__all_sync(0xffffffffu,
                      mbar_wait(acc_full(buf), (tc >> 1) & 1, wait_ns, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < C::kChunks; ++ch) {
        uint32_t r[32];
        tmem_ld32(lane_base + static_cast<uint32_t>(buf * 256 + half * 128 + ch * 32), r);
        if (live) {
          uint4 o[4];
          uint32_t* ow = reinterpret_cast<uint32_t*>(o);
          const uint32_t* rw = reinterpret_cast<const uint32_t*>(&res[ch * 4]);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 rv = unpack_bf16x2(rw[i]);
            ow[i] = pack_bf16x2(fmaf(scale, __uint_as_float(r[2 * i]), rv.x),
                                fmaf(scale, __uint_as_float(r[2 * i + 1]), rv.y));
          }
          uint4* dst = reinterpret_cast<uint4*>(P.out + elem(j0 + ch * 32));
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = o[i];
        }
      }
      // This warp is done with the buffer: release it on the even CTA.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0 + static_cast<uint32_t>(buf) * 8u);
      ++tc;
    }
    if (!ok) raise_timeout(P.err, abort_flag);
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  }
  // Every MMA has drained and every TMEM load is done in both CTAs (and no
  // CTA leaves while the other may still read its shared memory).
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::kCols);
  }
}

cudaError_t launch_proj_pair(const Ctx& c, const ProjArgs& a, ProjParams P) {
  using C = PJ2;
  CUtensorMap ma, mw;
  if (!make_tmap_bf16_heads4d(&ma, a.a, a.B, a.H, a.N, a.d) ||
      !make_tmap_bf16_2d(&mw, a.w, a.H * a.d, a.n_out))
    return cudaErrorInvalidValue;
  P.m_tiles = (a.N + 255) / 256;
  P.n_tiles = a.n_out / 256;
  P.tiles = static_cast<long long>(a.B) * P.m_tiles * P.n_tiles;
  cudaError_t e = cudaFuncSetAttribute(proj_pair_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const long long pairs_max = c.num_sms / 2;
  long long pairs = P.tiles < pairs_max ? P.tiles : pairs_max;
  if (pairs < 1) pairs = 1;
  proj_pair_kernel<<<static_cast<int>(2 * pairs), 320, C::kSmem, c.stream>>>(ma, mw, P);
  return cudaGetLastError();
}

template <int NT>
cudaError_t launch_proj_t(const Ctx& c, const ProjArgs& a, ProjParams P) {
  using C = PJ<NT>;
  CUtensorMap ma, mw;
  if (!make_tmap_bf16_heads4d(&ma, a.a, a.B, a.H, a.N, a.d) ||
      !make_tmap_bf16_2d(&mw, a.w, a.H * a.d, a.n_out))
    return cudaErrorInvalidValue;
  P.n_tiles = a.n_out / NT;
  P.tiles = static_cast<long long>(a.B) * P.m_tiles * P.n_tiles;
  cudaError_t e = cudaFuncSetAttribute(proj_kernel<NT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  long long grid = P.tiles < c.num_sms ? P.tiles : c.num_sms;
  if (grid < 1) grid = 1;
  proj_kernel<NT><<<static_cast<int>(grid), 320, C::kSmem, c.stream>>>(ma, mw, P);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_proj(const Ctx& c, const ProjArgs& a) {
  if (a.n_out < 64 || a.n_out % 64 != 0 || a.d % 64 != 0) return cudaErrorInvalidValue;
  if (a.out_per_head && a.n_out != a.H * a.d) return cudaErrorInvalidValue;
  ProjParams P;
  P.B = a.B;
  P.H = a.H;
  P.N = a.N;
  P.d = a.d;
  P.n_out = a.n_out;
  P.kblocks = a.H * a.d / 64;
  P.m_tiles = (a.N + 127) / 128;
  P.n_tiles = 0;
  P.tiles = 0;
  P.out_per_head = a.out_per_head;
  P.out = static_cast<__nv_bfloat16*>(a.out);
  P.resid = static_cast<const __nv_bfloat16*>(a.resid);
  P.s = a.s;
  P.drop = a.drop;
  P.err = c.err;
  P.wait_ns = c.wait_ns;
  if (a.n_out % 256 == 0) return launch_proj_pair(c, a, P);
  if (a.n_out % 128 == 0) return launch_proj_t<128>(c, a, P);
  return launch_proj_t<64>(c, a, P);
}

}  // namespace salad
