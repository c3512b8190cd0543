// attn.cu -- block-sparse / sliding-window / dense flash attention on
// tcgen05 tensor cores, with the hybrid epilogue of the SALAD layer fused in.
//
// Sparse branch ("SALAD ... (paper.rainbus.top)" 前置知识 Sparse Attention,
// 方法步骤详情 step 2; "视频扩散模型中的稀疏注意力机制解析 (ijyty.com)" 1.1, 1.2):
// softmax(Q K^T / sqrt(d) + M) V with M in {-inf, 0}.  Hybrid epilogue
// (方法步骤详情 steps 3-6):  O = O_sparse + s_b * phi(Q) G / (phi(Q) Z + eps)
// with G = H W_lin[h] (the projection folded into the linear state, an exact
// algebraic regrouping of (phi(Q) H / den) W_lin).
//
// Tiling for sm_100a.  One work item is a pair of 64-row query blocks
// (M = 128 rows, the full tcgen05 datapath).  Its key tiles are the merged,
// ascending list of the blocks either query block keeps (Top-K), the band of
// blocks its rows' windows touch (ST-SWA) or all blocks (dense).  For each
// 64-key tile:  S = Q K^T  (A = Q from TMEM, B = K tile from smem, N = 64),
// P = exp2(S*c - m) written back over S in TMEM as bf16, O += P V
// (A = P from TMEM, B = V tile from smem, MN-major).  Rows whose query block
// did not keep a tile get P = 0 for it.
//
// S tiles hold 128 keys (two 64-key blocks of the list), so the QK MMA has
// N = 128: a tcgen05.mma with M = 128 occupies the tensor pipe for at least
// ~64 cycles whatever its N, which leaves an N = 64 MMA at half rate.  The K
// ring keeps consecutive 64-key stages contiguous inside each 128-byte-
// swizzled d-half slab, so a block pair is one B operand.
//
// Eight softmax warps: four row quarters (the TMEM lane groups) times two
// column halves.  The two warps holding a row exchange their partial row max
// every tile (through a bounded mbarrier), so both apply the same running max
// and O stays a single accumulator; each warp exponentiates 64 of the 128
// columns, rescales its half of O when the max grows by more than 2^8, and
// writes its half of the output.  S is double-buffered so the QK of the next
// tile runs during the softmax of this one.  The linear term
// s_b * phi(Q) G / (phi(Q) Z + eps) is one more MMA (A = phi(Q) from TMEM,
// B = the bf16 image of G streamed into the V slots of a ring stage) into the
// S_0 columns, which are free once the last PV has run.
//
// Warp roles (320 threads, one CTA per SM, persistent over work items):
//   warp 0      TMA producer: K and V blocks (64 x d, 128B swizzle), two per
//               ring stage, and the G image.
//   warp 1      TMEM allocator and the single MMA-issuing thread.
//   warps 2..5  softmax, column half 0; also load Q and phi(Q).
//   warps 6..9  softmax, column half 1.
// TMEM columns (d = 128): O [0,128) S_0 [128,256) S_1 [256,384) Q [384,448)
// phi(Q) [448,512); the linear term lands in S_0.
//
// Barrier discipline: an mbarrier parity wait is only sound when the waiter is
// at most one phase behind.  Every barrier is observed by each of its waiters
// at every phase: in particular each softmax warp waits for its previous PV
// once per tile (after computing and storing P, so the wait overlaps its own
// work), rescales its O only then, and only then releases the tile.  Every
// wait is bounded; a wait that runs out raises the device error word and the
// CTA leaves through the common teardown (loads drained, MMAs committed, TMEM
// freed).
#include "common.cuh"
#include "internal.h"

namespace salad {
namespace {

constexpr int kSlab = 64 * 128;

template <int D, bool HYB>
struct AT {
  static constexpr int kKS = 6;                          // 64-key stages (even: pairs never wrap)
  static constexpr int kPairs = kKS / 2;                 // ring stages of two blocks
  static constexpr int kHalves = D / 64;                 // 128-byte d-slabs per row
  static constexpr int kTile = kHalves * kSlab;          // one 64-key K (or V) block
  static constexpr int kKRingHalf = kKS * kSlab;         // one d-slab of the K ring
  static constexpr int kKRing = kHalves * kKRingHalf;
  static constexpr int kVRing = kKS * kTile;
  static constexpr int kGImg = D * D * 2;                // bf16 G image bytes (own buffer)
  static constexpr int kXchg = (2 * 2 * 128 + 128) * 4;  // row max/sum per parity, den
  static constexpr int kBarBytes = 256;
  // The dynamic shared memory is declared 1024-byte aligned (the 128-byte
  // swizzle atoms need it), so no slack is reserved for aligning it.
  static constexpr int kSmemUsed = kKRing + kVRing + kGImg + kXchg + kBarBytes;
  static_assert(kSmemUsed <= 227 * 1024, "shared memory budget");
  // At least ~half of the SM's shared memory, so one CTA (and its 512 TMEM
  // columns) occupies each SM.
  static constexpr int kSmem = kSmemUsed > 120 * 1024 ? kSmemUsed : 120 * 1024;
  // TMEM columns.
  static constexpr uint32_t kO = 0;            // D columns
  static constexpr uint32_t kS0 = D;           // 128 columns (P aliases the first 64)
  static constexpr uint32_t kS1 = D + 128;     // 128 columns
  static constexpr uint32_t kL = D;            // linear term, D columns over S_0
  static constexpr uint32_t kQ = D + 256;      // D/2 columns (A operand)
  static constexpr uint32_t kPQ = kQ + D / 2;  // D/2 columns (A operand)
  static constexpr uint32_t kCols = 512;
  static_assert(kPQ + D / 2 <= kCols, "TMEM budget");
  static_assert(D <= 128, "the linear term must fit S_0");
};

struct Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* qp;
  short head_slot[256];       // slot in the regrouped copies, -1 = frame-major head
  int B, H, N, Hs, nb, npairs;
  int mode, window, F, Hh, Wh;
  const int32_t* lists;
  const int32_t* counts;
  int list_stride;
  const __nv_bfloat16* Gimg;  // [B*H][d*d] bf16 B-operand images of G
  const float* Z;
  const float* s;
  float gate_override;
  float drop;                 // the linear term of sample b is skipped when s_b < drop
  Rope3D rope;                // 3-D rotary encoding of phi(Q) in the linear term
  float eps;
  float scale_log2;
  __nv_bfloat16* o;
  unsigned* err;
  unsigned long long wait_ns;
};

struct Item {
  int bh, b, h, p;
  int ntiles;
  int jlo;                // first key block (band / dense)
  const int32_t* list;    // topk entries
  int slot;               // >= 0: regrouped (space-major) head
};

__device__ __forceinline__ Item make_item(const Params& P, long long w) {
  Item it;
  it.bh = static_cast<int>(w / P.npairs);
  it.p = static_cast<int>(w % P.npairs);
  it.b = it.bh / P.H;
  it.h = it.bh % P.H;
  it.slot = P.head_slot[it.h];
  it.list = nullptr;
  it.jlo = 0;
  if (P.mode == kModeTopk) {
    it.list = P.lists + w * static_cast<long long>(P.list_stride);
    it.ntiles = P.counts[w];
  } else if (P.mode == kModeDense) {
    it.ntiles = P.nb;
  } else {
    const int r0 = it.p * 128;
    const int r1 = min(P.N, r0 + 128) - 1;
    const int lo = max(0, r0 - P.window);
    const int hi = min(P.N - 1, r1 + P.window);
    it.jlo = lo / 64;
    it.ntiles = hi / 64 - it.jlo + 1;
  }
  return it;
}

// Whether sample b keeps its linear branch (post-training branch dropping:
// the branch is skipped when the gate value is below the threshold).
__device__ __forceinline__ bool lin_on(const Params& P, int b) {
  const float g = P.s != nullptr ? __ldg(P.s + b) : P.gate_override;
  return !(g < P.drop);
}

__device__ __forceinline__ void tile_of(const Item& it, int t, int mode, int& j, int& mask) {
  if (mode == kModeTopk) {
    const int e = __ldg(it.list + t);
    j = e & 0xFFFF;
    mask = e >> 16;
  } else {
    j = it.jlo + t;
    mask = 3;
  }
}

// Maximum of 64 values by a tree of three-input maxima (64 -> 22 -> 8 -> 3 -> 1).
__device__ __forceinline__ float max64(const float* v) {
  float a[22];
#pragma unroll
  for (int i = 0; i < 21; ++i) a[i] = fmax3(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
  a[21] = v[63];
  float b[8];
#pragma unroll
  for (int i = 0; i < 7; ++i) b[i] = fmax3(a[3 * i], a[3 * i + 1], a[3 * i + 2]);
  b[7] = a[21];
  return fmax3(fmax3(b[0], b[1], b[2]), fmax3(b[3], b[4], b[5]), fmaxf(b[6], b[7]));
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Bulk prefetch of [src, src + bytes) into L2 (16-byte aligned, multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Untiled bulk copy global -> shared completing on `bar` (16-byte aligned).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

template <int D, bool HYB>
__global__ void __launch_bounds__(320, 1) attn_kernel(const __grid_constant__ CUtensorMap mk,
                                                      const __grid_constant__ CUtensorMap mv,
                                                      const __grid_constant__ CUtensorMap mkp,
                                                      const __grid_constant__ CUtensorMap mvp,
                                                      const __grid_constant__ Params P) {
  using C = AT<D, HYB>;
  constexpr int NP = C::kPairs;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // The layout below assumes the declared alignment; refuse to run without it.
  if (reinterpret_cast<uintptr_t>(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(P.err, kErrLayout);
    return;
  }
  unsigned char* sm = smem_raw;
  unsigned char* kring = sm;                         // [d-slab][kKS x 64 rows x 128 B]
  unsigned char* vring = sm + C::kKRing;             // [kKS][d-slab][64 rows x 128 B]
  unsigned char* gbuf = vring + C::kVRing;           // G image of the current item's head
  float* xrow = reinterpret_cast<float*>(gbuf + C::kGImg);    // [parity][half][128] row max / sum
  float* xden = xrow + 2 * 2 * 128;                            // [128] phi(q) . Z + eps
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<unsigned char*>(xrow) + C::kXchg);
  // bars: full[NP] empty[NP] s_full[2] p_full[2] o_done q_ready lin_done drain x_row[4] g_full
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * NP + 13);
  static_assert((2 * NP + 13) * 8 + 8 <= C::kBarBytes, "barrier region");
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  auto full = [&](int p) { return smem_u32(bars + p); };
  auto empty = [&](int p) { return smem_u32(bars + NP + p); };
  auto s_full = [&](int b) { return smem_u32(bars + 2 * NP + b); };
  auto p_full = [&](int b) { return smem_u32(bars + 2 * NP + 2 + b); };
  const uint32_t o_done = smem_u32(bars + 2 * NP + 4);
  const uint32_t q_ready = smem_u32(bars + 2 * NP + 5);
  const uint32_t lin_done = smem_u32(bars + 2 * NP + 6);
  const uint32_t drain = smem_u32(bars + 2 * NP + 7);
  auto x_row = [&](int q) { return smem_u32(bars + 2 * NP + 8 + q); };
  const uint32_t g_full = smem_u32(bars + 2 * NP + 12);
  // Shared-memory addresses of the blocks of ring stage (pair) p.
  auto k_addr = [&](int p, int half) {   // rows of block 2p (then 2p+1) of one d-slab
    return smem_u32(kring + half * C::kKRingHalf + 2 * p * kSlab);
  };
  auto v_addr = [&](int p, int which) {  // V block 2p + which
    return smem_u32(vring + (2 * p + which) * C::kTile);
  };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long total = static_cast<long long>(P.B) * P.H * P.npairs;
  const unsigned long long wait_ns = P.wait_ns;

  if (threadIdx.x == 0) {
    for (int p = 0; p < NP; ++p) {
      mbar_init(full(p), 1);
      mbar_init(empty(p), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full(b), 1);
      mbar_init(p_full(b), 8);
    }
    mbar_init(o_done, 1);
    mbar_init(q_ready, 8);   // half 0 after writing Q, half 1 after its previous epilogue
    mbar_init(lin_done, 1);
    mbar_init(drain, 1);
    for (int q = 0; q < 4; ++q) mbar_init(x_row(q), 2);   // the two warps of a row quarter
    mbar_init(g_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&mk);
    tma_prefetch_map(&mv);
    if (P.Hs > 0) {
      tma_prefetch_map(&mkp);
      tma_prefetch_map(&mvp);
    }
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
      long long pc = 0;   // ring stages filled so far
      bool ok = true;
      for (long long w = blockIdx.x; w < total && ok; w += gridDim.x) {
        const Item it = make_item(P, w);
        const CUtensorMap* km = it.slot >= 0 ? &mkp : &mk;
        const CUtensorMap* vm = it.slot >= 0 ? &mvp : &mv;
        const int z = it.slot >= 0 ? it.b * P.Hs + it.slot : it.bh;
        const int npair = (it.ntiles + 1) / 2;
        if (w + gridDim.x < total) {
          // The next item's rows of Q into L2 (one contiguous run), an item
          // ahead of the softmax warps that load them.
          const Item nx = make_item(P, w + gridDim.x);
          const __nv_bfloat16* qsrc =
              nx.slot >= 0 ? P.qp + (static_cast<long long>(nx.b) * P.Hs + nx.slot) * P.N * D
                           : P.q + static_cast<long long>(nx.bh) * P.N * D;
          const int rows = min(128, P.N - nx.p * 128);
          prefetch_l2(qsrc + static_cast<long long>(nx.p) * 128 * D,
                      static_cast<uint32_t>(rows) * D * 2);
        }
        for (int u = 0; u < npair; ++u, ++pc) {
          const int p = static_cast<int>(pc % NP);
          const long long n = pc / NP;
          if (n > 0 && !mbar_wait(empty(p), static_cast<uint32_t>((n - 1) & 1), wait_ns, abort_flag)) {
            raise_timeout(P.err, abort_flag);
            ok = false;
            break;
          }
          if (u < npair) {
            const int nblk = (2 * u + 1 < it.ntiles) ? 2 : 1;
            mbar_arrive_expect_tx(full(p), nblk * 2 * C::kTile);
            for (int x = 0; x < nblk; ++x) {
              int j, mask;
              tile_of(it, 2 * u + x, P.mode, j, mask);
#pragma unroll
              for (int hh = 0; hh < D / 64; ++hh) {
                tma_load_3d(k_addr(p, hh) + x * kSlab, km, full(p), hh * 64, j * 64, z);
                tma_load_3d(v_addr(p, x) + hh * kSlab, vm, full(p), hh * 64, j * 64, z);
              }
            }
          }
        }
      }
      // Drain every issued load before leaving.
      for (int p = 0; p < NP && p < pc; ++p) {
        const long long last = p + ((pc - 1 - p) / NP) * NP;
        if (!mbar_wait(full(p), static_cast<uint32_t>((last / NP) & 1), wait_ns, nullptr))
          atomicOr(P.err, kErrTimeout);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ================================================= MMA issuer
      constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
      constexpr uint32_t idesc_lin = idesc_bf16(128, D, false, false);
      long long pc = 0;
      uint32_t ic = 0;
      uint32_t pf[2] = {0, 0};
      bool ok = true;
      auto wait_full = [&](long long c) -> bool {
        return mbar_wait(full(static_cast<int>(c % NP)), static_cast<uint32_t>((c / NP) & 1),
                         wait_ns, abort_flag);
      };
      auto issue_qk = [&](long long c, int b) {
        const int p = static_cast<int>(c % NP);
        const uint32_t sbuf = b ? C::kS1 : C::kS0;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_ts(tmem + sbuf, tmem + C::kQ + ks * 8,
                 sdesc_sw128(k_addr(p, ks / 4) + (ks % 4) * 32, 16, 1024), idesc_qk,
                 ks > 0 ? 1u : 0u);
        mma_commit(s_full(b));
      };
      uint32_t lc = 0;   // items with a linear term so far
      for (long long w = blockIdx.x; w < total && ok; w += gridDim.x, ++ic) {
        const Item it = make_item(P, w);
        const int npair = (it.ntiles + 1) / 2;
        if (!mbar_wait(q_ready, ic & 1, wait_ns, abort_flag)) { ok = false; break; }
        tc_fence_after();
        for (int u = 0; u < 2 && u < npair; ++u) {
          if (!wait_full(pc + u)) { ok = false; break; }
          tc_fence_after();
          issue_qk(pc + u, u);
        }
        if (!ok) break;
        for (int u = 0; u < npair; ++u) {
          const int b = u & 1;
          if (!mbar_wait(p_full(b), pf[b] & 1, wait_ns, abort_flag)) { ok = false; break; }
          ++pf[b];
          tc_fence_after();
          const int p = static_cast<int>((pc + u) % NP);
          const uint32_t pbuf = b ? C::kS1 : C::kS0;
          const int nks = (2 * u + 1 < it.ntiles) ? 8 : 4;   // K-steps: 16 keys each
          for (int ks = 0; ks < nks; ++ks)
            mma_ts(tmem + C::kO, tmem + pbuf + ks * 8,
                   sdesc_sw128(v_addr(p, ks / 4) + (ks % 4) * 2048, kSlab, 1024), idesc_pv,
                   (u > 0 || ks > 0) ? 1u : 0u);
          mma_commit(empty(p));
          mma_commit(o_done);
          if (u + 2 < npair) {
            if (!wait_full(pc + u + 2)) { ok = false; break; }
            tc_fence_after();
            issue_qk(pc + u + 2, b);   // same S buffer: runs after this PV in issue order
          }
        }
        if (!ok) break;
        pc += npair;
        if (HYB && lin_on(P, it.b)) {
          // Linear term into S_0 (free once the last PV has run): L = phi(Q) G,
          // B = the item's G image in its own buffer.
          if (!mbar_wait(g_full, lc & 1, wait_ns, abort_flag)) { ok = false; break; }
          ++lc;
          tc_fence_after();
          const uint32_t gaddr = smem_u32(gbuf);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            mma_ts(tmem + C::kL, tmem + C::kPQ + ks * 8,
                   sdesc_sw128(gaddr + (ks / 4) * (D * 128) + (ks % 4) * 32, 16, 1024), idesc_lin,
                   ks > 0 ? 1u : 0u);
          mma_commit(lin_done);
        }
      }
      if (!ok) raise_timeout(P.err, abort_flag);
      mma_commit(drain);
      if (!mbar_wait(drain, 0, wait_ns, nullptr)) atomicOr(P.err, kErrTimeout);
    }
  } else {
    // ================================================= softmax + epilogue
    const int hf = (warp - 2) / 4;              // column half of S, P, O and the output
    const int quarter = warp % 4;
    const int r = quarter * 32 + lane;          // row within the pair (TMEM lane)
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint32_t ic = 0, sf[2] = {0, 0}, xc = 0;
    long long pv_base = 0;                      // PVs completed before this item
    bool ok = true;
    // One thread streams each item's G image into its buffer: the first now,
    // each next one as soon as the linear term of the current item is done.
    // Items whose sample dropped its linear branch are skipped.
    const bool g_loader = HYB && warp == 2 && lane == 0;
    long long g_issued = 0;
    uint32_t lc = 0;   // items with a linear term so far
    auto load_g = [&](long long from) {
      for (long long w = from; w < total; w += gridDim.x) {
        const Item nx = make_item(P, w);
        if (!lin_on(P, nx.b)) continue;
        mbar_arrive_expect_tx(g_full, C::kGImg);
        bulk_load(smem_u32(gbuf), P.Gimg + static_cast<long long>(nx.bh) * D * D, C::kGImg,
                  g_full);
        ++g_issued;
        return;
      }
    };
    if (g_loader) load_g(blockIdx.x);
    // Exchange of a per-row value with the other half's warp of this quarter.
    auto exchange = [&](float mine) -> float {
      float* slot = xrow + (xc & 1) * 256;
      slot[hf * 128 + r] = mine;
      __syncwarp();
      if (lane == 0) mbar_arrive(x_row(quarter));
      const bool got = __all_sync(0xffffffffu, mbar_wait(x_row(quarter), xc & 1, wait_ns, abort_flag));
      ++xc;
      if (!got) {
        ok = false;
        return mine;
      }
      return slot[(1 - hf) * 128 + r];
    };
    for (long long w = blockIdx.x; w < total && ok; w += gridDim.x, ++ic) {
      const Item it = make_item(P, w);
      const int row_pos = it.p * 128 + r;        // position in the head's (possibly regrouped) order
      const bool row_valid = row_pos < P.N;
      const int npair = (it.ntiles + 1) / 2;
      const bool lin = HYB && lin_on(P, it.b);   // this item adds the linear term
      float den_row = 0.f;   // phi(q) . Z + eps of the row
      if (hf == 1) {
        // This warp's previous epilogue is complete: O, S and the linear
        // term may be overwritten by this item's MMAs.
        __syncwarp();
        if (lane == 0) mbar_arrive(q_ready);
        // Half 0 has written den for this item once q_ready completes; it
        // writes the next one only after this item's last PV, which needs
        // this warp's P, so the single slot is safe to read here.
        if (!__all_sync(0xffffffffu, mbar_wait(q_ready, ic & 1, wait_ns, abort_flag))) {
          ok = false;
          break;
        }
        if (lin) den_row = xden[r];
      } else {
        // ---- Q and phi(Q) into TMEM (A operands); den = phi(q) . Z + eps
        const __nv_bfloat16* qsrc =
            it.slot >= 0 ? P.qp + (static_cast<long long>(it.b) * P.Hs + it.slot) * P.N * D
                         : P.q + static_cast<long long>(it.bh) * P.N * D;
        const uint4* qrow = reinterpret_cast<const uint4*>(
            qsrc + static_cast<long long>(row_valid ? row_pos : 0) * D);
        const float* zrow = HYB ? P.Z + static_cast<long long>(it.bh) * D : nullptr;
        float den = 0.f;
        // Grid position of the row's token (its frame-major index) for the
        // rotary encoding of the linear term.
        const bool rope_on = lin && P.rope.on && row_valid;
        int rf = 0, ry = 0, rx = 0;
        if (rope_on) {
          int tok = row_pos;
          if (it.slot >= 0) {
            const int fr = row_pos % P.F, pos = row_pos / P.F;
            tok = fr * (P.Hh * P.Wh) + pos;
          }
          const int plane = P.rope.Hh * P.rope.Wh;   // token -> (frame, row, column)
          rf = tok / plane;
          ry = (tok / P.rope.Wh) % P.rope.Hh;
          rx = tok % P.rope.Wh;
        }
#pragma unroll
        for (int c0 = 0; c0 < D / 2; c0 += 16) {
          uint32_t pk[16];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint4 v = row_valid ? __ldg(qrow + c0 / 4 + u) : make_uint4(0, 0, 0, 0);
            pk[4 * u + 0] = v.x; pk[4 * u + 1] = v.y; pk[4 * u + 2] = v.z; pk[4 * u + 3] = v.w;
          }
          tmem_st16(lane_base + C::kQ + c0, pk);
          if (lin) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              pk[e] = relu_bf16x2(pk[e]);
              const float2 f = unpack_bf16x2(pk[e]);
              den = fmaf(f.x, __ldg(zrow + 2 * (c0 + e)), den);
              den = fmaf(f.y, __ldg(zrow + 2 * (c0 + e) + 1), den);
            }
            if (rope_on) {
              // The numerator's phi(q) is rotated (word c0 + e is pair c0 + e);
              // the denominator above is not.
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const float2 cs = rope_cs(P.rope, P.rope.theta, c0 + e, rf, ry, rx);
                const float2 a = unpack_bf16x2(pk[e]);
                pk[e] = pack_bf16x2(a.x * cs.x - a.y * cs.y, a.x * cs.y + a.y * cs.x);
              }
            }
            tmem_st16(lane_base + C::kPQ + c0, pk);
          }
        }
        den_row = den + P.eps;
        xden[r] = den_row;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(q_ready);
      }

      // ---- softmax over the item's S tiles (128 keys each)
      const float c2 = P.scale_log2;
      float m = -INFINITY;   // running max of the row in the exp2 domain (same in both halves)
      float l = 0.f;         // this half's share of the row sum
      const int half_bit = r >= 64 ? 2 : 1;
      for (int u = 0; u < npair; ++u) {
        const int b = u & 1;
        const uint32_t sbuf = b ? C::kS1 : C::kS0;
        // Waits and TMEM accesses are warp-collective: every decision that
        // guards one is made uniform across the warp first.
        if (!__all_sync(0xffffffffu, mbar_wait(s_full(b), sf[b] & 1, wait_ns, abort_flag))) {
          ok = false;
          break;
        }
        ++sf[b];
        tc_fence_after();
        const int t = 2 * u + hf;                  // this half's key block
        int j = 0, mask = 0;
        if (t < it.ntiles) tile_of(it, t, P.mode, j, mask);
        // Valid key columns of the block form one contiguous range [lo, hi].
        int lo = 0, hi = min(63, P.N - 1 - j * 64);
        if (P.mode == kModeBand) {
          lo = max(lo, row_pos - P.window - j * 64);
          hi = min(hi, row_pos + P.window - j * 64);
        }
        const bool live = row_valid && (mask & half_bit) && lo <= hi;
        const bool whole = live && lo == 0 && hi == 63;
        const bool any_live = __any_sync(0xffffffffu, live);
        float sv[64];
        float pm = -INFINITY;
        if (any_live) {
          {
            uint32_t s64[64];
            tmem_ld64(lane_base + sbuf + hf * 64, s64);
#pragma unroll
            for (int c = 0; c < 64; ++c) sv[c] = __uint_as_float(s64[c]);
          }
          // Columns outside [lo, hi] (and every column of a dead row) become
          // -inf; only blocks with a partial row in this warp pay for it.
          if (__any_sync(0xffffffffu, !whole)) {
#pragma unroll
            for (int c = 0; c < 64; ++c) sv[c] = (live && c >= lo && c <= hi) ? sv[c] : -INFINITY;
          }
          // Row max by a tree of three-input maxima (64 -> 22 -> 8 -> 3 -> 1).
          pm = max64(sv) * c2;   // c2 > 0: max of scaled = scaled max
        }
        // Both halves have loaded their S columns once the exchange completes,
        // so P may now be written over S.
        const float mx = fmaxf(pm, exchange(pm));
        if (!ok) break;
        float f = 1.0f;            // factor O must be rescaled by before this PV
        if (mx > m + 8.0f) {
          // Raise the running max.  O (earlier PVs) is rescaled below, once
          // the previous PV has landed; l is rescaled here.
          f = (m == -INFINITY) ? 1.0f : ex2(m - mx);
          l *= f;
          m = mx;
        }
        uint32_t pk[32];
        if (any_live) {
          // A row with no valid key so far keeps m = -inf: use 0 as the
          // offset so its -inf scores give exp2(-inf) = 0, never NaN.
          const float nm = (m == -INFINITY) ? 0.0f : -m;
          float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float a0 = ex2(fmaf(sv[c], c2, nm));
            const float a1 = ex2(fmaf(sv[c + 1], c2, nm));
            const float b0 = ex2(fmaf(sv[c + 32], c2, nm));
            const float b1 = ex2(fmaf(sv[c + 33], c2, nm));
            pk[c / 2] = pack_bf16x2(a0, a1);
            pk[16 + c / 2] = pack_bf16x2(b0, b1);
            ls0 += a0 + a1;
            ls1 += b0 + b1;
          }
          l += ls0 + ls1;
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) pk[e] = 0u;
        }
        tmem_st32(lane_base + sbuf + hf * 32, pk);
        // Observe PV(u-1): every warp observes every PV completion in order,
        // so each parity wait is at most one phase behind the barrier.
        if (u >= 1) {
          const long long g = pv_base + u - 1;
          if (!__all_sync(0xffffffffu, mbar_wait(o_done, static_cast<uint32_t>(g & 1), wait_ns, abort_flag))) {
            ok = false;
            break;
          }
        }
        if (__any_sync(0xffffffffu, f != 1.0f)) {
          tc_fence_after();
#pragma unroll
          for (int c0 = hf * (D / 2); c0 < (hf + 1) * (D / 2); c0 += 32) {
            uint32_t o32[32];
            tmem_ld32(lane_base + C::kO + c0, o32);
#pragma unroll
            for (int e = 0; e < 32; ++e) o32[e] = __float_as_uint(__uint_as_float(o32[e]) * f);
            tmem_st32(lane_base + C::kO + c0, o32);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(b));
      }
      if (!ok) break;
      {
        // The item's last PV has landed.
        const long long g = pv_base + npair - 1;
        if (!__all_sync(0xffffffffu, mbar_wait(o_done, static_cast<uint32_t>(g & 1), wait_ns, abort_flag))) {
          ok = false;
          break;
        }
        pv_base += npair;
      }
      // ---- row sum over both halves
      const float L = l + exchange(l);
      if (!ok) break;
      const float inv_l = 1.0f / L;
      float lin_scale = 0.f;
      if (lin) {
        const float gate = P.s != nullptr ? __ldg(P.s + it.b) : P.gate_override;
        const float den = den_row;
        lin_scale = den > 0.f ? gate / den : 0.f;
        if (!__all_sync(0xffffffffu, mbar_wait(lin_done, lc & 1, wait_ns, abort_flag))) {
          ok = false;
          break;
        }
        ++lc;
        // The linear term has read G: the next item's image may replace it.
        if (g_loader) load_g(w + gridDim.x);
      }
      tc_fence_after();
      // ---- epilogue: this warp writes columns [hf*D/2, (hf+1)*D/2) of the row
      long long out_row = row_pos;
      if (it.slot >= 0 && row_valid) {
        const int fr = row_pos % P.F, pos = row_pos / P.F;
        const int y = pos / P.Wh, x = pos % P.Wh;
        out_row = (static_cast<long long>(fr) * P.Hh + y) * P.Wh + x;
      }
      uint4* orow = reinterpret_cast<uint4*>(
          P.o + (static_cast<long long>(it.bh) * P.N + (row_valid ? out_row : 0)) * D);
#pragma unroll
      for (int c0 = hf * (D / 2); c0 < (hf + 1) * (D / 2); c0 += 32) {
        uint32_t o32[32];
        tmem_ld32(lane_base + C::kO + c0, o32);
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(o32[e]) * inv_l;
        if (lin) {
          uint32_t l32[32];
          tmem_ld32(lane_base + C::kL + c0, l32);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = fmaf(__uint_as_float(l32[e]), lin_scale, v[e]);
        }
        if (row_valid) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4 wv;
            wv.x = pack_bf16x2(v[8 * u + 0], v[8 * u + 1]);
            wv.y = pack_bf16x2(v[8 * u + 2], v[8 * u + 3]);
            wv.z = pack_bf16x2(v[8 * u + 4], v[8 * u + 5]);
            wv.w = pack_bf16x2(v[8 * u + 6], v[8 * u + 7]);
            orow[c0 / 8 + u] = wv;
          }
        }
      }
      tc_fence_before();
    }
    if (!ok) raise_timeout(P.err, abort_flag);
    // Drain the last G load before the CTA leaves (it has landed already
    // unless a wait above ran out).
    if (g_loader && g_issued > 0 &&
        !mbar_wait(g_full, static_cast<uint32_t>((g_issued - 1) & 1), wait_ns, nullptr))
      atomicOr(P.err, kErrTimeout);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kCols);
  }
}

// One CTA, one thread: wait on a barrier nothing arrives on.
__global__ void debug_wait_kernel(unsigned* err, unsigned long long wait_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
    if (!mbar_wait(smem_u32(&bar), 0, wait_ns, nullptr)) atomicOr(err, kErrTimeout);
  }
}

template <int D, bool HYB>
cudaError_t launch_attn_t(const Ctx& c, const AttnArgs& a, const Params& P) {
  using C = AT<D, HYB>;
  CUtensorMap mk, mv, mkp, mvp;
  const int BH = a.B * a.H;
  if (!make_tmap_bf16_3d(&mk, a.k, BH, a.N, D) || !make_tmap_bf16_3d(&mv, a.v, BH, a.N, D))
    return cudaErrorInvalidValue;
  if (a.Hs > 0) {
    if (!make_tmap_bf16_3d(&mkp, a.kp, a.B * a.Hs, a.N, D) ||
        !make_tmap_bf16_3d(&mvp, a.vp, a.B * a.Hs, a.N, D))
      return cudaErrorInvalidValue;
  } else {
    mkp = mk;
    mvp = mv;
  }
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D, HYB>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const long long items = static_cast<long long>(BH) * P.npairs;
  long long grid = items < c.num_sms ? items : c.num_sms;
  if (grid < 1) grid = 1;
  attn_kernel<D, HYB><<<static_cast<int>(grid), 320, C::kSmem, c.stream>>>(mk, mv, mkp, mvp, P);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const Ctx& c, const AttnArgs& a) {
  Params P;
  P.q = static_cast<const __nv_bfloat16*>(a.q);
  P.qp = static_cast<const __nv_bfloat16*>(a.qp);
  for (int h = 0; h < 256; ++h) P.head_slot[h] = -1;
  if (a.head_slot != nullptr)
    for (int h = 0; h < a.H && h < 256; ++h) P.head_slot[h] = static_cast<short>(a.head_slot[h]);
  P.B = a.B;
  P.H = a.H;
  P.N = a.N;
  P.Hs = a.Hs;
  P.nb = (a.N + 63) / 64;
  P.npairs = (P.nb + 1) / 2;
  P.mode = a.mode;
  P.window = a.window;
  P.F = a.F;
  P.Hh = a.Hh;
  P.Wh = a.Wh;
  P.lists = a.lists;
  P.counts = a.counts;
  P.list_stride = a.list_stride;
  P.Gimg = static_cast<const __nv_bfloat16*>(a.Gimg);
  P.Z = a.Z;
  P.s = a.s;
  P.gate_override = a.gate_override;
  P.drop = a.drop;
  P.rope = a.rope;
  P.eps = a.eps;
  P.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(a.d));
  P.o = static_cast<__nv_bfloat16*>(a.o);
  P.err = c.err;
  P.wait_ns = c.wait_ns;
  const bool hyb = a.Gimg != nullptr;
  if (a.d == 128) return hyb ? launch_attn_t<128, true>(c, a, P) : launch_attn_t<128, false>(c, a, P);
  return hyb ? launch_attn_t<64, true>(c, a, P) : launch_attn_t<64, false>(c, a, P);
}

cudaError_t launch_debug_wait(const Ctx& c) {
  debug_wait_kernel<<<1, 32, 0, c.stream>>>(c.err, c.wait_ns);
  return cudaGetLastError();
}

}  // namespace salad
