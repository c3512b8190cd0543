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
// (M = 128 rows, the full tcgen05 datapath).  Its key blocks are the merged,
// ascending list of the blocks either query block keeps (Top-K), the band of
// blocks its rows' windows touch (ST-SWA) or all blocks (dense), taken two
// at a time: a tile holds 128 keys, so the QK MMA has N = 128 (an M = 128
// tcgen05.mma occupies the tensor pipe for ~64 cycles at any N <= 128).
// A query block that did not keep one of a tile's blocks gets P = 0 there.
//
// Split-K ping-pong.  The item's tiles alternate between two slots, A (even
// tiles) and B (odd tiles), each with its own S and O accumulators in TMEM
// and its own running max and sum; the two partial results are merged once,
// at the end of the item.  The single MMA thread interleaves the slots: while
// the tensor pipe runs slot A's PV(t) and QK(t+2), slot B's softmax runs, and
// the reverse.  Each slot's softmax has four warps, one per TMEM lane
// quarter, one query row per thread: a pass over the tile's two 64-key halves
// finds the row max, a second pass exponentiates (exp2, running max raised
// lazily: O is rescaled only when it grows by more than 2^8) and writes P
// back over S as bf16.  S = Q K^T is an SS MMA (Q from shared memory, TMA-
// loaded, double-buffered across items); O += P V a TS MMA (P from TMEM).
// QK(t+2) is issued right behind PV(t) into the buffer PV(t) reads (tcgen05
// MMAs of one thread execute in issue order).
//
// K tiles, V tiles and the item's G image stream through one ring of stages
// in the order the MMA thread consumes them: K0, K1, then V(t), K(t+2) for
// each tile t, then G.  The linear term s_b * phi(Q) G / (phi(Q) Z + eps) is
// one more SS MMA (A = phi(Q), written over the item's Q buffer by the
// softmax threads once every QK has run; B = the G image) into slot A's S
// columns.  The epilogue merges the slots, adds the linear term and writes
// the rows; each slot writes half of the columns.
//
// Warp roles (320 threads, one CTA per SM, persistent over work items):
//   warp 0      TMA producer: Q (two 64-row boxes per d-slab), K and V
//               tiles (64 x 64 boxes, 128B swizzle), the G image.
//   warp 1      TMEM allocator and the single MMA-issuing thread.
//   warps 2..5  slot A softmax; warp w holds TMEM lane quarter w % 4.
//   warps 6..9  slot B softmax.
// TMEM columns (d = 128): O_A [0,128) O_B [128,256) S_A [256,384)
// S_B [384,512); the linear term lands in S_A.
//
// Barrier discipline: an mbarrier parity wait is only sound when the waiter is
// at most one phase behind.  Every barrier is observed by each of its waiters
// at every phase: in particular each softmax warp waits for its slot's
// previous PV once per tile, rescales its O only then, and only then releases
// the tile.  Every wait is bounded; a wait that runs out raises the device
// error word and the CTA leaves through the common teardown (loads drained,
// MMAs committed, TMEM accesses completed, TMEM freed).
#include "common.cuh"
#include "internal.h"

namespace salad {
namespace {

constexpr int kSlab = 64 * 128;   // one 64-row x 128-byte swizzled slab

template <int D, bool HYB>
struct AT {
  static constexpr int kHalves = D / 64;                 // 128-byte d-slabs per row
  static constexpr int kRowSlab = 128 * 128;             // 128 rows of one d-slab
  static constexpr int kQBuf = kHalves * kRowSlab;       // 128 rows of Q (or phi(Q))
  static constexpr int kStage = kHalves * kRowSlab;      // 128 keys of K or V, or a G image
  static constexpr int kStages = D == 128 ? 4 : 8;
  static constexpr int kGImg = D * D * 2;
  static_assert(kGImg <= kStage, "the G image fills one ring stage");
  static constexpr int kXchg = 2 * 128 * 16;             // per slot and row: m, l, den part
  static constexpr int kBarBytes = 512;
  static constexpr int kSmemUsed = 2 * kQBuf + kStages * kStage + kXchg + kBarBytes;
  static_assert(kSmemUsed <= 227 * 1024, "shared memory budget");
  // At least ~half of the SM's shared memory, so one CTA (and its 512 TMEM
  // columns) occupies each SM.
  static constexpr int kSmem = kSmemUsed > 120 * 1024 ? kSmemUsed : 120 * 1024;
  // TMEM columns.
  __host__ __device__ static constexpr uint32_t o_col(int slot) { return slot ? D : 0; }
  __host__ __device__ static constexpr uint32_t s_col(int slot) { return 2 * D + (slot ? 128 : 0); }
  static constexpr uint32_t kL = 2 * D;        // linear term, D columns over S_A
  static constexpr uint32_t kCols = 512;
  static_assert(2 * D + 256 <= kCols, "TMEM budget");
};

struct Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* qp;
  short head_slot[256];       // slot in the regrouped copies, -1 = frame-major head
  int B, H, N, Hs, nb, npairs;
  int mode, window, F, Hh, Wh;
  // Regrouping inside the loads (kernel instantiation RG): a regrouped head's
  // items and key tiles are rg_pos whole spatial positions, rg_rows =
  // rg_pos * F rows of the 128-row MMA, read from the frame-major tensors.
  int rg_rows, rg_pos;
  // RG: work items of sample b, head h are [b * per_b + head_base[h],
  // b * per_b + head_base[h + 1]).
  int per_b;
  int head_base[257];
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

// The kernel's parameters (six tensor maps and Params) stay within the
// classic 4 KB parameter space.
static_assert(sizeof(Params) + 6 * sizeof(CUtensorMap) <= 4096, "kernel parameter space");

struct Item {
  int bh, b, h, p;
  int ntiles;
  int jlo;                // first key block (band / dense), or key tile (rg)
  const int32_t* list;    // topk entries
  int slot;               // >= 0: regrouped (space-major) head
  bool rg;                // regrouped in the loads: position-aligned rows and key tiles
};

// Query rows of an item (and keys of one of its key tiles).
template <bool RG>
__device__ __forceinline__ int item_rows(const Params& P, const Item& it) {
  if constexpr (RG) return it.rg ? P.rg_rows : 128;
  return 128;
}

template <bool RG>
__device__ __forceinline__ Item make_item(const Params& P, long long w) {
  Item it;
  if constexpr (RG) {
    it.b = static_cast<int>(w / P.per_b);
    const int rem = static_cast<int>(w - static_cast<long long>(it.b) * P.per_b);
    int lo = 0, hi = P.H;   // head_base[lo] <= rem < head_base[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) / 2;
      if (P.head_base[mid] <= rem) lo = mid; else hi = mid;
    }
    it.h = lo;
    it.p = rem - P.head_base[lo];
    it.bh = it.b * P.H + it.h;
  } else {
    it.bh = static_cast<int>(w / P.npairs);
    it.p = static_cast<int>(w % P.npairs);
    it.b = it.bh / P.H;
    it.h = it.bh % P.H;
  }
  it.slot = P.head_slot[it.h];
  it.rg = RG && it.slot >= 0;
  it.list = nullptr;
  it.jlo = 0;
  if (P.mode == kModeTopk) {
    it.list = P.lists + w * static_cast<long long>(P.list_stride);
    it.ntiles = P.counts[w];
  } else if (P.mode == kModeDense) {
    it.ntiles = P.nb;
  } else {
    const int rows = item_rows<RG>(P, it);
    const int r0 = it.p * rows;
    const int r1 = min(P.N, r0 + rows) - 1;
    const int lo = max(0, r0 - P.window);
    const int hi = min(P.N - 1, r1 + P.window);
    if (RG && it.rg) {
      // Key tiles of rg_rows keys (whole positions), two half-tiles each.
      it.jlo = lo / rows;
      it.ntiles = 2 * (hi / rows - it.jlo + 1);
    } else {
      it.jlo = lo / 64;
      it.ntiles = hi / 64 - it.jlo + 1;
    }
  }
  return it;
}

// Whether sample b keeps its linear branch (post-training branch dropping:
// the branch is skipped when the gate value is below the threshold).
__device__ __forceinline__ bool lin_on(const Params& P, int b) {
  const float g = P.s != nullptr ? __ldg(P.s + b) : P.gate_override;
  return !(g < P.drop);
}

// Entry t of the item's key-block list: j | mask << 16 (mask bit 0: the
// first query block of the pair keeps block j, bit 1: the second); 0 past
// the end.  Band and dense items keep every block of their range for both.
__device__ __forceinline__ int list_entry(const Item& it, int t, int mode) {
  if (t >= it.ntiles) return 0;
  if (mode == kModeTopk) return __ldg(it.list + t);
  return (it.jlo + t) | (3 << 16);
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

// Zero [base, base + bytes) (a multiple of 16) with the whole CTA, then order
// these generic-proxy writes before later async-proxy accesses (TMA, MMA).
// Out of line: inlined, its loop costs the kernel a register spill.
__device__ __noinline__ void zero_smem(unsigned char* base, int bytes) {
  uint4* z = reinterpret_cast<uint4*>(base);
  for (int i = threadIdx.x; i < bytes / 16; i += blockDim.x) z[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
}

// RG: regrouped ST-SWA heads are read inside the loads (position-aligned
// items and key tiles, V staged [d-slab][128 rows]); a separate instantiation
// so that the default kernel carries none of it.
template <int D, bool HYB, bool RG>
__global__ void __launch_bounds__(320, 1) attn_kernel(const __grid_constant__ CUtensorMap mq,
                                                      const __grid_constant__ CUtensorMap mk,
                                                      const __grid_constant__ CUtensorMap mv,
                                                      const __grid_constant__ CUtensorMap mqp,
                                                      const __grid_constant__ CUtensorMap mkp,
                                                      const __grid_constant__ CUtensorMap mvp,
                                                      const __grid_constant__ Params P) {
  using C = AT<D, HYB>;
  constexpr int NS = C::kStages;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // The layout below assumes the declared alignment; refuse to run without it.
  if (reinterpret_cast<uintptr_t>(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(P.err, kErrLayout);
    return;
  }
  unsigned char* qbuf = smem_raw;                          // [2][d-slab][128 rows x 128 B]
  unsigned char* ring = qbuf + 2 * C::kQBuf;               // [NS] stages
  float4* xchg = reinterpret_cast<float4*>(ring + NS * C::kStage);  // [slot][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<unsigned char*>(xchg) + C::kXchg);
  // bars: full[NS] empty[NS] q_full[2] q_empty[2] s_full[2] p_full[2] o_done[2] q_free
  //       phiq_ready lin_done x_bar epi_done drain
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * NS + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  static_assert((2 * NS + 16) * 8 + 8 <= C::kBarBytes, "barrier region");

  auto full = [&](int i) { return smem_u32(bars + i); };
  auto empty = [&](int i) { return smem_u32(bars + NS + i); };
  auto q_full = [&](int i) { return smem_u32(bars + 2 * NS + i); };
  auto q_empty = [&](int i) { return smem_u32(bars + 2 * NS + 2 + i); };
  auto s_full = [&](int i) { return smem_u32(bars + 2 * NS + 4 + i); };
  auto p_full = [&](int i) { return smem_u32(bars + 2 * NS + 6 + i); };
  auto o_done = [&](int i) { return smem_u32(bars + 2 * NS + 8 + i); };
  const uint32_t q_free = smem_u32(bars + 2 * NS + 10);
  const uint32_t phiq_ready = smem_u32(bars + 2 * NS + 11);
  const uint32_t lin_done = smem_u32(bars + 2 * NS + 12);
  const uint32_t x_bar = smem_u32(bars + 2 * NS + 13);
  const uint32_t epi_done = smem_u32(bars + 2 * NS + 14);
  const uint32_t drain = smem_u32(bars + 2 * NS + 15);
  auto q_addr = [&](int b) { return smem_u32(qbuf + b * C::kQBuf); };
  auto st_addr = [&](long long c) { return smem_u32(ring + static_cast<int>(c % NS) * C::kStage); };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long total = RG ? static_cast<long long>(P.B) * P.per_b
                             : static_cast<long long>(P.B) * P.H * P.npairs;
  const unsigned long long wait_ns = P.wait_ns;

  // RG: position-aligned items fill rg_rows < 128 rows of Q and of each K/V
  // tile; the rows past them are read by the MMAs (their P columns are 0,
  // their output rows are not written) and must hold finite values: zero the
  // Q buffers and the ring once, before any load lands.
  if constexpr (RG) zero_smem(qbuf, 2 * C::kQBuf + NS * C::kStage);

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(full(i), 1);
      mbar_init(empty(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full(i), 1);
      mbar_init(q_empty(i), 1);
      mbar_init(s_full(i), 1);
      mbar_init(p_full(i), 4);   // the slot's four softmax warps
      mbar_init(o_done(i), 1);
    }
    mbar_init(q_free, 1);
    mbar_init(phiq_ready, 8);    // every softmax warp has written its part of phi(Q)
    mbar_init(lin_done, 1);
    mbar_init(x_bar, 8);         // every softmax warp has posted its row's m, l and den part
    mbar_init(epi_done, 8);      // every softmax warp has finished the item's epilogue
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&mq);
    tma_prefetch_map(&mk);
    tma_prefetch_map(&mv);
    if (P.Hs > 0) {
      tma_prefetch_map(&mqp);
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
      long long sc = 0;   // ring stages filled so far
      uint32_t qc = 0;    // items started (Q buffer qc & 1)
      uint32_t q_issued = 0;   // Q loads issued (drained at the end)
      bool ok = true;
      // Q rows of item number j (two 64-row boxes per d-slab; rows past N
      // read 0) into buffer j & 1, once the item two before it has freed it.
      auto load_q = [&](long long w, uint32_t j) -> bool {
        const Item it = make_item<RG>(P, w);
        const CUtensorMap* qm = it.slot >= 0 ? &mqp : &mq;
        const int z = it.slot >= 0 ? it.b * P.Hs + it.slot : it.bh;
        const int qb = static_cast<int>(j & 1);
        if (j >= 2 && !mbar_wait(q_empty(qb), ((j - 2) / 2) & 1, wait_ns, abort_flag)) return false;
        if (RG && it.rg) {
          // rg_pos whole positions, all F frames each, in space-major order:
          // one (64 channels, F, rg_pos) box per d-slab of the frame-major Q.
          mbar_arrive_expect_tx(q_full(qb), (D / 64) * P.rg_rows * 128);
#pragma unroll
          for (int hh = 0; hh < D / 64; ++hh)
            tma_load_4d(q_addr(qb) + hh * C::kRowSlab, qm, q_full(qb), hh * 64, 0,
                        it.p * P.rg_pos, it.bh);
          q_issued = j + 1;
          return true;
        }
        mbar_arrive_expect_tx(q_full(qb), C::kQBuf);
#pragma unroll
        for (int hh = 0; hh < D / 64; ++hh)
#pragma unroll
          for (int rb = 0; rb < 2; ++rb)
            tma_load_3d(q_addr(qb) + hh * C::kRowSlab + rb * kSlab, qm, q_full(qb), hh * 64,
                        it.p * 128 + rb * 64, z);
        q_issued = j + 1;
        return true;
      };
      if (static_cast<long long>(blockIdx.x) < total) ok = load_q(blockIdx.x, 0);
      for (long long w = blockIdx.x; w < total && ok; w += gridDim.x, ++qc) {
        const Item it = make_item<RG>(P, w);
        const CUtensorMap* km = it.slot >= 0 ? &mkp : &mk;
        const CUtensorMap* vm = it.slot >= 0 ? &mvp : &mv;
        const int z = it.slot >= 0 ? it.b * P.Hs + it.slot : it.bh;
        const int T = (it.ntiles + 1) / 2;
        const bool lin = HYB && lin_on(P, it.b);
        // The item's loads in the MMA thread's order: K0, K1, then V(t) and
        // K(t+2) for each tile t, then the G image.
        auto push = [&](int kind, int t) -> bool {
          const int si = static_cast<int>(sc % NS);
          const long long n = sc / NS;
          if (n > 0 && !mbar_wait(empty(si), static_cast<uint32_t>((n - 1) & 1), wait_ns, abort_flag))
            return false;
          const uint32_t dst = st_addr(sc);
          ++sc;
          if (kind == 2) {
            mbar_arrive_expect_tx(full(si), C::kGImg);
            bulk_load(dst, P.Gimg + static_cast<long long>(it.bh) * D * D, C::kGImg, full(si));
            return true;
          }
          if (RG && it.rg) {
            // Key tile jlo + t: rg_pos whole positions of the frame-major K
            // or V, [d-slab][rg_rows rows] like every tile of this kernel.
            mbar_arrive_expect_tx(full(si), (D / 64) * P.rg_rows * 128);
#pragma unroll
            for (int hh = 0; hh < D / 64; ++hh)
              tma_load_4d(dst + hh * C::kRowSlab, kind == 0 ? km : vm, full(si), hh * 64, 0,
                          (it.jlo + t) * P.rg_pos, it.bh);
            return true;
          }
          const int nblk = (2 * t + 1 < it.ntiles) ? 2 : 1;
          mbar_arrive_expect_tx(full(si), nblk * (D / 64) * kSlab);
          for (int x = 0; x < nblk; ++x) {
            const int j = list_entry(it, 2 * t + x, P.mode) & 0xFFFF;
#pragma unroll
            for (int hh = 0; hh < D / 64; ++hh) {
              if (kind == 0 || RG)   // K (and RG's V): [d-slab][128 rows]; block x from row 64x
                tma_load_3d(dst + hh * C::kRowSlab + x * kSlab, kind == 0 ? km : vm, full(si),
                            hh * 64, j * 64, z);
              else                   // V: [block][d-slab][64 rows]
                tma_load_3d(dst + x * (D / 64) * kSlab + hh * kSlab, vm, full(si), hh * 64, j * 64, z);
            }
          }
          return true;
        };
        ok = push(0, 0) && (T < 2 || push(0, 1));
        // The next item's Q, a whole item ahead: its buffer was the previous
        // item's, free once that item's MMAs have run (which needs nothing
        // more from this thread).
        if (ok && w + gridDim.x < total) ok = load_q(w + gridDim.x, qc + 1);
        for (int t = 0; t < T && ok; ++t) ok = push(1, t) && (t + 2 >= T || push(0, t + 2));
        if (ok && lin) ok = push(2, 0);
      }
      if (!ok) raise_timeout(P.err, abort_flag);
      // Drain every issued load before leaving.
      for (int i = 0; i < NS && i < sc; ++i) {
        const long long last = i + ((sc - 1 - i) / NS) * NS;
        if (!mbar_wait(full(i), static_cast<uint32_t>((last / NS) & 1), wait_ns, nullptr))
          atomicOr(P.err, kErrTimeout);
      }
      for (uint32_t b = 0; b < 2 && b < q_issued; ++b) {
        const uint32_t uses = (q_issued - b + 1) / 2;   // Q loads into buffer b
        if (!mbar_wait(q_full(b), (uses - 1) & 1, wait_ns, nullptr)) atomicOr(P.err, kErrTimeout);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ================================================= MMA issuer
      // Descriptors are built once per operand and advanced by constant
      // offsets per K-step (shared addresses stay below 2^18, so the 14-bit
      // address field never carries); the ring position is kept as a stage
      // index and a phase bit.  This thread shares its sub-partition with two
      // softmax warps, so every instruction it saves is issue time the tensor
      // pipe does not wait for.
      constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
      constexpr uint32_t idesc_lin = idesc_bf16(128, D, false, false);
      const uint32_t ring_base = smem_u32(ring);
      int stage = 0;
      uint32_t sphase = 0;
      uint32_t ic = 0, lc = 0, pf[2] = {0, 0};
      bool ok = true;
      auto wait_stage = [&]() -> bool { return mbar_wait(full(stage), sphase, wait_ns, abort_flag); };
      auto next_stage = [&]() {
        if (++stage == NS) {
          stage = 0;
          sphase ^= 1u;
        }
      };
      // S_slot = Q K(t)^T from the K tile in the current stage.
      auto issue_qk = [&](uint64_t qdesc, int slot) {
        const uint64_t kdesc = sdesc_sw128(ring_base + stage * C::kStage, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t off = static_cast<uint64_t>(((ks / 4) * C::kRowSlab + (ks % 4) * 32) >> 4);
          mma_ss(tmem + C::s_col(slot), qdesc + off, kdesc + off, idesc_qk, ks > 0 ? 1u : 0u);
        }
        mma_commit(empty(stage));
        mma_commit(s_full(slot));
        next_stage();
      };
      for (long long w = blockIdx.x; w < total && ok; w += gridDim.x, ++ic) {
        const Item it = make_item<RG>(P, w);
        const int T = (it.ntiles + 1) / 2;
        const bool lin = HYB && lin_on(P, it.b);
        const int qb = static_cast<int>(ic & 1);
        const uint64_t qdesc = sdesc_sw128(q_addr(qb), 16, 1024);
        // The previous item's epilogue has read O, S and the linear term.
        if (ic > 0 && !mbar_wait(epi_done, (ic - 1) & 1, wait_ns, abort_flag)) { ok = false; break; }
        if (!mbar_wait(q_full(qb), (ic / 2) & 1, wait_ns, abort_flag)) { ok = false; break; }
        tc_fence_after();
        for (int t = 0; t < 2 && t < T; ++t) {
          if (!wait_stage()) { ok = false; break; }
          tc_fence_after();
          issue_qk(qdesc, t);
        }
        if (!ok) break;
        if (T <= 2) mma_commit(q_free);   // every QK of the item is issued
        for (int t = 0; t < T; ++t) {
          const int slot = t & 1;
          if (!mbar_wait(p_full(slot), pf[slot] & 1, wait_ns, abort_flag)) { ok = false; break; }
          ++pf[slot];
          if (!wait_stage()) { ok = false; break; }
          tc_fence_after();
          // V (MN-major): d-slabs kSlab apart ([block][d-slab][64 rows]), or,
          // in RG, kRowSlab apart ([d-slab][128 rows]).
          const uint64_t vdesc =
              sdesc_sw128(ring_base + stage * C::kStage, RG ? C::kRowSlab : kSlab, 1024);
          const uint32_t sa = tmem + C::s_col(slot), oa = tmem + C::o_col(slot);
          const uint32_t acc0 = t >= 2 ? 1u : 0u;
          if (2 * t + 1 < it.ntiles) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {   // K-steps: 16 keys each
              const uint64_t off = static_cast<uint64_t>(
                  (RG ? ks * 2048 : (ks / 4) * (D / 64) * kSlab + (ks % 4) * 2048) >> 4);
              mma_ts(oa, sa + ks * 8, vdesc + off, idesc_pv, ks > 0 ? 1u : acc0);
            }
          } else {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {   // a single 64-key block
              const uint64_t off = static_cast<uint64_t>(((ks % 4) * 2048) >> 4);
              mma_ts(oa, sa + ks * 8, vdesc + off, idesc_pv, ks > 0 ? 1u : acc0);
            }
          }
          mma_commit(empty(stage));
          mma_commit(o_done(slot));
          next_stage();
          if (t + 2 < T) {
            if (!wait_stage()) { ok = false; break; }
            tc_fence_after();
            issue_qk(qdesc, slot);   // same S buffer: runs after this PV in issue order
            if (t + 3 == T) mma_commit(q_free);   // that was the item's last QK
          }
        }
        if (!ok) break;
        if (lin) {
          // Linear term into S_A (every S of the item has been read):
          // L = phi(Q) G, A = phi(Q) over the Q buffer, B = the G image.
          if (!mbar_wait(phiq_ready, lc & 1, wait_ns, abort_flag)) { ok = false; break; }
          if (!wait_stage()) { ok = false; break; }
          tc_fence_after();
          const uint64_t gdesc = sdesc_sw128(ring_base + stage * C::kStage, 16, 1024);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint64_t qoff = static_cast<uint64_t>(((ks / 4) * C::kRowSlab + (ks % 4) * 32) >> 4);
            const uint64_t goff = static_cast<uint64_t>(((ks / 4) * (D * 128) + (ks % 4) * 32) >> 4);
            mma_ss(tmem + C::kL, qdesc + qoff, gdesc + goff, idesc_lin, ks > 0 ? 1u : 0u);
          }
          mma_commit(empty(stage));
          mma_commit(lin_done);
          next_stage();
          ++lc;
        }
        mma_commit(q_empty(qb));   // the item's Q buffer is free once these MMAs ran
      }
      if (!ok) raise_timeout(P.err, abort_flag);
      mma_commit(drain);
      if (!mbar_wait(drain, 0, wait_ns, nullptr)) atomicOr(P.err, kErrTimeout);
    }
  } else {
    // ================================================= softmax + epilogue
    // Slot A = warps 2..5 (even tiles), slot B = warps 6..9 (odd tiles); one
    // query row per thread, warp w on TMEM lane quarter w % 4.
    const int slot = (warp - 2) / 4;
    const int quarter = warp % 4;
    const int r = quarter * 32 + lane;            // row within the pair (TMEM lane)
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const int half_bit = r >= 64 ? 2 : 1;         // the row's query block inside the pair
    const float c2 = P.scale_log2;
    constexpr int HC = D / 16;                    // 16-byte chunks in half a row of Q
    uint32_t ic = 0, lc = 0, sf = 0;
    long long pv_base = 0;                        // this slot's PVs completed before this item
    bool ok = true;
    for (long long w = blockIdx.x; w < total && ok; w += gridDim.x, ++ic) {
      const Item it = make_item<RG>(P, w);
      const int rows = item_rows<RG>(P, it);
      const int row_pos = it.p * rows + r;       // position in the head's (possibly regrouped) order
      const bool row_valid = (!RG || r < rows) && row_pos < P.N;
      const int T = (it.ntiles + 1) / 2;
      const int nt = (T - slot + 1) / 2;          // this slot's tiles: t = slot, slot + 2, ...
      const bool lin = HYB && lin_on(P, it.b);   // this item adds the linear term
      const int qb = static_cast<int>(ic & 1);
      // The item's Q rows have landed (observed every item, in order).
      if (!__all_sync(0xffffffffu, mbar_wait(q_full(qb), (ic / 2) & 1, wait_ns, abort_flag))) {
        ok = false;
        break;
      }
      // Chunk c (8 columns) of this thread's row of the item's Q buffer.
      unsigned char* qrow = qbuf + qb * C::kQBuf + r * 128;
      auto q_chunk = [&](int c) -> uint4* {
        return reinterpret_cast<uint4*>(qrow + (c / 8) * C::kRowSlab + ((c % 8) ^ (r % 8)) * 16);
      };
      // This slot's half of phi(q) . Z.
      float den_part = 0.f;
      if (lin) {
        const float* zrow = P.Z + static_cast<long long>(it.bh) * D;
#pragma unroll
        for (int cc = 0; cc < HC; ++cc) {
          const int c = slot * HC + cc;
          const uint4 v = *q_chunk(c);
          const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 fz = unpack_bf16x2(relu_bf16x2(wv[e]));
            den_part = fmaf(fz.x, __ldg(zrow + 8 * c + 2 * e), den_part);
            den_part = fmaf(fz.y, __ldg(zrow + 8 * c + 2 * e + 1), den_part);
          }
        }
      }

      // ---- softmax over this slot's tiles (128 keys each)
      float m = -INFINITY;   // running max of the row in the exp2 domain
      float l = 0.f;         // row sum of exp2(S*c - m) over this slot's keys
      int e0 = list_entry(it, 2 * slot, P.mode), e1 = list_entry(it, 2 * slot + 1, P.mode);
      const uint32_t sbuf = lane_base + C::s_col(slot);
      for (int k = 0; k < nt; ++k) {
        const int t = slot + 2 * k;
        // The next tile's list entries travel while this one is processed.
        const int e0n = list_entry(it, 2 * t + 4, P.mode), e1n = list_entry(it, 2 * t + 5, P.mode);
        // Waits and TMEM accesses are warp-collective: every decision that
        // guards one is made uniform across the warp first.
        if (!__all_sync(0xffffffffu, mbar_wait(s_full(slot), sf & 1, wait_ns, abort_flag))) {
          ok = false;
          break;
        }
        ++sf;
        tc_fence_after();
        // The tile's two key blocks; inside each, the row's valid keys form
        // one contiguous range [lo, hi] of the block's 64 columns.
        const int mk[2] = {e0 >> 16, e1 >> 16};
        // First key of each 64-column half: block j at 64 j, or, on a
        // position-aligned tile (RG), rg_rows (jlo + t) + 64 x; kend is one
        // past the tile's last key.
        int kb[2] = {(e0 & 0xFFFF) * 64, (e1 & 0xFFFF) * 64};
        int kend = P.N;
        if (RG && it.rg) {
          kb[0] = rows * (it.jlo + t);
          kb[1] = kb[0] + 64;
          kend = min(P.N, kb[0] + rows);
        }
        int lo[2], hi[2];
        bool live[2], any[2], part[2];
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          lo[x] = 0;
          hi[x] = min(63, kend - 1 - kb[x]);
          if (P.mode == kModeBand) {
            lo[x] = max(lo[x], row_pos - P.window - kb[x]);
            hi[x] = min(hi[x], row_pos + P.window - kb[x]);
          }
          live[x] = row_valid && (mk[x] & half_bit) && lo[x] <= hi[x];
          any[x] = __any_sync(0xffffffffu, live[x]);
          part[x] = any[x] && __any_sync(0xffffffffu, !(live[x] && lo[x] == 0 && hi[x] == 63));
        }
        // Pass 1: the row max over both halves (keys outside the row's range
        // count as -inf; only halves with a partial or dead row pay for it).
        float pm = -INFINITY;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          if (!any[x]) continue;
          uint32_t s64[64];
          tmem_ld64(sbuf + 64 * x, s64);
          float sv[64];
#pragma unroll
          for (int c = 0; c < 64; ++c) sv[c] = __uint_as_float(s64[c]);
          if (part[x]) {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              sv[c] = (live[x] && c >= lo[x] && c <= hi[x]) ? sv[c] : -INFINITY;
          }
          pm = fmaxf(pm, max64(sv));
        }
        pm *= c2;                    // c2 > 0: max of scaled = scaled max
        float f = 1.0f;              // factor O must be rescaled by before this PV
        if (pm > m + 8.0f) {
          f = (m == -INFINITY) ? 1.0f : ex2(m - pm);
          l *= f;
          m = pm;
        }
        // A row with no valid key so far keeps m = -inf: use 0 as the offset
        // so its -inf scores give exp2(-inf) = 0, never NaN.
        const float nm = (m == -INFINITY) ? 0.0f : -m;
        // Pass 2: exponentiate each half; P (bf16 pairs) goes over the first
        // 64 columns of S (half x -> columns 32x .. 32x+31, already read).
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          uint32_t pk[32];
          if (any[x]) {
            uint32_t s64[64];
            tmem_ld64(sbuf + 64 * x, s64);
            float sv[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) sv[c] = __uint_as_float(s64[c]);
            if (part[x]) {
#pragma unroll
              for (int c = 0; c < 64; ++c)
                sv[c] = (live[x] && c >= lo[x] && c <= hi[x]) ? sv[c] : -INFINITY;
            }
            float ls0 = 0.f, ls1 = 0.f, ls2 = 0.f, ls3 = 0.f;
#pragma unroll
            for (int c = 0; c < 64; c += 4) {
              const float p0 = ex2(fmaf(sv[c], c2, nm)), p1 = ex2(fmaf(sv[c + 1], c2, nm));
              const float p2 = ex2(fmaf(sv[c + 2], c2, nm)), p3 = ex2(fmaf(sv[c + 3], c2, nm));
              pk[c / 2] = pack_bf16x2(p0, p1);
              pk[c / 2 + 1] = pack_bf16x2(p2, p3);
              ls0 += p0;
              ls1 += p1;
              ls2 += p2;
              ls3 += p3;
            }
            l += (ls0 + ls1) + (ls2 + ls3);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) pk[e] = 0u;
          }
          tmem_st32(sbuf + 32 * x, pk);
        }
        // Observe this slot's previous PV: every warp observes every PV of
        // its slot in order, so each parity wait is at most one phase behind.
        if (k >= 1) {
          const long long g = pv_base + k - 1;
          if (!__all_sync(0xffffffffu,
                          mbar_wait(o_done(slot), static_cast<uint32_t>(g & 1), wait_ns, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        if (__any_sync(0xffffffffu, f != 1.0f)) {
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o32[32];
            tmem_ld32(lane_base + C::o_col(slot) + c0, o32);
#pragma unroll
            for (int e = 0; e < 32; ++e) o32[e] = __float_as_uint(__uint_as_float(o32[e]) * f);
            tmem_st32(lane_base + C::o_col(slot) + c0, o32);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(slot));
        e0 = e0n;
        e1 = e1n;
      }
      if (!ok) break;
      if (nt > 0) {
        // This slot's last PV has landed.
        const long long g = pv_base + nt - 1;
        if (!__all_sync(0xffffffffu,
                        mbar_wait(o_done(slot), static_cast<uint32_t>(g & 1), wait_ns, abort_flag))) {
          ok = false;
          break;
        }
        pv_base += nt;
      }
      // ---- every QK of the item has run: phi(Q) (rotated with the 3-D
      // rotary encoding when on) over the Q buffer, this slot's half.
      if (!__all_sync(0xffffffffu, mbar_wait(q_free, ic & 1, wait_ns, abort_flag))) {
        ok = false;
        break;
      }
      if (lin) {
        const bool rope_on = P.rope.on && row_valid;
        int rf = 0, ry = 0, rx = 0;
        if (rope_on) {
          int tok = row_pos;   // frame-major index of the row's token
          if (it.slot >= 0) tok = (row_pos % P.F) * (P.Hh * P.Wh) + row_pos / P.F;
          const int plane = P.rope.Hh * P.rope.Wh;
          rf = tok / plane;
          ry = (tok / P.rope.Wh) % P.rope.Hh;
          rx = tok % P.rope.Wh;
        }
#pragma unroll
        for (int cc = 0; cc < HC; ++cc) {
          const int c = slot * HC + cc;
          uint4* pq = q_chunk(c);
          const uint4 v = *pq;
          uint32_t wv[4] = {relu_bf16x2(v.x), relu_bf16x2(v.y), relu_bf16x2(v.z), relu_bf16x2(v.w)};
          if (rope_on) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 cs = rope_cs(P.rope, P.rope.theta, 4 * c + e, rf, ry, rx);
              const float2 a = unpack_bf16x2(wv[e]);
              wv[e] = pack_bf16x2(a.x * cs.x - a.y * cs.y, a.x * cs.y + a.y * cs.x);
            }
          }
          *pq = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
        fence_proxy_async_smem();   // generic-proxy writes -> the MMA's operand reads
        __syncwarp();
        if (lane == 0) mbar_arrive(phiq_ready);
      }
      // ---- merge the two slots' partial results for this row
      xchg[slot * 128 + r] = make_float4(m, l, den_part, 0.f);
      __syncwarp();
      if (lane == 0) mbar_arrive(x_bar);
      if (!__all_sync(0xffffffffu, mbar_wait(x_bar, ic & 1, wait_ns, abort_flag))) {
        ok = false;
        break;
      }
      const float4 ot = xchg[(1 - slot) * 128 + r];
      const float mA = slot ? ot.x : m, mB = slot ? m : ot.x;
      const float lA = slot ? ot.y : l, lB = slot ? l : ot.y;
      const float dA = slot ? ot.z : den_part, dB = slot ? den_part : ot.z;
      const float M = fmaxf(mA, mB);
      const float fA = (mA == -INFINITY) ? 0.0f : ex2(mA - M);
      const float fB = (mB == -INFINITY) ? 0.0f : ex2(mB - M);
      const float Lsum = lA * fA + lB * fB;
      const float inv_l = Lsum > 0.f ? 1.0f / Lsum : 0.0f;
      float lin_scale = 0.f;
      if (lin) {
        const float gate = P.s != nullptr ? __ldg(P.s + it.b) : P.gate_override;
        const float dd = (dA + dB) + P.eps;
        lin_scale = dd > 0.f ? gate / dd : 0.f;
        if (!__all_sync(0xffffffffu, mbar_wait(lin_done, lc & 1, wait_ns, abort_flag))) {
          ok = false;
          break;
        }
        ++lc;
      }
      tc_fence_after();
      // ---- epilogue: this slot writes columns [slot*D/2, (slot+1)*D/2) of the row
      long long out_row = row_pos;
      if (it.slot >= 0 && row_valid) {
        const int fr = row_pos % P.F, pos = row_pos / P.F;
        const int y = pos / P.Wh, x = pos % P.Wh;
        out_row = (static_cast<long long>(fr) * P.Hh + y) * P.Wh + x;
      }
      uint4* orow = reinterpret_cast<uint4*>(
          P.o + (static_cast<long long>(it.bh) * P.N + (row_valid ? out_row : 0)) * D + slot * (D / 2));
      const bool has_b = T > 1;                 // slot B ran at least one tile
#pragma unroll
      for (int c0 = 0; c0 < D / 2; c0 += 32) {
        const uint32_t col = slot * (D / 2) + c0;
        uint32_t o32[32];
        float v[32];
        tmem_ld32(lane_base + C::o_col(0) + col, o32);
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(o32[e]) * fA;
        if (has_b) {
          tmem_ld32(lane_base + C::o_col(1) + col, o32);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = fmaf(__uint_as_float(o32[e]), fB, v[e]);
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] *= inv_l;
        if (lin) {
          tmem_ld32(lane_base + C::kL + col, o32);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = fmaf(__uint_as_float(o32[e]), lin_scale, v[e]);
        }
        if (row_valid) {
#pragma unroll
          for (int u4 = 0; u4 < 4; ++u4) {
            uint4 wv;
            wv.x = pack_bf16x2(v[8 * u4 + 0], v[8 * u4 + 1]);
            wv.y = pack_bf16x2(v[8 * u4 + 2], v[8 * u4 + 3]);
            wv.z = pack_bf16x2(v[8 * u4 + 4], v[8 * u4 + 5]);
            wv.w = pack_bf16x2(v[8 * u4 + 6], v[8 * u4 + 7]);
            orow[c0 / 8 + u4] = wv;
          }
        }
      }
      // This warp is done with O, S and the linear term of the item.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(epi_done);
    }
    if (!ok) raise_timeout(P.err, abort_flag);
    // No TMEM access of this warp may be in flight at the teardown.
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    tmem_st_wait();
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

template <int D, bool HYB, bool RG>
cudaError_t launch_attn_t(const Ctx& c, const AttnArgs& a, const Params& P) {
  using C = AT<D, HYB>;
  CUtensorMap mq, mk, mv, mqp, mkp, mvp;
  const int BH = a.B * a.H;
  if (!make_tmap_bf16_3d(&mq, a.q, BH, a.N, D) || !make_tmap_bf16_3d(&mk, a.k, BH, a.N, D) ||
      !make_tmap_bf16_3d(&mv, a.v, BH, a.N, D))
    return cudaErrorInvalidValue;
  if (RG) {
    // Regrouped heads read in the loads: (channel, frame, position, head)
    // views of the frame-major tensors, one box = rg_pos whole positions.
    const int npos = a.N / a.F;
    if (!make_tmap_bf16_regroup(&mqp, a.q, BH, a.F, npos, D, P.rg_pos) ||
        !make_tmap_bf16_regroup(&mkp, a.k, BH, a.F, npos, D, P.rg_pos) ||
        !make_tmap_bf16_regroup(&mvp, a.v, BH, a.F, npos, D, P.rg_pos))
      return cudaErrorInvalidValue;
  } else if (a.Hs > 0) {
    if (!make_tmap_bf16_3d(&mqp, a.qp, a.B * a.Hs, a.N, D) ||
        !make_tmap_bf16_3d(&mkp, a.kp, a.B * a.Hs, a.N, D) ||
        !make_tmap_bf16_3d(&mvp, a.vp, a.B * a.Hs, a.N, D))
      return cudaErrorInvalidValue;
  } else {
    mqp = mq;
    mkp = mk;
    mvp = mv;
  }
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D, HYB, RG>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const long long items = RG ? static_cast<long long>(a.B) * P.per_b
                             : static_cast<long long>(BH) * P.npairs;
  long long grid = items < c.num_sms ? items : c.num_sms;
  if (grid < 1) grid = 1;
  attn_kernel<D, HYB, RG><<<static_cast<int>(grid), 320, C::kSmem, c.stream>>>(mq, mk, mv, mqp, mkp,
                                                                             mvp, P);
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
  // Regrouping inside the loads: items of rg_pos whole positions for the
  // regrouped heads, 128-row pairs of query blocks for the others.
  const bool rg = a.mode == kModeBand && a.Hs > 0 && a.regroup_rows > 0 && a.head_slot != nullptr;
  P.rg_pos = rg ? a.regroup_rows / a.F : 0;
  P.rg_rows = P.rg_pos * a.F;
  P.head_base[0] = 0;
  for (int h = 0; h < a.H; ++h) {
    const int n = rg && a.head_slot[h] >= 0 ? (a.N / a.F + P.rg_pos - 1) / P.rg_pos : P.npairs;
    P.head_base[h + 1] = P.head_base[h] + n;
  }
  P.per_b = P.head_base[a.H];
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
  if (rg) {
    if (P.rg_pos < 1) return cudaErrorInvalidValue;
    if (a.d == 128)
      return hyb ? launch_attn_t<128, true, true>(c, a, P) : launch_attn_t<128, false, true>(c, a, P);
    return hyb ? launch_attn_t<64, true, true>(c, a, P) : launch_attn_t<64, false, true>(c, a, P);
  }
  if (a.d == 128)
    return hyb ? launch_attn_t<128, true, false>(c, a, P) : launch_attn_t<128, false, false>(c, a, P);
  return hyb ? launch_attn_t<64, true, false>(c, a, P) : launch_attn_t<64, false, false>(c, a, P);
}

cudaError_t launch_debug_wait(const Ctx& c) {
  debug_wait_kernel<<<1, 32, 0, c.stream>>>(c.err, c.wait_ns);
  return cudaGetLastError();
}

}  // namespace salad
