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
// 64-key tile:  S = Q K^T  (A = Q from TMEM, B = K tile from smem, N = 64)
// then P = exp2(S*c - m) written back to TMEM as bf16 and O += P V
// (A = P from TMEM, B = V tile from smem, MN-major).  Only K and V tiles are
// read from shared memory.  Rows whose query block did not keep a tile get
// P = 0 for it.  Online softmax with a lazily raised running max (the O row
// is rescaled only when the max grows by more than 2^8).
//
// Barrier discipline: an mbarrier parity wait is only sound when the waiter is
// at most one phase behind.  Every barrier here is therefore observed by each
// of its waiters at every phase: in particular each softmax warp waits for
// PV(t-1) once per tile (after computing and storing P(t), so the wait
// overlaps its own work), rescales O only then, and only then releases tile t.
//
// Warp roles (192 threads, one CTA per SM, persistent over work items):
//   warp 0      TMA producer: K and V tiles (64 x d, 128B swizzle) into a
//               ring of stages.
//   warp 1      TMEM allocator and the single MMA-issuing thread.
//   warps 2..5  one query row per thread: Q (and relu(Q)) into TMEM, softmax
//               per tile, and the epilogue (normalise, add the gated linear
//               term, write bf16 rows; ST-SWA rows go back to frame-major).
// Every wait is bounded; a wait that runs out raises the device error word
// and the CTA leaves through the common teardown (loads drained, MMAs
// committed, TMEM freed).
#include "common.cuh"
#include "internal.h"

namespace salad {

namespace {

constexpr int kSlab = 64 * 128;

template <int D, bool HYB>
struct AT {
  static constexpr int kStages = (D == 128) ? 4 : 6;
  static constexpr int kTile = (D / 64) * kSlab;
  static constexpr int kStage = 2 * kTile;
  static constexpr int kImg = HYB ? D * D * 2 : 0;
  static constexpr int kZ = HYB ? D * 4 : 0;
  static constexpr int kBarBytes = 512;
  static constexpr int kSmemUsed = 1024 + kStages * kStage + 2 * kImg + kZ + kBarBytes;
  // At least ~half of the SM's shared memory, so one CTA (and its 512 TMEM
  // columns) occupies each SM.
  static constexpr int kSmem = kSmemUsed > 120 * 1024 ? kSmemUsed : 120 * 1024;
  // TMEM columns.
  static constexpr uint32_t kO = 0;
  static constexpr uint32_t kS = D;              // two 64-column S/P buffers
  static constexpr uint32_t kQ = D + 128;        // Q as A operand (D/2 columns)
  static constexpr uint32_t kPQ = kQ + D / 2;    // relu(Q) as A operand
  static constexpr uint32_t kL = kPQ + D / 2;    // linear-term accumulator (D columns)
  static constexpr uint32_t kCols = 512;
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
  const float* G;
  const float* Z;
  const float* s;
  float gate_override;
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

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D, bool HYB>
__global__ void __launch_bounds__(192, 1) attn_kernel(const __grid_constant__ CUtensorMap mk,
                                                      const __grid_constant__ CUtensorMap mv,
                                                      const __grid_constant__ CUtensorMap mkp,
                                                      const __grid_constant__ CUtensorMap mvp,
                                                      const __grid_constant__ Params P) {
  using C = AT<D, HYB>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* stages = sm;
  unsigned char* img_hi = sm + C::kStages * C::kStage;
  unsigned char* img_lo = img_hi + C::kImg;
  float* zs = reinterpret_cast<float*>(img_lo + C::kImg);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<unsigned char*>(zs) + C::kZ);
  // bars: full[S] empty[S] s_full[2] p_full[2] o_done q_ready lin_done drain
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * C::kStages + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  auto full = [&](int s) { return smem_u32(bars + s); };
  auto empty = [&](int s) { return smem_u32(bars + C::kStages + s); };
  auto s_full = [&](int b) { return smem_u32(bars + 2 * C::kStages + b); };
  auto p_full = [&](int b) { return smem_u32(bars + 2 * C::kStages + 2 + b); };
  const uint32_t o_done = smem_u32(bars + 2 * C::kStages + 4);
  const uint32_t q_ready = smem_u32(bars + 2 * C::kStages + 5);
  const uint32_t lin_done = smem_u32(bars + 2 * C::kStages + 6);
  const uint32_t drain = smem_u32(bars + 2 * C::kStages + 7);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long total = static_cast<long long>(P.B) * P.H * P.npairs;
  const unsigned long long wait_ns = P.wait_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full(b), 1);
      mbar_init(p_full(b), 4);
    }
    mbar_init(o_done, 1);
    mbar_init(q_ready, 4);
    mbar_init(lin_done, 1);
    mbar_init(drain, 1);
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
      long long tc = 0;
      bool ok = true;
      for (long long w = blockIdx.x; w < total && ok; w += gridDim.x) {
        const Item it = make_item(P, w);
        const CUtensorMap* km = it.slot >= 0 ? &mkp : &mk;
        const CUtensorMap* vm = it.slot >= 0 ? &mvp : &mv;
        const int z = it.slot >= 0 ? it.b * P.Hs + it.slot : it.bh;
        for (int t = 0; t < it.ntiles; ++t, ++tc) {
          int j, mask;
          tile_of(it, t, P.mode, j, mask);
          const int s = static_cast<int>(tc % C::kStages);
          const long long n = tc / C::kStages;
          if (n > 0 && !mbar_wait(empty(s), static_cast<uint32_t>((n - 1) & 1), wait_ns, abort_flag)) {
            raise_timeout(P.err, abort_flag);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full(s), C::kStage);
          const uint32_t kdst = smem_u32(stages + s * C::kStage);
          const uint32_t vdst = kdst + C::kTile;
#pragma unroll
          for (int hh = 0; hh < D / 64; ++hh) {
            tma_load_3d(kdst + hh * kSlab, km, full(s), hh * 64, j * 64, z);
            tma_load_3d(vdst + hh * kSlab, vm, full(s), hh * 64, j * 64, z);
          }
        }
      }
      // Drain every issued load before leaving.
      for (int s = 0; s < C::kStages && s < tc; ++s) {
        const long long last = s + ((tc - 1 - s) / C::kStages) * C::kStages;
        if (!mbar_wait(full(s), static_cast<uint32_t>((last / C::kStages) & 1), wait_ns, nullptr))
          atomicOr(P.err, kErrTimeout);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ================================================= MMA issuer
      constexpr uint32_t idesc_qk = idesc_bf16(128, 64, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
      constexpr uint32_t idesc_lin = idesc_bf16(128, D, false, false);
      long long tc = 0;
      uint32_t ic = 0;
      uint32_t pf_count[2] = {0, 0};
      bool ok = true;
      for (long long w = blockIdx.x; w < total && ok; w += gridDim.x, ++ic) {
        const Item it = make_item(P, w);
        if (!mbar_wait(q_ready, ic & 1, wait_ns, abort_flag)) {
          raise_timeout(P.err, abort_flag);
          ok = false;
          break;
        }
        tc_fence_after();
        if constexpr (HYB) {
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t off = (ks / 4) * (D * 128) + (ks % 4) * 32;
            mma_ts(tmem + C::kL, tmem + C::kPQ + ks * 8,
                   sdesc_sw128(smem_u32(img_hi) + off, 16, 1024), idesc_lin, ks > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t off = (ks / 4) * (D * 128) + (ks % 4) * 32;
            mma_ts(tmem + C::kL, tmem + C::kPQ + ks * 8,
                   sdesc_sw128(smem_u32(img_lo) + off, 16, 1024), idesc_lin, 1u);
          }
          mma_commit(lin_done);
        }
        const long long tc0 = tc;
        auto issue_pv = [&](int t) -> bool {
          const int sb = t & 1;
          if (!mbar_wait(p_full(sb), pf_count[sb] & 1, wait_ns, abort_flag)) return false;
          ++pf_count[sb];
          tc_fence_after();
          const int s = static_cast<int>((tc0 + t) % C::kStages);
          const uint32_t vaddr = smem_u32(stages + s * C::kStage) + C::kTile;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_ts(tmem + C::kO, tmem + C::kS + sb * 64 + ks * 8,
                   sdesc_sw128(vaddr + ks * 2048, kSlab, 1024), idesc_pv,
                   (t > 0 || ks > 0) ? 1u : 0u);
          mma_commit(empty(s));
          mma_commit(o_done);
          return true;
        };
        for (int t = 0; t < it.ntiles; ++t, ++tc) {
          const int s = static_cast<int>(tc % C::kStages);
          if (!mbar_wait(full(s), static_cast<uint32_t>((tc / C::kStages) & 1), wait_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int sb = t & 1;
          const uint32_t kaddr = smem_u32(stages + s * C::kStage);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            mma_ts(tmem + C::kS + sb * 64, tmem + C::kQ + ks * 8,
                   sdesc_sw128(kaddr + (ks / 4) * kSlab + (ks % 4) * 32, 16, 1024), idesc_qk,
                   ks > 0 ? 1u : 0u);
          mma_commit(s_full(sb));
          if (t >= 1 && !issue_pv(t - 1)) {
            ok = false;
            break;
          }
        }
        if (ok && it.ntiles >= 1 && !issue_pv(it.ntiles - 1)) ok = false;
        if (!ok) raise_timeout(P.err, abort_flag);
      }
      mma_commit(drain);
      if (!mbar_wait(drain, 0, wait_ns, nullptr)) atomicOr(P.err, kErrTimeout);
    }
  } else {
    // ================================================= softmax + epilogue
    const int quarter = warp % 4;
    const int r = quarter * 32 + lane;          // row within the pair (TMEM lane)
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const int tid = threadIdx.x - 64;
    uint32_t ic = 0;
    uint32_t sf_count[2] = {0, 0};
    long long pv_base = 0;                      // PVs completed before this item
    int prev_bh = -1;
    bool ok = true;
    for (long long w = blockIdx.x; w < total && ok; w += gridDim.x, ++ic) {
      const Item it = make_item(P, w);
      const int row_pos = it.p * 128 + r;        // position in the head's (possibly regrouped) order
      const bool row_valid = row_pos < P.N;
      // ---- operands of this item: Q (and relu(Q), G, Z) into TMEM / smem
      if constexpr (HYB) {
        if (it.bh != prev_bh) {
          build_b_image_hilo<D>(P.G + static_cast<long long>(it.bh) * D * D, img_hi, img_lo, tid, 128);
          for (int c = tid; c < D; c += 128) zs[c] = P.Z[static_cast<long long>(it.bh) * D + c];
          fence_proxy_async_smem();
          asm volatile("bar.sync 1, 128;" ::: "memory");
        }
      }
      prev_bh = it.bh;
      const __nv_bfloat16* qsrc =
          it.slot >= 0 ? P.qp + (static_cast<long long>(it.b) * P.Hs + it.slot) * P.N * D
                       : P.q + static_cast<long long>(it.bh) * P.N * D;
      const uint4* qrow = reinterpret_cast<const uint4*>(qsrc + static_cast<long long>(row_valid ? row_pos : 0) * D);
      float den = 0.f;
#pragma unroll
      for (int c0 = 0; c0 < D / 2; c0 += 16) {
        uint32_t pk[16], pr[16];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint4 v = row_valid ? __ldg(qrow + c0 / 4 + u) : make_uint4(0, 0, 0, 0);
          pk[4 * u + 0] = v.x; pk[4 * u + 1] = v.y; pk[4 * u + 2] = v.z; pk[4 * u + 3] = v.w;
        }
        tmem_st16(lane_base + C::kQ + c0, pk);
        if constexpr (HYB) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            pr[e] = relu_bf16x2(pk[e]);
            const float2 f = unpack_bf16x2(pr[e]);
            den = fmaf(f.x, zs[2 * (c0 + e)], den);
            den = fmaf(f.y, zs[2 * (c0 + e) + 1], den);
          }
          tmem_st16(lane_base + C::kPQ + c0, pr);
        }
      }
      den += P.eps;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);

      // ---- softmax over the key tiles
      const float c2 = P.scale_log2;
      float m = -INFINITY;   // running max in the exp2 domain
      float l = 0.f;
      const int half_bit = r >= 64 ? 2 : 1;
      for (int t = 0; t < it.ntiles; ++t) {
        const int sb = t & 1;
        // Waits and TMEM accesses are warp-collective: every decision that
        // guards one is made uniform across the warp first.
        if (!__all_sync(0xffffffffu, mbar_wait(s_full(sb), sf_count[sb] & 1, wait_ns, abort_flag))) {
          ok = false;
          break;
        }
        ++sf_count[sb];
        tc_fence_after();
        int j, mask;
        tile_of(it, t, P.mode, j, mask);
        // Valid key columns of this tile form one contiguous range [lo, hi].
        int lo = 0, hi = min(63, P.N - 1 - j * 64);
        if (P.mode == kModeBand) {
          lo = max(lo, row_pos - P.window - j * 64);
          hi = min(hi, row_pos + P.window - j * 64);
        }
        const bool live = row_valid && (mask & half_bit) && lo <= hi;
        const bool whole = live && lo == 0 && hi == 63;
        uint32_t pk[32];
        float f = 1.0f;            // factor O must be rescaled by before PV(t)
        if (__any_sync(0xffffffffu, live)) {
          float sv[64];
          {
            uint32_t s0[32], s1[32];
            tmem_ld32(lane_base + C::kS + sb * 64, s0);
            tmem_ld32(lane_base + C::kS + sb * 64 + 32, s1);
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              sv[c] = __uint_as_float(s0[c]);
              sv[c + 32] = __uint_as_float(s1[c]);
            }
          }
          // Columns outside [lo, hi] (and every column of a dead row) become
          // -inf; only tiles with a partial row in this warp pay for it.
          if (__any_sync(0xffffffffu, !whole)) {
#pragma unroll
            for (int c = 0; c < 64; ++c) sv[c] = (live && c >= lo && c <= hi) ? sv[c] : -INFINITY;
          }
          float t32[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) t32[c] = fmaxf(sv[c], sv[c + 32]);
#pragma unroll
          for (int w2 = 16; w2 >= 1; w2 >>= 1)
#pragma unroll
            for (int c = 0; c < w2; ++c) t32[c] = fmaxf(t32[c], t32[c + w2]);
          const float mx = t32[0] * c2;   // c2 > 0: max of scaled = scaled max
          if (mx > m + 8.0f) {
            // Raise the running max.  O (from PV up to t-1) is rescaled below,
            // once PV(t-1) has landed; l is rescaled here.
            f = (m == -INFINITY) ? 1.0f : ex2(m - mx);
            l *= f;
            m = mx;
          }
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
        tmem_st32(lane_base + C::kS + sb * 64, pk);
        // Observe PV(t-1) -- every warp observes every PV completion in order,
        // so each parity wait is at most one phase behind the barrier.
        if (t >= 1) {
          const long long g = pv_base + t - 1;
          if (!__all_sync(0xffffffffu, mbar_wait(o_done, static_cast<uint32_t>(g & 1), wait_ns, abort_flag))) {
            ok = false;
            break;
          }
        }
        if (__any_sync(0xffffffffu, f != 1.0f)) {
          tc_fence_after();
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
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
        if (lane == 0) mbar_arrive(p_full(sb));
      }
      if (!ok) break;
      // ---- epilogue
      if (it.ntiles >= 1) {
        const long long g = pv_base + it.ntiles - 1;
        if (!__all_sync(0xffffffffu, mbar_wait(o_done, static_cast<uint32_t>(g & 1), wait_ns, abort_flag))) { ok = false; break; }
      }
      if constexpr (HYB) {
        if (!__all_sync(0xffffffffu, mbar_wait(lin_done, ic & 1, wait_ns, abort_flag))) { ok = false; break; }
      }
      tc_fence_after();
      pv_base += it.ntiles;
      float gate = 0.f;
      if constexpr (HYB) gate = P.s != nullptr ? __ldg(P.s + it.b) : P.gate_override;
      const float inv_l = 1.0f / l;
      const float lin_scale = gate / den;
      long long out_row = row_pos;
      if (it.slot >= 0 && row_valid) {
        const int f = row_pos % P.F, pos = row_pos / P.F;
        const int y = pos / P.Wh, x = pos % P.Wh;
        out_row = (static_cast<long long>(f) * P.Hh + y) * P.Wh + x;
      }
      uint4* orow = reinterpret_cast<uint4*>(P.o + (static_cast<long long>(it.bh) * P.N + (row_valid ? out_row : 0)) * D);
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o32[32];
        tmem_ld32(lane_base + C::kO + c0, o32);
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(o32[e]) * inv_l;
        if constexpr (HYB) {
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
  const int grid = static_cast<int>(items < c.num_sms ? items : c.num_sms);
  attn_kernel<D, HYB><<<grid, 192, C::kSmem, c.stream>>>(mk, mv, mkp, mvp, P);
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
  P.G = a.G;
  P.Z = a.Z;
  P.s = a.s;
  P.gate_override = a.gate_override;
  P.eps = a.eps;
  P.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(a.d));
  P.o = static_cast<__nv_bfloat16*>(a.o);
  P.err = c.err;
  P.wait_ns = c.wait_ns;
  const bool hyb = a.G != nullptr;
  if (a.d == 128) return hyb ? launch_attn_t<128, true>(c, a, P) : launch_attn_t<128, false>(c, a, P);
  return hyb ? launch_attn_t<64, true>(c, a, P) : launch_attn_t<64, false>(c, a, P);
}

cudaError_t launch_debug_wait(const Ctx& c) {
  debug_wait_kernel<<<1, 32, 0, c.stream>>>(c.err, c.wait_ns);
  return cudaGetLastError();
}

}  // namespace salad
