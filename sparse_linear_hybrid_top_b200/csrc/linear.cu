// linear.cu -- the linear-attention branch of the hybrid layer.
//
// "SALAD ... (paper.rainbus.top)" 前置知识 Linear Attention and 方法步骤详情
// step 3: phi = ReLU, H = phi(K)^T V (d x d), Z = phi(K)^T 1, output
// phi(Q) H / (phi(Q) Z); eps is added to the denominator.
//
// linear_state: split-N on tensor cores.  Each CTA streams a run of 64-token
// K/V tiles (TMA, 128-byte swizzle) through a 3-4 stage ring; four warps
// apply ReLU to the K tile in place (and accumulate Z), one thread issues
// tcgen05.mma with A = relu(K)^T and B = V, both read MN-major straight from
// the TMA tiles, accumulating the d x d partial in TMEM.  Partials go to the
// workspace and a fixed-order reduction forms H and Z (deterministic).
// HBM-bound: 2 * N * d * 2 bytes per head read once.
//
// linear_apply: A = phi(Q) rows in TMEM (one row per thread), B = H split
// into bf16 hi + lo parts (H ~= hi + lo to ~16 mantissa bits) in a K-major
// swizzled shared-memory image, two MMAs into one TMEM accumulator; the
// denominator phi(q) . Z + eps is a per-thread float32 dot product.
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace salad {
namespace {

constexpr int kSlab = 64 * 128;   // one [64 rows x 64 bf16] 128B-swizzled slab

// ---------------------------------------------------------- linear_state --
template <int D>
struct LS {
  static constexpr int kStages = 3;
  static constexpr int kTile = (D / 64) * kSlab;         // K or V tile bytes
  static constexpr int kStage = 2 * kTile;
  static constexpr int kZero = (D == 64) ? kSlab : 0;    // zero slab pads M to 128
  static constexpr int kRed = 128 * 16 * 4;              // Z partials
  static constexpr int kBars = 256;
  static constexpr int kTheta = 64 * 8;                  // rotary rates, one per channel pair
  static constexpr int kSmem = 1024 /*align slack*/ + kStages * kStage + kZero + kRed + kBars + kTheta;
};

__device__ __forceinline__ bool branch_dropped(const BranchDrop& d, int b) {
  const float g = d.s != nullptr ? __ldg(d.s + b) : d.gate_override;
  return g < d.thr;
}

template <int D>
__global__ void __launch_bounds__(192, 1) linear_state_kernel(
    const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv, int nblk,
    int blocks_per_cta, int ctas_per_head, float* __restrict__ partH, float* __restrict__ partZ,
    unsigned* err, unsigned long long wait_ns, BranchDrop drop, int H, Rope3D rope, int N) {
  using C = LS<D>;
  // A sample whose linear branch is dropped needs no state: the whole CTA
  // leaves before touching shared memory, barriers or TMEM.
  if (branch_dropped(drop, static_cast<int>(blockIdx.x / ctas_per_head) / H)) return;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* stage_base = sm;
  unsigned char* zero_slab = sm + C::kStages * C::kStage;
  float* zred = reinterpret_cast<float*>(zero_slab + C::kZero);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<unsigned char*>(zred) + C::kRed);
  // bars: full[0..S), relu[S..2S), empty[2S..3S), acc, drain; then tmem holder, abort
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 3 * C::kStages + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  double* theta = reinterpret_cast<double*>(reinterpret_cast<unsigned char*>(bars) + C::kBars);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.x / ctas_per_head;
  const int chunk = blockIdx.x % ctas_per_head;
  const int b0 = chunk * blocks_per_cta;
  const int nt = min(nblk, b0 + blocks_per_cta) - b0;

  auto full = [&](int s) { return smem_u32(bars + s); };
  auto relu_bar = [&](int s) { return smem_u32(bars + C::kStages + s); };
  auto empty = [&](int s) { return smem_u32(bars + 2 * C::kStages + s); };
  const uint32_t acc_bar = smem_u32(bars + 3 * C::kStages);
  const uint32_t drain_bar = smem_u32(bars + 3 * C::kStages + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(relu_bar(s), 4);
      mbar_init(empty(s), 1);
    }
    mbar_init(acc_bar, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&mk);
    tma_prefetch_map(&mv);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), 128);
    tmem_relinquish();
  }
  if constexpr (D == 64) {
    for (int i = threadIdx.x; i < kSlab / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(zero_slab)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int issued = 0;
      for (int t = 0; t < nt; ++t) {
        const int s = t % C::kStages;
        if (t >= C::kStages &&
            !mbar_wait(empty(s), ((t / C::kStages) - 1) & 1, wait_ns, abort_flag)) {
          raise_timeout(err, abort_flag);
          break;
        }
        mbar_arrive_expect_tx(full(s), C::kStage);
        const uint32_t kdst = smem_u32(stage_base + s * C::kStage);
        const uint32_t vdst = kdst + C::kTile;
        const int row = (b0 + t) * 64;
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          tma_load_3d(kdst + h * kSlab, &mk, full(s), h * 64, row, bh);
          tma_load_3d(vdst + h * kSlab, &mv, full(s), h * 64, row, bh);
        }
        ++issued;
      }
      // Drain: every issued load has landed before the CTA may exit.
      for (int s = 0; s < C::kStages && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / C::kStages) * C::kStages;  // last t on stage s
        if (!mbar_wait(full(s), (last / C::kStages) & 1, wait_ns, nullptr)) atomicOr(err, kErrTimeout);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: acc[d_k][d_v] += relu(K)^T V
      constexpr uint32_t idesc = idesc_bf16(128, D, true, true);
      bool ok = true;
      for (int t = 0; t < nt && ok; ++t) {
        const int s = t % C::kStages;
        if (!mbar_wait(relu_bar(s), (t / C::kStages) & 1, wait_ns, abort_flag)) {
          raise_timeout(err, abort_flag);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kaddr = smem_u32(stage_base + s * C::kStage);
        const uint32_t vaddr = kaddr + C::kTile;
        // A (M = d_k, MN-major): rows 0..63 in the first K slab, rows 64..127
        // in the second slab (D = 128) or in the zero slab (D = 64).
        const uint32_t lbo_a = (D == 128) ? kSlab : (smem_u32(zero_slab) - kaddr);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t a = sdesc_sw128(kaddr + ks * 2048, lbo_a, 1024);
          const uint64_t b = sdesc_sw128(vaddr + ks * 2048, kSlab, 1024);
          mma_ss(tmem, a, b, idesc, (t > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(empty(s));
      }
      if (ok) mma_commit(acc_bar);
      mma_commit(drain_bar);
      if (!mbar_wait(drain_bar, 0, wait_ns, nullptr)) atomicOr(err, kErrTimeout);
    }
  } else {
    // ---------------- ReLU + Z workers (warps 2..5) and the epilogue
    const int tid = threadIdx.x - 64;
    if (rope.on) {
      if (tid < D / 2) theta[tid] = rope.theta[tid];
      asm volatile("bar.sync 1, 128;" ::: "memory");
    }
    float zacc[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) zacc[e] = 0.f;
    bool ok = true;
    for (int t = 0; t < nt; ++t) {
      const int s = t % C::kStages;
      if (!__all_sync(0xffffffffu, mbar_wait(full(s), (t / C::kStages) & 1, wait_ns, abort_flag))) {
        raise_timeout(err, abort_flag);
        ok = false;
        break;
      }
      unsigned char* ktile = stage_base + s * C::kStage;
#pragma unroll
      for (int i = 0; i < (D / 64) * 4; ++i) {
        const int half = i / 4;
        const int q = tid + 128 * (i % 4);
        uint4* p = reinterpret_cast<uint4*>(ktile + half * kSlab + q * 16);
        uint4 v = *p;
        uint32_t w4[4] = {relu_bf16x2(v.x), relu_bf16x2(v.y), relu_bf16x2(v.z), relu_bf16x2(v.w)};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = unpack_bf16x2(w4[e]);
          zacc[half * 8 + 2 * e] += f.x;
          zacc[half * 8 + 2 * e + 1] += f.y;
        }
        if (rope.on) {
          // The numerator's features are rotated; Z above is not.  Chunk q
          // of the swizzled slab holds channels half*64 + 8L .. +7 of tile
          // row q/8, with L = (q%8) ^ (row%8): pairs half*32 + 4L + e.
          const int row = q / 8;
          const int tok = (b0 + t) * 64 + row;
          if (tok < N) {
            const int L = (q % 8) ^ (row % 8);
            const int plane = rope.Hh * rope.Wh;
            const int f = tok / plane, y = (tok / rope.Wh) % rope.Hh, x = tok % rope.Wh;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 cs = rope_cs(rope, theta, half * 32 + 4 * L + e, f, y, x);
              const float2 a = unpack_bf16x2(w4[e]);
              w4[e] = pack_bf16x2(a.x * cs.x - a.y * cs.y, a.x * cs.y + a.y * cs.x);
            }
          }
        }
        v.x = w4[0];
        v.y = w4[1];
        v.z = w4[2];
        v.w = w4[3];
        *p = v;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(relu_bar(s));
    }
    // Z: thread tid holds columns half*64 + L*8 + e with L = (tid%8)^((tid/8)%8).
#pragma unroll
    for (int e = 0; e < 16; ++e) zred[tid * 16 + e] = zacc[e];
    asm volatile("bar.sync 1, 128;" ::: "memory");
    for (int c = tid; c < D; c += 128) {
      const int half = c / 64, l = (c % 64) / 8, e = c % 8;
      float z = 0.f;
      for (int t2 = 0; t2 < 128; ++t2)
        if ((((t2 & 7) ^ ((t2 >> 3) & 7))) == l) z += zred[t2 * 16 + half * 8 + e];
      partZ[static_cast<long long>(blockIdx.x) * D + c] = z;
    }
    const bool acc_ok = __all_sync(0xffffffffu, ok && mbar_wait(acc_bar, 0, wait_ns, abort_flag));
    if (acc_ok) {
      tc_fence_after();
      const int quarter = warp % 4;
      const int row = quarter * 32 + lane;  // d_k index
      float* dst = partH + static_cast<long long>(blockIdx.x) * D * D + static_cast<long long>(row) * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem_addr(tmem, quarter * 32, c0), r);
        if (row < D) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + c0 + e) =
                make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]),
                            __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
        }
      }
    } else if (ok) {
      raise_timeout(err, abort_flag);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// Sum over c = 0..n-1 of src[c * stride], in ascending c, with eight loads in
// flight at a time (the partials live in L2 or HBM; a dependent chain of
// loads would leave the reduction latency-bound).
__device__ __forceinline__ float sum_strided(const float* __restrict__ src, long long stride,
                                             int n) {
  float acc = 0.f;
  int c = 0;
  for (; c + 8 <= n; c += 8) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = __ldg(src + (c + u) * stride);
#pragma unroll
    for (int u = 0; u < 8; ++u) acc += v[u];
  }
  for (; c < n; ++c) acc += __ldg(src + c * stride);
  return acc;
}

// Fixed-order reduction of the split-N partials.
__global__ void linear_reduce_kernel(const float* __restrict__ partH,
                                     const float* __restrict__ partZ, int D, int cph,
                                     float* __restrict__ Hst, float* __restrict__ Z) {
  const long long bh = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  const int DD = D * D;
  if (e < DD) Hst[bh * DD + e] = sum_strided(partH + bh * cph * DD + e, DD, cph);
  if (e < D) Z[bh * D + e] = sum_strided(partZ + bh * cph * D + e, D, cph);
}

// The linear state's reduction fused with the fold of W_lin, for the forward
// pass.  CTA (x, bh): rows [4x, 4x + 4) of Hst[bh] = sum of the per-CTA
// partials in ascending order (written out, as by linear_reduce_kernel), Z[bh]
// in CTA x = 0, then rows [4x, 4x + 4) of G[bh] = Hst[bh] W_lin[h] (float32
// accumulation in ascending m, W_lin in bf16) written as the bf16 B-operand
// image of D[row][j] += A[row][c] G[c][j]: K-major (K = c), 128-byte swizzle,
// slab c/64 of d rows x 128 bytes.
constexpr int kFoldRows = 4;
__global__ void __launch_bounds__(256) linear_reduce_fold_kernel(
    const float* __restrict__ partH, const float* __restrict__ partZ, int H, int D, int cph,
    const __nv_bfloat16* __restrict__ W, float* __restrict__ Hst, float* __restrict__ Z,
    __nv_bfloat16* __restrict__ Gimg, BranchDrop drop) {
  if (branch_dropped(drop, static_cast<int>(blockIdx.y) / H)) return;
  extern __shared__ __align__(16) float fold_sm[];
  float* hrows = fold_sm;                                                       // [4][D]
  __nv_bfloat16* wsm = reinterpret_cast<__nv_bfloat16*>(fold_sm + kFoldRows * D);  // [D][D]
  const long long bh = blockIdx.y;
  const int h = static_cast<int>(bh % H);
  const int r0 = blockIdx.x * kFoldRows;
  const int DD = D * D;
  const uint4* wsrc = reinterpret_cast<const uint4*>(W + static_cast<long long>(h) * DD);
  for (int e = threadIdx.x; e < DD / 8; e += blockDim.x)
    reinterpret_cast<uint4*>(wsm)[e] = __ldg(wsrc + e);
  for (int e = threadIdx.x; e < kFoldRows * D; e += blockDim.x) {
    const long long off = static_cast<long long>(r0) * D + e;
    const float acc = sum_strided(partH + bh * cph * DD + off, DD, cph);
    hrows[e] = acc;
    Hst[bh * DD + off] = acc;
  }
  if (blockIdx.x == 0) {
    for (int e = threadIdx.x; e < D; e += blockDim.x)
      Z[bh * D + e] = sum_strided(partZ + bh * cph * D + e, D, cph);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kFoldRows * D; e += blockDim.x) {
    const int r = e / D, j = e % D;
    float acc = 0.f;
    for (int m = 0; m < D; ++m) acc = fmaf(hrows[r * D + m], __bfloat162float(wsm[m * D + j]), acc);
    const int c = r0 + r;
    const uint32_t off = (c / 64) * (D * 128) + sw128_offset(j, c % 64);
    Gimg[bh * DD + off / 2] = __float2bfloat16_rn(acc);
  }
}

}  // namespace

namespace {

// ---------------------------------------------------------- linear_apply --
template <int D>
struct LA {
  static constexpr int kImg = D * D * 2;   // one bf16 image (hi or lo)
  static constexpr int kSmem = 1024 + 2 * kImg + D * 4 + 64;
};

template <int D>
__global__ void __launch_bounds__(128, 1) linear_apply_kernel(
    const __nv_bfloat16* __restrict__ q, const float* __restrict__ Hst,
    const float* __restrict__ Z, float eps, int N, int ntiles, __nv_bfloat16* __restrict__ o,
    unsigned* err, unsigned long long wait_ns, const __grid_constant__ Rope3D rope) {
  using C = LA<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* img_hi = sm;
  unsigned char* img_lo = sm + C::kImg;
  float* zs = reinterpret_cast<float*>(sm + 2 * C::kImg);
  uint64_t* bar = reinterpret_cast<uint64_t*>(zs + D);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long bh = blockIdx.x / ntiles;
  const int tile = blockIdx.x % ntiles;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(bar), 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), 256);
    tmem_relinquish();
  }
  build_b_image_hilo<D>(Hst + bh * D * D, img_hi, img_lo, threadIdx.x, 128);
  for (int c = threadIdx.x; c < D; c += 128) zs[c] = Z[bh * D + c];
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t acc_col = 0, a_col = D;  // accumulator [0, D), A = phi(Q) [D, D + D/2)

  // Row r of the tile: phi(q) into TMEM (A operand), denominator in a register.
  const int r = warp * 32 + lane;
  const long long row = static_cast<long long>(tile) * 128 + r;
  const bool valid = row < N;
  const uint4* qrow = reinterpret_cast<const uint4*>(q + (bh * N + (valid ? row : 0)) * D);
  float den = 0.f;
  // 3-D rotary encoding: the numerator's phi(q) turns by the token's frame,
  // row and column positions; the denominator keeps the unrotated phi(q).
  const bool rope_on = rope.on && valid;
  int rf = 0, ry = 0, rx = 0;
  if (rope_on) {
    const int tok = static_cast<int>(row);
    rf = tok / (rope.Hh * rope.Wh);
    ry = (tok / rope.Wh) % rope.Hh;
    rx = tok % rope.Wh;
  }
#pragma unroll
  for (int c0 = 0; c0 < D / 2; c0 += 16) {  // 16 packed columns = 32 bf16 per step
    uint32_t pk[16];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint4 v = valid ? __ldg(qrow + c0 / 4 + u) : make_uint4(0, 0, 0, 0);
      pk[4 * u + 0] = relu_bf16x2(v.x);
      pk[4 * u + 1] = relu_bf16x2(v.y);
      pk[4 * u + 2] = relu_bf16x2(v.z);
      pk[4 * u + 3] = relu_bf16x2(v.w);
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float2 f = unpack_bf16x2(pk[e]);
      den = fmaf(f.x, zs[2 * (c0 + e)], den);
      den = fmaf(f.y, zs[2 * (c0 + e) + 1], den);
      if (rope_on) {   // pair c0 + e = channels 2(c0 + e), 2(c0 + e) + 1
        const float2 cs = rope_cs(rope, rope.theta, c0 + e, rf, ry, rx);
        pk[e] = pack_bf16x2(f.x * cs.x - f.y * cs.y, f.x * cs.y + f.y * cs.x);
      }
    }
    tmem_st16(tmem_addr(tmem, warp * 32, a_col + c0), pk);
  }
  den += eps;
  tmem_st_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) {
    constexpr uint32_t idesc = idesc_bf16(128, D, false, false);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const uint32_t off = (ks / 4) * (D * 128) + (ks % 4) * 32;
      mma_ts(tmem + acc_col, tmem + a_col + ks * 8, sdesc_sw128(smem_u32(img_hi) + off, 16, 1024),
             idesc, ks > 0 ? 1u : 0u);
    }
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const uint32_t off = (ks / 4) * (D * 128) + (ks % 4) * 32;
      mma_ts(tmem + acc_col, tmem + a_col + ks * 8, sdesc_sw128(smem_u32(img_lo) + off, 16, 1024),
             idesc, 1u);
    }
    mma_commit(smem_u32(bar));
  }
  __syncwarp();
  const bool done = __all_sync(0xffffffffu, mbar_wait(smem_u32(bar), 0, wait_ns, nullptr));
  if (!done) atomicOr(err, kErrTimeout);
  tc_fence_after();
  if (done) {
    const float inv = 1.0f / den;
    uint4* orow = reinterpret_cast<uint4*>(o + (bh * N + (valid ? row : 0)) * D);
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t rr[32];
      tmem_ld32(tmem_addr(tmem, warp * 32, acc_col + c0), rr);
      if (valid) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(rr[8 * u + 0]) * inv, __uint_as_float(rr[8 * u + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(rr[8 * u + 2]) * inv, __uint_as_float(rr[8 * u + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(rr[8 * u + 4]) * inv, __uint_as_float(rr[8 * u + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(rr[8 * u + 6]) * inv, __uint_as_float(rr[8 * u + 7]) * inv);
          orow[c0 / 8 + u] = w;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

struct LSPlan {
  int nblk, blocks_per_cta, ctas_per_head;
};
LSPlan ls_plan(int B, int H, int N, int num_sms) {
  LSPlan p;
  p.nblk = (N + 63) / 64;
  const int BH = B * H;
  int cph = (2 * num_sms) / BH;
  if (cph < 1) cph = 1;
  if (cph > p.nblk) cph = p.nblk;
  p.blocks_per_cta = (p.nblk + cph - 1) / cph;
  p.ctas_per_head = (p.nblk + p.blocks_per_cta - 1) / p.blocks_per_cta;
  return p;
}

}  // namespace

size_t linear_state_ws_bytes(int B, int H, int N, int d) {
  const LSPlan p = ls_plan(B, H, N, 256);
  const size_t parts = static_cast<size_t>(B) * H * p.ctas_per_head;
  return align256(parts * d * d * sizeof(float)) + align256(parts * d * sizeof(float));
}

cudaError_t launch_linear_state(const Ctx& c, const void* k, const void* v, int B, int H, int N,
                                int d, float* Hst, float* Z, void* ws, const void* w_lin,
                                void* Gimg, BranchDrop drop, Rope3D rope) {
  const LSPlan p = ls_plan(B, H, N, c.num_sms < 256 ? c.num_sms : 256);
  const int BH = B * H;
  const size_t parts = static_cast<size_t>(BH) * p.ctas_per_head;
  float* partH = static_cast<float*>(ws);
  float* partZ = reinterpret_cast<float*>(static_cast<char*>(ws) +
                                          align256(parts * d * d * sizeof(float)));
  CUtensorMap mk, mv;
  if (!make_tmap_bf16_3d(&mk, k, BH, N, d) || !make_tmap_bf16_3d(&mv, v, BH, N, d))
    return cudaErrorInvalidValue;
  const int grid = BH * p.ctas_per_head;
  cudaError_t e;
  if (d == 128) {
    e = cudaFuncSetAttribute(linear_state_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             LS<128>::kSmem);
    if (e != cudaSuccess) return e;
    linear_state_kernel<128><<<grid, 192, LS<128>::kSmem, c.stream>>>(
        mk, mv, p.nblk, p.blocks_per_cta, p.ctas_per_head, partH, partZ, c.err, c.wait_ns, drop,
        H, rope, N);
  } else {
    e = cudaFuncSetAttribute(linear_state_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             LS<64>::kSmem);
    if (e != cudaSuccess) return e;
    linear_state_kernel<64><<<grid, 192, LS<64>::kSmem, c.stream>>>(
        mk, mv, p.nblk, p.blocks_per_cta, p.ctas_per_head, partH, partZ, c.err, c.wait_ns, drop,
        H, rope, N);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (w_lin == nullptr) {
    linear_reduce_kernel<<<dim3((d * d + 255) / 256, BH), 256, 0, c.stream>>>(
        partH, partZ, d, p.ctas_per_head, Hst, Z);
    return cudaGetLastError();
  }
  const size_t smem = kFoldRows * d * sizeof(float) + static_cast<size_t>(d) * d * 2;
  e = cudaFuncSetAttribute(linear_reduce_fold_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  linear_reduce_fold_kernel<<<dim3(d / kFoldRows, BH), 256, smem, c.stream>>>(
      partH, partZ, H, d, p.ctas_per_head, static_cast<const __nv_bfloat16*>(w_lin), Hst, Z,
      static_cast<__nv_bfloat16*>(Gimg), drop);
  return cudaGetLastError();
}

Rope3D make_rope3d(int d, int F, int Hh, int Wh, float base) {
  Rope3D r;
  r.on = 1;
  r.F = F;
  r.Hh = Hh;
  r.Wh = Wh;
  const int gy = 2 * (d / 6), gt = d - 2 * gy;
  r.gt2 = gt / 2;
  r.gy2 = gy / 2;
  for (int m = 0; m < d / 2; ++m) {
    int i, g;
    if (m < r.gt2) {
      i = m; g = gt;
    } else if (m < r.gt2 + r.gy2) {
      i = m - r.gt2; g = gy;
    } else {
      i = m - r.gt2 - r.gy2; g = gy;
    }
    r.theta[m] = std::pow(static_cast<double>(base), -2.0 * i / g);
  }
  return r;
}

cudaError_t launch_linear_apply(const Ctx& c, const void* q, const float* Hst, const float* Z,
                                float eps, int B, int H, int N, int d, void* o, Rope3D rope) {
  const int ntiles = (N + 127) / 128;
  const int grid = B * H * ntiles;
  cudaError_t e;
  if (d == 128) {
    e = cudaFuncSetAttribute(linear_apply_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             LA<128>::kSmem);
    if (e != cudaSuccess) return e;
    linear_apply_kernel<128><<<grid, 128, LA<128>::kSmem, c.stream>>>(
        static_cast<const __nv_bfloat16*>(q), Hst, Z, eps, N, ntiles,
        static_cast<__nv_bfloat16*>(o), c.err, c.wait_ns, rope);
  } else {
    e = cudaFuncSetAttribute(linear_apply_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             LA<64>::kSmem);
    if (e != cudaSuccess) return e;
    linear_apply_kernel<64><<<grid, 128, LA<64>::kSmem, c.stream>>>(
        static_cast<const __nv_bfloat16*>(q), Hst, Z, eps, N, ntiles,
        static_cast<__nv_bfloat16*>(o), c.err, c.wait_ns, rope);
  }
  return cudaGetLastError();
}

}  // namespace salad
