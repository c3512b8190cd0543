// permute.cu -- token regrouping of the spatio-temporal sliding-window heads.
//
// "视频扩散模型中的稀疏注意力机制解析 (ijyty.com)" 1.1: the 3-D latent is
// flattened with time slowest, t = (f*Hh + y)*Wh + x, so one spatial
// position's frames sit Hh*Wh apart; heads with temporal locality regroup the
// tokens by spatial position, r = (y*Wh + x)*F + f, before the 1-D window.
// Pure data movement (HBM-bound): 16-byte vector copies, one row per
// (d/8)-thread group, coalesced on both sides within a row; each CTA moves
// 64 rows with every thread's loads issued before its stores.
#include "common.cuh"
#include "internal.h"

namespace salad {
namespace {

// Frame-major index t of space-major position r.
__device__ __forceinline__ int sm_to_fm(int r, int F, int Hh, int Wh) {
  const int f = r % F;
  const int pos = r / F;
  const int y = pos / Wh, x = pos % Wh;
  return (f * Hh + y) * Wh + x;
}

// Rows copied per CTA, and rows each thread keeps in flight.
constexpr int kRowsPerCta = 64;

// CTA (row block, slab): destination rows [64 x, 64 x + 64) of slab s.
// inverse = 0: dst[s][r] = src[s][t(r)]; inverse = 1: dst[s][t(r)] = src[s][r].
// Thread (rsub, chunk) moves 16-byte chunk `chunk` of rows rsub, rsub + RPI,
// ... with all its loads issued before its stores.
template <int CPR>
__global__ void __launch_bounds__(256) permute_kernel(const uint4* __restrict__ src,
                                                      uint4* __restrict__ dst, int N, int F,
                                                      int Hh, int Wh, int inverse) {
  constexpr int RPI = 256 / CPR;
  constexpr int U = kRowsPerCta / RPI;
  const long long base = static_cast<long long>(blockIdx.y) * N;
  const int chunk = threadIdx.x % CPR, rsub = threadIdx.x / CPR;
  const int r0 = blockIdx.x * kRowsPerCta;
  uint4 v[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int r = r0 + rsub + u * RPI;
    if (r < N) {
      const int from = inverse ? r : sm_to_fm(r, F, Hh, Wh);
      v[u] = __ldcs(src + (base + from) * CPR + chunk);
    }
  }
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int r = r0 + rsub + u * RPI;
    if (r < N) {
      const int to = inverse ? sm_to_fm(r, F, Hh, Wh) : r;
      dst[(base + to) * CPR + chunk] = v[u];
    }
  }
}

struct HeadList {
  int n;
  short heads[256];
};

// dst_x[b][i][r] = src_x[b][heads[i]][t(r)] for x in {q, k, v} (blockIdx.z).
// CTA (row block, b * n + i, x), the same row-block scheme as permute_kernel.
template <int CPR>
__global__ void __launch_bounds__(256) gather_sm_kernel(
    const uint4* __restrict__ q, const uint4* __restrict__ k, const uint4* __restrict__ v,
    uint4* __restrict__ qp, uint4* __restrict__ kp, uint4* __restrict__ vp, int H, int N, int F,
    int Hh, int Wh, const __grid_constant__ HeadList L) {
  constexpr int RPI = 256 / CPR;
  constexpr int U = kRowsPerCta / RPI;
  const uint4* src = blockIdx.z == 0 ? q : (blockIdx.z == 1 ? k : v);
  uint4* dst = blockIdx.z == 0 ? qp : (blockIdx.z == 1 ? kp : vp);
  const int slab = blockIdx.y;   // b * n + i
  const int i = slab % L.n, b = slab / L.n;
  const uint4* s = src + (static_cast<long long>(b) * H + L.heads[i]) * N * CPR;
  uint4* d = dst + static_cast<long long>(slab) * N * CPR;
  const int chunk = threadIdx.x % CPR, rsub = threadIdx.x / CPR;
  const int r0 = blockIdx.x * kRowsPerCta;
  uint4 val[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int r = r0 + rsub + u * RPI;
    if (r < N) val[u] = __ldcs(s + static_cast<long long>(sm_to_fm(r, F, Hh, Wh)) * CPR + chunk);
  }
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int r = r0 + rsub + u * RPI;
    if (r < N) d[static_cast<long long>(r) * CPR + chunk] = val[u];
  }
}

}  // namespace

cudaError_t launch_permute(const Ctx& c, const void* src, void* dst, int S, int N, int d, int F,
                           int Hh, int Wh, int inverse) {
  const dim3 grid((N + kRowsPerCta - 1) / kRowsPerCta, S);
  if (d == 128)
    permute_kernel<16><<<grid, 256, 0, c.stream>>>(static_cast<const uint4*>(src),
                                                   static_cast<uint4*>(dst), N, F, Hh, Wh, inverse);
  else
    permute_kernel<8><<<grid, 256, 0, c.stream>>>(static_cast<const uint4*>(src),
                                                  static_cast<uint4*>(dst), N, F, Hh, Wh, inverse);
  return cudaGetLastError();
}

cudaError_t launch_gather_heads_space_major(const Ctx& c, const void* q, const void* k,
                                            const void* v, void* qp, void* kp, void* vp, int B,
                                            int H, int N, int d, int F, int Hh, int Wh,
                                            const int* sel, int nsel) {
  HeadList L;
  L.n = nsel;
  for (int i = 0; i < nsel && i < 256; ++i) L.heads[i] = static_cast<short>(sel[i]);
  const dim3 grid((N + kRowsPerCta - 1) / kRowsPerCta, B * nsel, 3);
  auto qq = static_cast<const uint4*>(q), kk = static_cast<const uint4*>(k),
       vv = static_cast<const uint4*>(v);
  auto qd = static_cast<uint4*>(qp), kd = static_cast<uint4*>(kp), vd = static_cast<uint4*>(vp);
  if (d == 128)
    gather_sm_kernel<16><<<grid, 256, 0, c.stream>>>(qq, kk, vv, qd, kd, vd, H, N, F, Hh, Wh, L);
  else
    gather_sm_kernel<8><<<grid, 256, 0, c.stream>>>(qq, kk, vv, qd, kd, vd, H, N, F, Hh, Wh, L);
  return cudaGetLastError();
}

}  // namespace salad
