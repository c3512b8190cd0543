// permute.cu -- token regrouping of the spatio-temporal sliding-window heads.
//
// "视频扩散模型中的稀疏注意力机制解析 (ijyty.com)" 1.1: the 3-D latent is
// flattened with time slowest, t = (f*Hh + y)*Wh + x, so one spatial
// position's frames sit Hh*Wh apart; heads with temporal locality regroup the
// tokens by spatial position, r = (y*Wh + x)*F + f, before the 1-D window.
// Pure data movement (HBM-bound): 16-byte vector copies, one row per
// (d/8)-thread group, coalesced on both sides within a row.
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

__global__ void permute_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int N,
                               int CPR, int F, int Hh, int Wh, int inverse, long long total) {
  const long long q = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (q >= total) return;
  const int chunk = static_cast<int>(q % CPR);
  const long long row = q / CPR;
  const long long s = row / N;
  const int r = static_cast<int>(row % N);
  const int t = sm_to_fm(r, F, Hh, Wh);
  const long long base = s * N;
  if (!inverse)
    dst[(base + r) * CPR + chunk] = __ldcs(src + (base + t) * CPR + chunk);
  else
    dst[(base + t) * CPR + chunk] = __ldcs(src + (base + r) * CPR + chunk);
}

struct HeadList {
  int n;
  short heads[256];
};

// dst_x[b][i][r] = src_x[b][heads[i]][t(r)] for x in {q, k, v} (blockIdx.y).
__global__ void gather_sm_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k,
                                 const uint4* __restrict__ v, uint4* __restrict__ qp,
                                 uint4* __restrict__ kp, uint4* __restrict__ vp, int B, int H,
                                 int N, int CPR, int F, int Hh, int Wh,
                                 const __grid_constant__ HeadList L) {
  const long long total = static_cast<long long>(B) * L.n * N * CPR;
  const long long qi = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (qi >= total) return;
  const uint4* src = blockIdx.y == 0 ? q : (blockIdx.y == 1 ? k : v);
  uint4* dst = blockIdx.y == 0 ? qp : (blockIdx.y == 1 ? kp : vp);
  const int chunk = static_cast<int>(qi % CPR);
  const long long row = qi / CPR;
  const int r = static_cast<int>(row % N);
  const long long slab = row / N;  // b * n + i
  const int i = static_cast<int>(slab % L.n);
  const int b = static_cast<int>(slab / L.n);
  const int t = sm_to_fm(r, F, Hh, Wh);
  const long long sidx = ((static_cast<long long>(b) * H + L.heads[i]) * N + t) * CPR + chunk;
  dst[qi] = __ldcs(src + sidx);
}

}  // namespace

cudaError_t launch_permute(const Ctx& c, const void* src, void* dst, int S, int N, int d, int F,
                           int Hh, int Wh, int inverse) {
  const int CPR = d / 8;
  const long long total = static_cast<long long>(S) * N * CPR;
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  permute_kernel<<<static_cast<unsigned>(blocks), threads, 0, c.stream>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), N, CPR, F, Hh, Wh, inverse, total);
  return cudaGetLastError();
}

cudaError_t launch_gather_heads_space_major(const Ctx& c, const void* q, const void* k,
                                            const void* v, void* qp, void* kp, void* vp, int B,
                                            int H, int N, int d, int F, int Hh, int Wh,
                                            const int* sel, int nsel) {
  HeadList L;
  L.n = nsel;
  for (int i = 0; i < nsel && i < 256; ++i) L.heads[i] = static_cast<short>(sel[i]);
  const int CPR = d / 8;
  const long long total = static_cast<long long>(B) * nsel * N * CPR;
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  gather_sm_kernel<<<dim3(static_cast<unsigned>(blocks), 3), threads, 0, c.stream>>>(
      static_cast<const uint4*>(q), static_cast<const uint4*>(k), static_cast<const uint4*>(v),
      static_cast<uint4*>(qp), static_cast<uint4*>(kp), static_cast<uint4*>(vp), B, H, N, CPR, F,
      Hh, Wh, L);
  return cudaGetLastError();
}

}  // namespace salad
