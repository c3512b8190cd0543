// gate.cu -- the input-aware scalar gate of the hybrid layer.
//
// "SALAD ... (paper.rainbus.top)" 方法步骤详情 step 5 and "视频扩散模型中的稀疏
// 注意力机制解析" 2.3: average the hidden state over tokens, apply a linear map
// and a sigmoid:  s_b = sigmoid(w . mean_n X[b, n, :] + bias).
// Because the map is linear, w . mean_n X = (1/N) sum_{n,c} w_c X[b,n,c]: one
// streaming pass over X (the only HBM traffic), a per-CTA partial in float32,
// then a fixed-order float64 sum of the partials (deterministic: the
// partition depends only on B, N, D and the SM count).
#include "common.cuh"
#include "internal.h"

namespace salad {
namespace {

constexpr int kGateThreads = 256;
constexpr int kGateUnroll = 4;

__device__ __forceinline__ float dot8(const uint4& xv, const uint4& wv) {
  const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w};
  const uint32_t ws[4] = {wv.x, wv.y, wv.z, wv.w};
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 a = unpack_bf16x2(xs[i]);
    float2 b = unpack_bf16x2(ws[i]);
    acc = fmaf(a.x, b.x, acc);
    acc = fmaf(a.y, b.y, acc);
  }
  return acc;
}

// grid (ctas_per_b, B).  X[b] is read as a flat run of 16-byte chunks; chunk
// q covers columns 8*(q % CD) .. +7 with CD = D / 8.
__global__ void __launch_bounds__(kGateThreads) gate_partial_kernel(
    const uint4* __restrict__ x, const uint4* __restrict__ w, long long chunks_per_b, int CD,
    float* __restrict__ partial) {
  const int b = blockIdx.y;
  const uint4* xb = x + static_cast<long long>(b) * chunks_per_b;
  const long long stride = static_cast<long long>(gridDim.x) * kGateThreads;
  long long q = static_cast<long long>(blockIdx.x) * kGateThreads + threadIdx.x;
  int col = static_cast<int>(q % CD);
  const int col_step = static_cast<int>(stride % CD);
  float acc = 0.f;
  // Main loop: kGateUnroll independent loads in flight per thread.
  for (; q + (kGateUnroll - 1) * stride < chunks_per_b; q += kGateUnroll * stride) {
    uint4 xv[kGateUnroll];
    int cs[kGateUnroll];
#pragma unroll
    for (int u = 0; u < kGateUnroll; ++u) {
      xv[u] = __ldcs(xb + q + u * stride);
      cs[u] = col;
      col += col_step;
      if (col >= CD) col -= CD;
    }
#pragma unroll
    for (int u = 0; u < kGateUnroll; ++u) acc += dot8(xv[u], __ldg(w + cs[u]));
  }
  for (; q < chunks_per_b; q += stride) {
    acc += dot8(__ldcs(xb + q), __ldg(w + col));
    col += col_step;
    if (col >= CD) col -= CD;
  }
  // Block reduction (fixed order).
  __shared__ float red[kGateThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int i = 0; i < kGateThreads / 32; ++i) t += red[i];
    partial[static_cast<long long>(b) * gridDim.x + blockIdx.x] = t;
  }
}

// Column-resident variant, used when D/8 is a multiple of 32 and at most
// 1024: thread c owns 16-byte column chunk c of every row, so its 8 weights
// stay in registers; CTA (part, b) streams rows [part*rows_per, ...) of X[b]
// with kGateRowUnroll independent 16-byte loads in flight per thread.
constexpr int kGateRowUnroll = 16;
__global__ void gate_rows_kernel(const uint4* __restrict__ x, const uint4* __restrict__ w, int N,
                                 int rows_per, float* __restrict__ partial) {
  const int CD = blockDim.x;
  const int b = blockIdx.y;
  const int c = threadIdx.x;
  const uint4 wv = __ldg(w + c);
  const int r0 = blockIdx.x * rows_per;
  const int r1 = min(N, r0 + rows_per);
  const uint4* xb = x + (static_cast<long long>(b) * N) * CD + c;
  float acc = 0.f;
  int r = r0;
  for (; r + kGateRowUnroll <= r1; r += kGateRowUnroll) {
    uint4 xv[kGateRowUnroll];
#pragma unroll
    for (int u = 0; u < kGateRowUnroll; ++u)
      xv[u] = __ldcs(xb + static_cast<long long>(r + u) * CD);
#pragma unroll
    for (int u = 0; u < kGateRowUnroll; ++u) acc += dot8(xv[u], wv);
  }
  for (; r < r1; ++r) acc += dot8(__ldcs(xb + static_cast<long long>(r) * CD), wv);
  // Block reduction (fixed order).
  __shared__ float red[32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int i = 0; i < CD / 32; ++i) t += red[i];
    partial[static_cast<long long>(b) * gridDim.x + blockIdx.x] = t;
  }
}

bool gate_rows_ok(int D) { return D % 256 == 0 && D / 8 <= 1024; }

// Row-split CTAs per sample for gate_rows_kernel: about as many CTAs as fit
// on the device at once, at least 8 rows each.
int gate_rows_parts(int B, int N, int D, int num_sms) {
  const int per_sm = 2048 / (D / 8);
  long long want = (static_cast<long long>(num_sms) * (per_sm > 0 ? per_sm : 1) + B - 1) / B;
  const long long cap = (N + 7) / 8;
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  return static_cast<int>(want);
}

__global__ void gate_final_kernel(const float* __restrict__ partial, int nparts, int N,
                                  float bias, float* __restrict__ s) {
  const int b = blockIdx.x;
  __shared__ double red[32];
  double acc = 0.0;
  for (int i = threadIdx.x; i < nparts; i += blockDim.x)
    acc += static_cast<double>(partial[static_cast<long long>(b) * nparts + i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < static_cast<int>(blockDim.x) / 32; ++i) t += red[i];
    const double z = t / static_cast<double>(N) + static_cast<double>(bias);
    s[b] = static_cast<float>(1.0 / (1.0 + exp(-z)));
  }
}

__global__ void fill_f32_kernel(float* dst, float value, int n) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = value;
}

int gate_ctas_per_b(int B, int N, int D, int num_sms) {
  const long long chunks = static_cast<long long>(N) * (D / 8);
  long long want = (chunks + kGateThreads * kGateUnroll - 1) / (kGateThreads * kGateUnroll);
  long long cap = (static_cast<long long>(num_sms) * 8 + B - 1) / B;  // ~8 CTAs per SM overall
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  return static_cast<int>(want);
}

}  // namespace

size_t gate_ws_bytes(int B, int N, int D) {
  // Sized for the largest grid either kernel can pick on a part with up to
  // 256 SMs, independent of the device.
  const int parts = gate_rows_ok(D) ? gate_rows_parts(B, N, D, 256) : gate_ctas_per_b(B, N, D, 256);
  return align256(static_cast<size_t>(B) * parts * sizeof(float));
}

// Enqueues the partial-sum kernel and the final kernel with the partial sums
// in `partial`.  At most `max_parts_total` partials (B x parts) are used: the
// regular gate passes its workspace's capacity, which its partition never
// exceeds, so the cap only binds for the fixed array of the allocation-free
// variant.
cudaError_t launch_gate_parts(const Ctx& c, const void* x, const void* w, float bias, int B,
                              int N, int D, float* s, float* partial, long long max_parts_total) {
  const int sms = c.num_sms < 256 ? c.num_sms : 256;
  const long long cap = max_parts_total / B > 0 ? max_parts_total / B : 1;
  int nparts;
  if (gate_rows_ok(D)) {
    nparts = gate_rows_parts(B, N, D, sms);
    if (nparts > cap) nparts = static_cast<int>(cap);
    // Whole unrolled groups per CTA; no empty CTA.
    const int rows_per = ((N + nparts - 1) / nparts + kGateRowUnroll - 1) / kGateRowUnroll * kGateRowUnroll;
    nparts = (N + rows_per - 1) / rows_per;
    gate_rows_kernel<<<dim3(nparts, B), D / 8, 0, c.stream>>>(
        static_cast<const uint4*>(x), static_cast<const uint4*>(w), N, rows_per, partial);
  } else {
    nparts = gate_ctas_per_b(B, N, D, sms);
    if (nparts > cap) nparts = static_cast<int>(cap);
    const long long chunks_per_b = static_cast<long long>(N) * (D / 8);
    gate_partial_kernel<<<dim3(nparts, B), kGateThreads, 0, c.stream>>>(
        static_cast<const uint4*>(x), static_cast<const uint4*>(w), chunks_per_b, D / 8, partial);
  }
  gate_final_kernel<<<B, 256, 0, c.stream>>>(partial, nparts, N, bias, s);
  return cudaGetLastError();
}

cudaError_t launch_gate(const Ctx& c, const void* x, const void* w, float bias, int B, int N,
                        int D, float* s, void* ws) {
  return launch_gate_parts(c, x, w, bias, B, N, D, s, static_cast<float*>(ws),
                           static_cast<long long>(gate_ws_bytes(B, N, D) / sizeof(float)));
}

cudaError_t launch_fill_f32(const Ctx& c, float* dst, float value, int n) {
  fill_f32_kernel<<<(n + 255) / 256, 256, 0, c.stream>>>(dst, value, n);
  return cudaGetLastError();
}

}  // namespace salad

// ---------------------------------------------------------------------------
// Gate without caller-provided scratch.
//
// For callers that cannot allocate device memory at all -- code that runs
// inside a host that owns every allocation (a plug-in handed only its input
// and output buffers), or code on a path where an allocator call is not
// allowed -- the gate's per-CTA partial sums live in this file-scope device
// array instead of a workspace.  The array is part of the library image: every
// GPU that loads the library holds it (64 KB) until the process exits.
// ---------------------------------------------------------------------------
#include <mutex>

#include "salad.h"

namespace salad {
namespace {

constexpr int kNoAllocMaxBatch = 256;        // largest B the array serves
constexpr int kNoAllocFloats = 16384;        // partial sums the array holds (64 KB)
static_assert(kNoAllocFloats / kNoAllocMaxBatch >= 64, "at least 64 partial sums per sample");

static __device__ __align__(256) float g_gate_scratch[kNoAllocFloats];

struct NoAllocDev {
  bool ready = false;
  bool supported = false;
  int num_sms = 0;
  float* scratch = nullptr;   // device address of g_gate_scratch on this device
};
NoAllocDev g_noalloc_dev[64];
std::mutex g_noalloc_mu;

// One-time set-up per device, with that device current: look up the device
// address of the array (its host-side name is only a stand-in).
salad_status noalloc_setup(int dev, NoAllocDev** out) {
  if (dev < 0 || dev >= 64) return SALAD_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocDev& d = g_noalloc_dev[dev];
  if (!d.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return SALAD_ERR_CUDA;
    d.supported = (major == 10 && minor == 0);
    d.num_sms = sms;
    if (d.supported) {
      float* ptr = nullptr;
      if (cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_gate_scratch) != cudaSuccess)
        return SALAD_ERR_CUDA;
      d.scratch = ptr;
    }
    d.ready = true;
  }
  if (!d.supported) return SALAD_ERR_UNSUPPORTED;
  *out = &d;
  return SALAD_OK;
}

}  // namespace
}  // namespace salad

extern "C" salad_status salad_gate_noalloc(const void* x, const void* w, float bias, int B, int N,
                                           int D, float* s, salad_stream stream) {
  using namespace salad;
  if (B < 1 || N < 1 || D < 8 || D % 8 != 0) return SALAD_ERR_INVALID_ARG;
  if (B > kNoAllocMaxBatch) return SALAD_ERR_INVALID_ARG;   // beyond the array's capacity
  const uintptr_t ax = reinterpret_cast<uintptr_t>(x), aw = reinterpret_cast<uintptr_t>(w),
                  as = reinterpret_cast<uintptr_t>(s);
  if (x == nullptr || w == nullptr || s == nullptr || ax % 16 || aw % 16 || as % 4)
    return SALAD_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SALAD_ERR_CUDA;
  NoAllocDev* d = nullptr;
  const salad_status st = noalloc_setup(dev, &d);
  if (st != SALAD_OK) return st;
  // The same partition as salad_gate whenever its B x parts partial sums fit
  // the array (then the result is bit-identical); otherwise fewer parts per
  // sample, which changes only the float32 rounding of the partial sums.
  // Every partial slot the final kernel reads is written first by this
  // call's partial kernel, so nothing needs clearing between calls.
  Ctx c;
  c.stream = static_cast<cudaStream_t>(stream);
  c.err = nullptr;
  c.num_sms = d->num_sms;
  c.wait_ns = 0;
  if (launch_gate_parts(c, x, w, bias, B, N, D, s, d->scratch, kNoAllocFloats) != cudaSuccess)
    return SALAD_ERR_CUDA;
  return SALAD_OK;
}
