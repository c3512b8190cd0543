// api.cu -- the C ABI declared in include/salad.h: host-side argument checks,
// workspace carve-up, tensor-map creation and the launch sequence of the
// hybrid layer.  Every check runs before the first launch of a call.
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "salad.h"

namespace salad {

// The library's device error word (one per device, read by salad_check_error).
__device__ unsigned g_err_word;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxN = 262144;
constexpr int kMaxHeads = 256;
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;  // 2 s

struct DevInfo {
  bool ready = false;
  bool supported = false;
  int num_sms = 0;
  unsigned* err = nullptr;
};
DevInfo g_dev[kMaxDevices];
std::mutex g_mu;

// salad_forward's side streams and fork/join events, one set per caller
// stream (created on first use, kept until the process exits).  Calls on
// different caller streams use different sets, so they neither wait for each
// other on the host nor gain false dependencies on the GPU, and a stream being
// captured into a CUDA graph never shares a side stream with another caller.
// Calls on the same caller stream are ordered anyway; the set's mutex keeps
// their fork/join records from interleaving.
struct SideSet {
  cudaStream_t caller = nullptr;
  cudaStream_t side[2] = {nullptr, nullptr};
  cudaEvent_t fork = nullptr, join_gate = nullptr, join_lin = nullptr;
  std::mutex enqueue_mu;
};
constexpr int kMaxSideSets = 32;   // per device; beyond this a call runs on one stream
struct SideTable {
  SideSet sets[kMaxSideSets];
  int used = 0;
};
SideTable g_side[kMaxDevices];

// The side set of `caller` on the current device, or null when the table is
// full (the call then enqueues every step on the caller's stream, in order).
// A CUDA failure while creating a set is reported through *cuda_failed.
SideSet* side_resources(cudaStream_t caller, bool* cuda_failed) {
  *cuda_failed = false;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *cuda_failed = true;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  SideTable& t = g_side[dev];
  for (int i = 0; i < t.used; ++i)
    if (t.sets[i].caller == caller) return &t.sets[i];
  if (t.used == kMaxSideSets) return nullptr;
  SideSet& d = t.sets[t.used];
  bool ok = true;
  for (int i = 0; i < 2 && ok; ++i)
    ok = cudaStreamCreateWithFlags(&d.side[i], cudaStreamNonBlocking) == cudaSuccess;
  ok = ok && cudaEventCreateWithFlags(&d.fork, cudaEventDisableTiming) == cudaSuccess &&
       cudaEventCreateWithFlags(&d.join_gate, cudaEventDisableTiming) == cudaSuccess &&
       cudaEventCreateWithFlags(&d.join_lin, cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    for (cudaStream_t& x : d.side)
      if (x != nullptr) { cudaStreamDestroy(x); x = nullptr; }
    for (cudaEvent_t* e : {&d.fork, &d.join_gate, &d.join_lin})
      if (*e != nullptr) { cudaEventDestroy(*e); *e = nullptr; }
    *cuda_failed = true;
    return nullptr;
  }
  d.caller = caller;
  ++t.used;
  return &d;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

unsigned long long wait_limit_ns() {
  const char* s = std::getenv("SALAD_WAIT_NS");
  if (s != nullptr) {
    const unsigned long long v = std::strtoull(s, nullptr, 10);
    if (v > 0) return v;
  }
  return kDefaultWaitNs;
}

// Fills the launch context for the current device.  Returns SALAD_OK, or an
// error when no usable sm_100 device is current.
salad_status get_ctx(salad_stream stream, Ctx* c) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SALAD_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DevInfo& d = g_dev[dev];
  if (!d.ready) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return SALAD_ERR_CUDA;
    d.supported = (prop.major == 10 && prop.minor == 0);
    d.num_sms = prop.multiProcessorCount;
    if (d.supported) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_err_word) != cudaSuccess) return SALAD_ERR_CUDA;
      d.err = static_cast<unsigned*>(p);
    }
    d.ready = true;
  }
  if (!d.supported) return SALAD_ERR_UNSUPPORTED;
  c->stream = static_cast<cudaStream_t>(stream);
  c->err = d.err;
  c->num_sms = d.num_sms;
  c->wait_ns = wait_limit_ns();
  return SALAD_OK;
}

inline bool aligned(const void* p, size_t a) {
  return p != nullptr && (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

inline salad_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SALAD_OK : SALAD_ERR_CUDA; }

// Common shape checks for [B, H, N, d] attention tensors.
salad_status check_bhnd(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1) return SALAD_ERR_INVALID_ARG;
  if (H > kMaxHeads || N > kMaxN) return SALAD_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 65535) return SALAD_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SALAD_ERR_UNSUPPORTED;
  return SALAD_OK;
}

salad_status check_ws(void* ws, size_t have, size_t need) {
  if (need == 0) return SALAD_OK;
  if (ws == nullptr || have < need || !aligned(ws, 256)) return SALAD_ERR_WORKSPACE;
  return SALAD_OK;
}

inline int nblocks(int N) { return (N + 63) / 64; }

// Regrouped (space-major) heads of an SWA call: slots and count.
int space_major_slots(int H, const uint8_t* flags, int* slot) {
  int n = 0;
  for (int h = 0; h < H; ++h) slot[h] = (flags != nullptr && flags[h] != 0) ? n++ : -1;
  return n;
}

}  // namespace

bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, int S, int N, int d) {
  return make_tmap_bf16_3d_rows(map, base, S, N, d, 64);
}

bool make_tmap_bf16_3d_rows(CUtensorMap* map, const void* base, int S, int N, int d, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr || rows < 1 || rows > 256) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(S)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(N) * d * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [B][H][N][d] bf16 viewed as 4-D (d, N, H, B), box 64 x 128 x 1 x 1, 128-byte
// swizzle: one box is 128 token rows of 64 channels of one head.
bool make_tmap_bf16_heads4d(CUtensorMap* map, const void* base, int B, int H, int N, int d) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(N) * d * 2,
                                 static_cast<cuuint64_t>(H) * N * d * 2};
  const cuuint32_t box[4] = {64, 128, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major [rows][cols] bf16 viewed as 2-D (cols, rows), box 64 x 64, 128-byte
// swizzle.
bool make_tmap_bf16_regroup(CUtensorMap* map, const void* base, int S, int F, int npos, int d,
                            int box_pos) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr || F < 1 || F > 256 || box_pos < 1 || box_pos > 256) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(F),
                              static_cast<cuuint64_t>(npos), static_cast<cuuint64_t>(S)};
  // Byte strides of the frame, position and head dimensions.
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(npos) * d * 2,
                                 static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(F) * npos * d * 2};
  const cuuint32_t box[4] = {64, static_cast<cuuint32_t>(F), static_cast<cuuint32_t>(box_pos), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, int rows, int cols) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  const cuuint32_t box[2] = {64, 64};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------- forward layout --
struct FwdLayout {
  size_t gate, s, sel, idx, lists, counts, lin, hst, z, g, olin, qp, kp, vp, total;
  int Hs;
  int slot[kMaxHeads];
};

static FwdLayout forward_layout(const salad_forward_args* a) {
  FwdLayout L;
  std::memset(&L, 0, sizeof(L));
  const size_t B = a->B, H = a->H, N = a->N, d = a->d;
  const size_t nb = static_cast<size_t>(nblocks(a->N));
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  L.gate = take(gate_ws_bytes(a->B, a->N, a->D));
  L.s = take(B * sizeof(float));
  if (a->mode == SALAD_MODE_TOPK) {
    L.sel = take(select_ws_bytes(a->B, a->H, a->N, a->d, 64));
    L.idx = take(B * H * nb * a->topk * sizeof(int32_t));
    const size_t items = B * H * ((nb + 1) / 2);
    L.lists = take(items * 2 * a->topk * sizeof(int32_t));
    L.counts = take(items * sizeof(int32_t));
  }
  L.lin = take(linear_state_ws_bytes(a->B, a->H, a->N, a->d));
  L.hst = take(B * H * d * d * sizeof(float));
  L.z = take(B * H * d * sizeof(float));
  if (a->w_lin_full != nullptr) L.olin = take(B * H * N * d * 2);   // O_l, bf16 [B,H,N,d]
  else L.g = take(B * H * d * d * 2);                                // folded H W_lin images
  L.Hs = 0;
  for (int h = 0; h < kMaxHeads; ++h) L.slot[h] = -1;
  if (a->mode == SALAD_MODE_SWA && a->H <= kMaxHeads)
    L.Hs = space_major_slots(a->H, a->space_major_heads, L.slot);
  if (L.Hs > 0 && !a->regroup_in_load) {   // the space-major copies
    const size_t bytes = B * static_cast<size_t>(L.Hs) * N * d * 2;
    L.qp = take(bytes);
    L.kp = take(bytes);
    L.vp = take(bytes);
  }
  L.total = off;
  return L;
}

}  // namespace salad

using namespace salad;

extern "C" {

const char* salad_status_string(salad_status s) {
  switch (s) {
    case SALAD_OK: return "ok";
    case SALAD_ERR_INVALID_ARG: return "invalid argument";
    case SALAD_ERR_UNSUPPORTED: return "unsupported configuration or device";
    case SALAD_ERR_CUDA: return "CUDA error";
    case SALAD_ERR_TIMEOUT: return "bounded device wait timed out";
    case SALAD_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    default: return "unknown status";
  }
}

int salad_version(void) { return 40200; }

// ------------------------------------------------------------------ gate --
size_t salad_gate_workspace_bytes(int B, int N, int D) {
  if (B < 1 || N < 1 || D < 8) return 0;
  return gate_ws_bytes(B, N, D);
}

salad_status salad_gate(const void* x, const void* w, float bias, int B, int N, int D, float* s,
                        void* workspace, size_t workspace_bytes, salad_stream stream) {
  if (B < 1 || N < 1 || D < 8 || D % 8 != 0 || B > 65535) return SALAD_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(w, 16) || !aligned(s, 4)) return SALAD_ERR_INVALID_ARG;
  salad_status st = check_ws(workspace, workspace_bytes, gate_ws_bytes(B, N, D));
  if (st != SALAD_OK) return st;
  Ctx c;
  if ((st = get_ctx(stream, &c)) != SALAD_OK) return st;
  return from_cuda(launch_gate(c, x, w, bias, B, N, D, s, workspace));
}

// ---------------------------------------------------------------- select --
size_t salad_select_workspace_bytes(int B, int H, int N, int d, int block) {
  if (check_bhnd(B, H, N, d) != SALAD_OK || block != 64) return 0;
  return select_ws_bytes(B, H, N, d, block);
}

salad_status salad_select_blocks(const void* q, const void* k, int B, int H, int N, int d,
                                 int block, int topk, int32_t* idx, void* workspace,
                                 size_t workspace_bytes, salad_stream stream) {
  salad_status st = check_bhnd(B, H, N, d);
  if (st != SALAD_OK) return st;
  if (block != 64) return SALAD_ERR_UNSUPPORTED;
  if (topk < 1 || topk > nblocks(N)) return SALAD_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(idx, 4)) return SALAD_ERR_INVALID_ARG;
  if ((st = check_ws(workspace, workspace_bytes, select_ws_bytes(B, H, N, d, block))) != SALAD_OK)
    return st;
  Ctx c;
  if ((st = get_ctx(stream, &c)) != SALAD_OK) return st;
  return from_cuda(launch_select(c, q, k, B, H, N, d, topk, idx, workspace));
}

// ---------------------------------------------------------------- linear --
size_t salad_linear_state_workspace_bytes(int B, int H, int N, int d) {
  if (check_bhnd(B, H, N, d) != SALAD_OK) return 0;
  return linear_state_ws_bytes(B, H, N, d);
}

salad_status salad_linear_state(const void* k, const void* v, int B, int H, int N, int d,
                                float* Hst, float* Z, void* workspace, size_t workspace_bytes,
                                salad_stream stream) {
  salad_status st = check_bhnd(B, H, N, d);
  if (st != SALAD_OK) return st;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(Hst, 16) || !aligned(Z, 4))
    return SALAD_ERR_INVALID_ARG;
  if ((st = check_ws(workspace, workspace_bytes, linear_state_ws_bytes(B, H, N, d))) != SALAD_OK)
    return st;
  Ctx c;
  if ((st = get_ctx(stream, &c)) != SALAD_OK) return st;
  return from_cuda(launch_linear_state(c, k, v, B, H, N, d, Hst, Z, workspace));
}

salad_status salad_linear_apply(const void* q, const float* Hst, const float* Z, float eps, int B,
                                int H, int N, int d, void* o_lin, salad_stream stream) {
  salad_status st = check_bhnd(B, H, N, d);
  if (st != SALAD_OK) return st;
  if (!aligned(q, 16) || !aligned(Hst, 4) || !aligned(Z, 4) || !aligned(o_lin, 16))
    return SALAD_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return SALAD_ERR_INVALID_ARG;
  Ctx c;
  if ((st = get_ctx(stream, &c)) != SALAD_OK) return st;
  return from_cuda(launch_linear_apply(c, q, Hst, Z, eps, B, H, N, d, o_lin));
}

// ------------------------------------------------------------- project --
static bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const char* x = static_cast<const char*>(a);
  const char* y = static_cast<const char*>(b);
  return x < y + nb && y < x + na;
}

salad_status salad_project(const void* a, int B, int H, int N, int d, const void* w, int n_out,
                           void* out, int out_per_head, const void* resid, const float* s,
                           float drop_threshold, salad_stream stream) {
  salad_status st = check_bhnd(B, H, N, d);
  if (st != SALAD_OK) return st;
  if (n_out < 64 || n_out % 64 != 0 || n_out > 65536) return SALAD_ERR_INVALID_ARG;
  if (out_per_head != 0 && out_per_head != 1) return SALAD_ERR_INVALID_ARG;
  if (out_per_head && n_out != H * d) return SALAD_ERR_INVALID_ARG;
  if (!aligned(a, 16) || !aligned(w, 16) || !aligned(out, 16)) return SALAD_ERR_INVALID_ARG;
  if (resid != nullptr && !aligned(resid, 16)) return SALAD_ERR_INVALID_ARG;
  if (s != nullptr && !aligned(s, 4)) return SALAD_ERR_INVALID_ARG;
  if (std::isinf(drop_threshold)) return SALAD_ERR_INVALID_ARG;
  const size_t a_bytes = static_cast<size_t>(B) * H * N * d * 2;
  const size_t w_bytes = static_cast<size_t>(H) * d * n_out * 2;
  const size_t o_bytes = static_cast<size_t>(B) * N * n_out * 2;
  if (overlaps(out, o_bytes, a, a_bytes) || overlaps(out, o_bytes, w, w_bytes))
    return SALAD_ERR_INVALID_ARG;
  if (resid != nullptr && resid != out && overlaps(out, o_bytes, resid, o_bytes))
    return SALAD_ERR_INVALID_ARG;
  Ctx c;
  if ((st = get_ctx(stream, &c)) != SALAD_OK) return st;
  ProjArgs p;
  p.a = a;
  p.B = B; p.H = H; p.N = N; p.d = d;
  p.w = w;
  p.n_out = n_out;
  p.out = out;
  p.out_per_head = out_per_head;
  p.resid = resid;
  p.s = s;
  p.drop = std::isnan(drop_threshold) ? 0.0f : drop_threshold;
  return from_cuda(launch_proj(c, p));
}

// --------------------------------------------------------------- permute --
salad_status salad_permute_tokens(const void* src, void* dst, int S, int N, int d, int F, int Hh,
                                  int Wh, int inverse, salad_stream stream) {
  if (S < 1 || S > 65535 || N < 1 || F < 1 || Hh < 1 || Wh < 1) return SALAD_ERR_INVALID_ARG;
  if (static_cast<long long>(F) * Hh * Wh != N) return SALAD_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SALAD_ERR_UNSUPPORTED;
  if (!aligned(src, 16) || !aligned(dst, 16) || (inverse != 0 && inverse != 1))
    return SALAD_ERR_INVALID_ARG;
  const size_t bytes = static_cast<size_t>(S) * N * d * 2;
  const char* a = static_cast<const char*>(src);
  const char* b = static_cast<const char*>(dst);
  if (a < b + bytes && b < a + bytes) return SALAD_ERR_INVALID_ARG;  // overlap
  salad_status st;
  Ctx c;
  if ((st = get_ctx(stream, &c)) != SALAD_OK) return st;
  return from_cuda(launch_permute(c, src, dst, S, N, d, F, Hh, Wh, inverse));
}

// ----------------------------------------------------------- sparse attn --
size_t salad_sparse_attn_workspace_bytes(int B, int H, int N, int d, int mode, int topk,
                                         const uint8_t* space_major_heads) {
  if (check_bhnd(B, H, N, d) != SALAD_OK) return 0;
  if (mode == SALAD_MODE_TOPK) {
    if (topk < 1 || topk > nblocks(N)) return 0;
    return pairs_ws_bytes(B, H, N, topk);
  }
  if (mode == SALAD_MODE_SWA) {
    int slot[kMaxHeads];
    const int hs = space_major_slots(H, space_major_heads, slot);
    return 3 * align256(static_cast<size_t>(B) * hs * N * d * 2);
  }
  return 0;
}

salad_status salad_sparse_attn(const void* q, const void* k, const void* v, int B, int H, int N,
                               int d, int mode, int block, int topk, const int32_t* idx,
                               int window, const uint8_t* space_major_heads, int F, int Hh,
                               int Wh, void* o_sparse, void* workspace, size_t workspace_bytes,
                               salad_stream stream) {
  salad_status st = check_bhnd(B, H, N, d);
  if (st != SALAD_OK) return st;
  if (block != 64) return SALAD_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o_sparse, 16))
    return SALAD_ERR_INVALID_ARG;
  if (mode != SALAD_MODE_TOPK && mode != SALAD_MODE_SWA && mode != SALAD_MODE_DENSE)
    return SALAD_ERR_INVALID_ARG;
  int slot[kMaxHeads];
  int Hs = 0;
  if (mode == SALAD_MODE_TOPK) {
    if (topk < 1 || topk > nblocks(N) || !aligned(idx, 4)) return SALAD_ERR_INVALID_ARG;
  } else if (mode == SALAD_MODE_SWA) {
    if (window < 0) return SALAD_ERR_INVALID_ARG;
    Hs = space_major_slots(H, space_major_heads, slot);
    if (Hs > 0 && (F < 1 || Hh < 1 || Wh < 1 || static_cast<long long>(F) * Hh * Wh != N))
      return SALAD_ERR_INVALID_ARG;
  }
  const size_t need =
      salad_sparse_attn_workspace_bytes(B, H, N, d, mode, topk, space_major_heads);
  if ((st = check_ws(workspace, workspace_bytes, need)) != SALAD_OK) return st;
  Ctx c;
  if ((st = get_ctx(stream, &c)) != SALAD_OK) return st;

  AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q = q; a.k = k; a.v = v;
  a.B = B; a.H = H; a.N = N; a.d = d;
  a.window = window; a.F = F; a.Hh = Hh; a.Wh = Wh;
  a.o = o_sparse;
  a.gate_override = 0.f;
  char* ws = static_cast<char*>(workspace);
  if (mode == SALAD_MODE_TOPK) {
    const int nb = nblocks(N);
    const size_t items = static_cast<size_t>(B) * H * ((nb + 1) / 2);
    int32_t* lists = reinterpret_cast<int32_t*>(ws);
    int32_t* counts = reinterpret_cast<int32_t*>(ws + align256(items * 2 * topk * sizeof(int32_t)));
    cudaError_t e = launch_pair_union(c, idx, B * H, nb, topk, lists, counts);
    if (e != cudaSuccess) return SALAD_ERR_CUDA;
    a.mode = kModeTopk;
    a.lists = lists;
    a.counts = counts;
    a.list_stride = 2 * topk;
  } else if (mode == SALAD_MODE_SWA) {
    a.mode = kModeBand;
    if (Hs > 0) {
      const size_t bytes = align256(static_cast<size_t>(B) * Hs * N * d * 2);
      a.qp = ws;
      a.kp = ws + bytes;
      a.vp = ws + 2 * bytes;
      a.Hs = Hs;
      a.head_slot = slot;
      int sel[kMaxHeads];
      for (int h = 0; h < H; ++h)
        if (slot[h] >= 0) sel[slot[h]] = h;
      cudaError_t e = launch_gather_heads_space_major(c, q, k, v, ws, ws + bytes, ws + 2 * bytes,
                                                      B, H, N, d, F, Hh, Wh, sel, Hs);
      if (e != cudaSuccess) return SALAD_ERR_CUDA;
    }
  } else {
    a.mode = kModeDense;
  }
  return from_cuda(launch_attention(c, a));
}

salad_status salad_dense_attn(const void* q, const void* k, const void* v, int B, int H, int N,
                              int d, void* o, salad_stream stream) {
  return salad_sparse_attn(q, k, v, B, H, N, d, SALAD_MODE_DENSE, 64, 0, nullptr, 0, nullptr, 0,
                           0, 0, o, nullptr, 0, stream);
}

// --------------------------------------------------------------- forward --
size_t salad_forward_workspace_bytes(const salad_forward_args* a) {
  if (a == nullptr || check_bhnd(a->B, a->H, a->N, a->d) != SALAD_OK) return 0;
  if (a->D < 8) return 0;
  if (a->mode == SALAD_MODE_TOPK && (a->topk < 1 || a->topk > nblocks(a->N))) return 0;
  return forward_layout(a).total;
}

salad_status salad_forward(const salad_forward_args* a, salad_stream stream) {
  if (a == nullptr) return SALAD_ERR_INVALID_ARG;
  salad_status st = check_bhnd(a->B, a->H, a->N, a->d);
  if (st != SALAD_OK) return st;
  if (a->block != 64) return SALAD_ERR_UNSUPPORTED;
  if (a->mode != SALAD_MODE_TOPK && a->mode != SALAD_MODE_SWA && a->mode != SALAD_MODE_DENSE)
    return SALAD_ERR_INVALID_ARG;
  const bool full = a->w_lin_full != nullptr;
  if (!aligned(a->q, 16) || !aligned(a->k, 16) || !aligned(a->v, 16) || !aligned(a->o, 16) ||
      !aligned(a->x, 16) || !aligned(a->w_gate, 16) ||
      !aligned(full ? a->w_lin_full : a->w_lin, 16))
    return SALAD_ERR_INVALID_ARG;
  if (a->w_out != nullptr && (!aligned(a->w_out, 16) || !aligned(a->out, 16) ||
                              a->d_out < 64 || a->d_out % 64 != 0 || a->d_out > 65536))
    return SALAD_ERR_INVALID_ARG;
  if (a->w_out != nullptr &&
      overlaps(a->out, static_cast<size_t>(a->B) * a->N * a->d_out * 2, a->o,
               static_cast<size_t>(a->B) * a->H * a->N * a->d * 2))
    return SALAD_ERR_INVALID_ARG;
  if (a->D < 8 || a->D % 8 != 0) return SALAD_ERR_INVALID_ARG;
  if (!(a->eps >= 0.0f) || !std::isfinite(a->eps)) return SALAD_ERR_INVALID_ARG;
  if (a->s_out != nullptr && !aligned(a->s_out, 4)) return SALAD_ERR_INVALID_ARG;
  if (a->idx_out != nullptr && !aligned(a->idx_out, 4)) return SALAD_ERR_INVALID_ARG;
  const bool override_gate = !std::isnan(a->gate_override);
  if (override_gate && !std::isfinite(a->gate_override)) return SALAD_ERR_INVALID_ARG;
  if (std::isinf(a->drop_threshold)) return SALAD_ERR_INVALID_ARG;
  if (a->rope3d != 0 && a->rope3d != 1) return SALAD_ERR_INVALID_ARG;
  if (a->rope3d && (a->F < 1 || a->Hh < 1 || a->Wh < 1 ||
                    static_cast<long long>(a->F) * a->Hh * a->Wh != a->N ||
                    !(a->rope_base > 1.0f) || !std::isfinite(a->rope_base)))
    return SALAD_ERR_INVALID_ARG;
  if (a->mode == SALAD_MODE_TOPK && (a->topk < 1 || a->topk > nblocks(a->N)))
    return SALAD_ERR_INVALID_ARG;
  if (a->mode == SALAD_MODE_SWA && a->window < 0) return SALAD_ERR_INVALID_ARG;
  const FwdLayout L = forward_layout(a);
  if (L.Hs > 0 && (a->F < 1 || a->Hh < 1 || a->Wh < 1 ||
                   static_cast<long long>(a->F) * a->Hh * a->Wh != a->N))
    return SALAD_ERR_INVALID_ARG;
  if (a->regroup_in_load != 0 && a->regroup_in_load != 1) return SALAD_ERR_INVALID_ARG;
  // Regrouping in the loads needs a whole position (F rows) per 128-row tile.
  if (L.Hs > 0 && a->regroup_in_load && a->F > 128) return SALAD_ERR_UNSUPPORTED;
  if ((st = check_ws(a->workspace, a->workspace_bytes, L.total)) != SALAD_OK) return st;
  Ctx c;
  if ((st = get_ctx(stream, &c)) != SALAD_OK) return st;

  bool side_failed = false;
  SideSet* dv = side_resources(c.stream, &side_failed);
  if (side_failed) return SALAD_ERR_CUDA;
  // Fork/join on this caller stream's events: enqueues of concurrent calls on
  // the same caller stream must not interleave.  Without a side set (table
  // full) there is nothing to fork: every step goes on the caller's stream.
  std::unique_lock<std::mutex> enqueue_lock;
  if (dv != nullptr) enqueue_lock = std::unique_lock<std::mutex>(dv->enqueue_mu);

  char* ws = static_cast<char*>(a->workspace);
  const int B = a->B, H = a->H, N = a->N, d = a->d;
  const int nb = nblocks(N);
  // Three chains run side by side: the sparse pattern on the caller's
  // stream, the gate and the linear branch on two side streams forked from
  // it; the attention waits for both.  The side chains are joined back even
  // when a launch fails, so the caller's stream never runs ahead of them.
  Ctx cg = c, cl = c;
  if (dv != nullptr) {
    cg.stream = dv->side[0];
    cl.stream = dv->side[1];
  }
  auto mark = [&](int i, cudaStream_t st) -> bool {
    if (a->phase_events == nullptr || a->phase_events[i] == nullptr) return true;
    return cudaEventRecord(static_cast<cudaEvent_t>(a->phase_events[i]), st) == cudaSuccess;
  };
  if (!mark(0, c.stream)) return SALAD_ERR_CUDA;
  bool ok = true;
  auto check = [&](cudaError_t e) { ok = ok && e == cudaSuccess; };
  // Top-K: the selection chain is enqueued first and the side chains fork
  // once its pooling pass has read Q and K.  The pool then has the memory
  // bandwidth to itself, and the gate and the linear branch share it with
  // the scores and the decision instead, which read little (measured: the
  // attention can start 8 us earlier at 480p, 100 us at 720p).
  const bool topk = a->mode == SALAD_MODE_TOPK;
  int32_t* idx = a->idx_out != nullptr ? a->idx_out : reinterpret_cast<int32_t*>(ws + L.idx);
  int32_t* lists = reinterpret_cast<int32_t*>(ws + L.lists);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + L.counts);
  if (topk)
    check(launch_select(c, a->q, a->k, B, H, N, d, a->topk, idx, ws + L.sel, lists, counts,
                        dv != nullptr ? dv->fork : nullptr));
  else if (dv != nullptr && cudaEventRecord(dv->fork, c.stream) != cudaSuccess)
    return SALAD_ERR_CUDA;
  if (dv != nullptr && (cudaStreamWaitEvent(cg.stream, dv->fork, 0) != cudaSuccess ||
                        cudaStreamWaitEvent(cl.stream, dv->fork, 0) != cudaSuccess))
    return SALAD_ERR_CUDA;

  // 1. gate (paper.rainbus.top 方法步骤详情 step 5), side stream 0
  float* s = a->s_out != nullptr ? a->s_out : reinterpret_cast<float*>(ws + L.s);
  if (override_gate) check(launch_fill_f32(cg, s, a->gate_override, B));
  else check(launch_gate(cg, a->x, a->w_gate, a->gate_bias, B, N, a->D, s, ws + L.gate));
  ok = ok && mark(1, cg.stream);
  if (dv != nullptr) check(cudaEventRecord(dv->join_gate, cg.stream));

  AttnArgs at;
  std::memset(&at, 0, sizeof(at));
  at.q = a->q; at.k = a->k; at.v = a->v;
  at.B = B; at.H = H; at.N = N; at.d = d;
  at.window = a->window; at.F = a->F; at.Hh = a->Hh; at.Wh = a->Wh;
  at.o = a->o;
  at.eps = a->eps;
  at.s = s;
  // NaN compares false: never drop.
  at.drop = std::isnan(a->drop_threshold) ? 0.0f : a->drop_threshold;

  // 3. linear branch state and the folded projection G = H W_lin (steps 3-4),
  // side stream 1.  Branch dropping reads the gate's output: only then does
  // this chain wait for the gate.
  float* Hst = reinterpret_cast<float*>(ws + L.hst);
  float* Z = reinterpret_cast<float*>(ws + L.z);
  void* G = ws + L.g;
  BranchDrop drop;   // default: never drop, reads nothing
  if (at.drop > 0.0f) {
    // Only here does this chain read s: it waits for the gate first.
    if (dv != nullptr) check(cudaStreamWaitEvent(cl.stream, dv->join_gate, 0));
    drop.s = s;
    drop.thr = at.drop;
  }
  Rope3D rope;
  if (a->rope3d) rope = make_rope3d(d, a->F, a->Hh, a->Wh, a->rope_base);
  at.rope = rope;
  void* olin = ws + L.olin;
  if (!full) {
    if (ok)
      check(launch_linear_state(cl, a->k, a->v, B, H, N, d, Hst, Z, ws + L.lin, a->w_lin, G, drop,
                                rope));
    at.Gimg = G;
    at.Z = Z;
  } else {
    // Full-width projection: the linear branch stops at O_l; the attention
    // runs plain and the projection GEMM adds s_b (O_l W) afterwards.
    if (ok)
      check(launch_linear_state(cl, a->k, a->v, B, H, N, d, Hst, Z, ws + L.lin, nullptr, nullptr,
                                drop, rope));
    if (ok) check(launch_linear_apply(cl, a->q, Hst, Z, a->eps, B, H, N, d, olin, rope));
  }
  if (dv != nullptr) check(cudaEventRecord(dv->join_lin, cl.stream));

  // 2. sparse-branch pattern (ijyty.com 1.1 / 1.2), the caller's stream
  if (topk) {
    // (enqueued above)
    at.mode = kModeTopk;
    at.lists = lists;
    at.counts = counts;
    at.list_stride = 2 * a->topk;
  } else if (a->mode == SALAD_MODE_SWA) {
    at.mode = kModeBand;
    if (L.Hs > 0 && a->regroup_in_load) {
      // Regrouped inside the attention's loads: whole positions per tile.
      at.regroup_rows = (128 / a->F) * a->F;
      at.Hs = L.Hs;
      at.head_slot = L.slot;
    } else if (L.Hs > 0) {
      int sel[kMaxHeads];
      for (int h = 0; h < H; ++h)
        if (L.slot[h] >= 0) sel[L.slot[h]] = h;
      if (ok)
        check(launch_gather_heads_space_major(c, a->q, a->k, a->v, ws + L.qp, ws + L.kp,
                                              ws + L.vp, B, H, N, d, a->F, a->Hh, a->Wh, sel,
                                              L.Hs));
      at.qp = ws + L.qp;
      at.kp = ws + L.kp;
      at.vp = ws + L.vp;
      at.Hs = L.Hs;
      at.head_slot = L.slot;
    }
  } else {
    at.mode = kModeDense;
  }
  ok = ok && mark(2, c.stream);

  // Join the side chains, then 4. sparse attention with the gated residual
  // epilogue (steps 2, 6).
  const bool joined = dv == nullptr ||
                      (cudaStreamWaitEvent(c.stream, dv->join_gate, 0) == cudaSuccess &&
                       cudaStreamWaitEvent(c.stream, dv->join_lin, 0) == cudaSuccess);
  if (!ok || !joined || !mark(3, c.stream)) return SALAD_ERR_CUDA;
  if (launch_attention(c, at) != cudaSuccess || !mark(4, c.stream)) return SALAD_ERR_CUDA;

  // 5. full-width projections (steps 4 and 7): O += s_b (cat(O_l) W_full) in
  // place, then out = cat(O) W_out.
  if (full) {
    ProjArgs p;
    p.a = olin;
    p.B = B; p.H = H; p.N = N; p.d = d;
    p.w = a->w_lin_full;
    p.n_out = H * d;
    p.out = a->o;
    p.out_per_head = 1;
    p.resid = a->o;
    p.s = s;
    p.drop = at.drop;
    if (launch_proj(c, p) != cudaSuccess) return SALAD_ERR_CUDA;
  }
  if (a->w_out != nullptr) {
    ProjArgs p;
    p.a = a->o;
    p.B = B; p.H = H; p.N = N; p.d = d;
    p.w = a->w_out;
    p.n_out = a->d_out;
    p.out = a->out;
    p.out_per_head = 0;
    p.resid = nullptr;
    p.s = nullptr;
    p.drop = 0.0f;
    if (launch_proj(c, p) != cudaSuccess) return SALAD_ERR_CUDA;
  }
  return SALAD_OK;
}

// ------------------------------------------------------------- errors --
salad_status salad_check_error(salad_stream stream) {
  Ctx c;
  salad_status st = get_ctx(stream, &c);
  if (st != SALAD_OK) return st;
  if (cudaStreamSynchronize(c.stream) != cudaSuccess) return SALAD_ERR_CUDA;
  unsigned word = 0;
  if (cudaMemcpy(&word, c.err, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return SALAD_ERR_CUDA;
  if (word != 0) {
    const unsigned zero = 0;
    if (cudaMemcpy(c.err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return SALAD_ERR_CUDA;
    return (word & kErrTimeout) ? SALAD_ERR_TIMEOUT : SALAD_ERR_CUDA;
  }
  return SALAD_OK;
}

salad_status salad_debug_wait_timeout(unsigned long long timeout_ns, salad_stream stream) {
  if (timeout_ns == 0 || timeout_ns > 10000000000ull) return SALAD_ERR_INVALID_ARG;
  Ctx c;
  salad_status st = get_ctx(stream, &c);
  if (st != SALAD_OK) return st;
  c.wait_ns = timeout_ns;
  return from_cuda(launch_debug_wait(c));
}

}  // extern "C"
