// internal.h -- launch wrappers shared between the kernel files and the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace salad {

// Per-call launch context.
struct Ctx {
  cudaStream_t stream;
  unsigned* err;              // device error word
  int num_sms;
  unsigned long long wait_ns; // limit of every bounded device wait
};

// Round up to a multiple of 256 bytes (workspace carve-up alignment).
inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// ---- gate (gate.cu)
size_t gate_ws_bytes(int B, int N, int D);
cudaError_t launch_gate(const Ctx& c, const void* x, const void* w, float bias, int B, int N,
                        int D, float* s, void* ws);
cudaError_t launch_fill_f32(const Ctx& c, float* dst, float value, int n);

// ---- block selection (select.cu)
size_t select_ws_bytes(int B, int H, int N, int d, int block);
// Kept lists idx [B,H,nb,topk] (ascending; may be null) and, when lists is
// not null, the pair unions of launch_pair_union in the same launch.
// `pooled` (optional) is recorded on c.stream once the pooling pass, the
// chain's only full read of Q and K, has been enqueued.
cudaError_t launch_select(const Ctx& c, const void* q, const void* k, int B, int H, int N, int d,
                          int topk, int32_t* idx, void* ws, int32_t* lists = nullptr,
                          int32_t* counts = nullptr, cudaEvent_t pooled = nullptr);
// Merge the kept lists of query blocks (2p, 2p+1) into one ascending list of
// entries (j | mask << 16), mask bit 0 = block 2p keeps j, bit 1 = block 2p+1.
size_t pairs_ws_bytes(int B, int H, int N, int topk);
cudaError_t launch_pair_union(const Ctx& c, const int32_t* idx, int BH, int nb, int topk,
                              int32_t* lists, int32_t* counts);

// ---- linear branch (linear.cu)
size_t linear_state_ws_bytes(int B, int H, int N, int d);
// Hst = phi(K)^T V and Z = phi(K)^T 1 per (b, h).  With w_lin given, also
// G[b,h] = Hst[b,h] W_lin[h], written as bf16 MMA B-operand images
// [B*H][d*d] (K-major over the row index of G, 128-byte swizzle) into Gimg.
// 3-D rotary encoding of the linear branch: adjacent channel pairs (2m,
// 2m+1) of phi(q) and phi(k) turn by angle pos * theta[m], pos being the
// token's frame, row or column on the F x Hh x Wh grid for the first gt2
// pairs, the next gy2 pairs and the remaining pairs.  on == 0: no encoding.
struct Rope3D {
  int on = 0;
  int F = 0, Hh = 0, Wh = 0;
  int gt2 = 0, gy2 = 0;
  double theta[64] = {};
};
// theta[m] = base^(-2i/g) for pair i of a group of g channels.
Rope3D make_rope3d(int d, int F, int Hh, int Wh, float base);

#ifdef __CUDACC__
// (cos, sin) of the angle of pair m for a token at frame f, row y, column x.
// The angle pos * theta[m] is formed and reduced modulo 2 pi in float64 (its
// error stays near 1e-11 rad for every position the library accepts); the
// reduced angle in [-pi, pi] is turned by the CUDA intrinsic __sincosf,
// accurate to about 2^-21 absolute there.
__device__ __forceinline__ float2 rope_cs(const Rope3D& r, const double* theta, int m, int f,
                                          int y, int x) {
  const int pos = m < r.gt2 ? f : (m < r.gt2 + r.gy2 ? y : x);
  const double a = static_cast<double>(pos) * theta[m];
  const double k = rint(a * 0.15915494309189535);     // a / (2 pi), rounded
  const float red = static_cast<float>(fma(-k, 6.283185307179586, a));
  float sn, cs;
  __sincosf(red, &sn, &cs);
  return make_float2(cs, sn);
}
#endif

// Post-training branch dropping on the device: sample b's linear branch is
// skipped when its gate value (s[b], or gate_override when s is null) is
// below thr.  thr = 0 or NaN never drops (gate values are >= 0).
struct BranchDrop {
  const float* s = nullptr;
  float gate_override = 0.0f;
  float thr = 0.0f;
};
cudaError_t launch_linear_state(const Ctx& c, const void* k, const void* v, int B, int H, int N,
                                int d, float* Hst, float* Z, void* ws,
                                const void* w_lin = nullptr, void* Gimg = nullptr,
                                BranchDrop drop = BranchDrop(), Rope3D rope = Rope3D());
cudaError_t launch_linear_apply(const Ctx& c, const void* q, const float* Hst, const float* Z,
                                float eps, int B, int H, int N, int d, void* o,
                                Rope3D rope = Rope3D());

// ---- permutation (permute.cu)
cudaError_t launch_permute(const Ctx& c, const void* src, void* dst, int S, int N, int d, int F,
                           int Hh, int Wh, int inverse);
// Gather the listed heads (host list, nsel <= 256) of Q, K, V [B,H,N,d] into
// space-major slabs [B,nsel,N,d].
cudaError_t launch_gather_heads_space_major(const Ctx& c, const void* q, const void* k,
                                            const void* v, void* qp, void* kp, void* vp, int B,
                                            int H, int N, int d, int F, int Hh, int Wh,
                                            const int* sel, int nsel);

// ---- attention (attn.cu)
enum AttnMode : int { kModeTopk = 0, kModeBand = 1, kModeDense = 2 };

struct AttnArgs {
  // Frame-major inputs [B,H,N,d] and, for space-major heads, the regrouped
  // copies [B,Hs,N,d] (may be null when no head is regrouped).
  const void* q;
  const void* k;
  const void* v;
  const void* qp;
  const void* kp;
  const void* vp;
  const int* head_slot;       // HOST [H] (or null): slot in the regrouped copies or -1
  int B, H, N, d, Hs;
  int mode;                   // AttnMode
  int window;                 // band half-width
  int F, Hh, Wh;              // grid of the regrouped heads
  // > 0: the regrouped heads are read inside the attention's loads, items
  // and key tiles of floor(regroup_rows / F) whole positions (regroup_rows
  // <= 128, >= F); qp, kp, vp are then unused.
  int regroup_rows;
  const int32_t* lists;       // topk: [B*H*npairs][2*topk] entries j | mask<<16
  const int32_t* counts;      // topk: [B*H*npairs]
  int list_stride;            // 2*topk
  // Hybrid epilogue (null Gimg = plain normalised attention output).
  const void* Gimg;           // bf16 images [B*H][d*d] of Hst W_lin (see launch_linear_state)
  const float* Z;             // [B,H,d]
  const float* s;             // [B] gate values (device)
  float gate_override;        // used when s is null
  float drop = 0.0f;          // the linear term of sample b is skipped when s_b < drop
  Rope3D rope;                // 3-D rotary encoding of phi(Q) in the linear term
  float eps;
  void* o;                    // bf16 [B,H,N,d]
};
cudaError_t launch_attention(const Ctx& c, const AttnArgs& a);

// Debug: one CTA waits on an mbarrier nothing arrives on, bounded.
cudaError_t launch_debug_wait(const Ctx& c);

// Tensor map for a bf16 [S, N, d] tensor viewed as 3-D (d, N, S), box
// (64, 64, 1), 128-byte swizzle.  Returns false on failure.
bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, int S, int N, int d);
// The same view with a box of (64, rows, 1), rows <= 256.
bool make_tmap_bf16_3d_rows(CUtensorMap* map, const void* base, int S, int N, int d, int rows);
bool make_tmap_bf16_heads4d(CUtensorMap* map, const void* base, int B, int H, int N, int d);
// Frame-major [S][F * npos][d] bf16 (token t = f npos + p) viewed as 4-D
// (d, F, npos, S) with the frame dimension first: box (64, F, box_pos, 1)
// lands box_pos whole positions, F rows each, in space-major order.
bool make_tmap_bf16_regroup(CUtensorMap* map, const void* base, int S, int F, int npos, int d,
                            int box_pos);
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, int rows, int cols);

// ---- full-width projections (proj.cu)
// out = resid + s_b * (A_cat W) per sample b, where A_cat [N][H*d] is A
// [B][H][N][d] with the heads of a token concatenated (column h*d + c) and W
// is row-major [H*d][n_out].  out (and resid, if given) is per-head [B][H][N][d]
// when n_out == H*d and out_per_head, else token-major [B][N][n_out].  s null:
// scale 1.  Samples with s_b < drop are skipped (out must equal resid then).
struct ProjArgs {
  const void* a;
  int B, H, N, d;
  const void* w;
  int n_out;
  void* out;
  int out_per_head;
  const void* resid;
  const float* s;
  float drop;
};
cudaError_t launch_proj(const Ctx& c, const ProjArgs& a);

}  // namespace salad
