/*
 * salad.h -- C ABI of the SALAD hybrid-attention forward library (sm_100a).
 *
 * SALAD runs two attention branches on shared Q, K, V and mixes them with a
 * gated, projected residual:
 *     O = O_sparse + s_b * ((phi(Q) H / (phi(Q) Z + eps)) W_lin[h])
 * with phi = ReLU, H = phi(K)^T V, Z = phi(K)^T 1 and
 * s_b = sigmoid(w . mean_tokens(X[b]) + bias).
 * Sources, by page title and section:
 *   "SALAD ... (paper.rainbus.top)": 前置知识 (sparse mask, linear attention),
 *       方法步骤详情 steps 2-6 (parallel branches, zero-init projection, gate,
 *       residual sum).
 *   "视频扩散模型中的稀疏注意力机制解析 (ijyty.com)": 1.1 (ST-SWA token
 *       regrouping + sliding window), 1.2 (Top-K block selection from block
 *       means), 2.3 (gate: token mean, linear, sigmoid).
 *
 * Conventions shared by every entry point
 *   - Tensors Q, K, V, O are bf16, contiguous, [B, H, N, d] with the exact
 *     token count N (no caller padding).  d must be 64 or 128; the block
 *     size must be 64.  N must be in [1, 262144].
 *   - All tensor pointers are DEVICE pointers, 16-byte aligned, owned by the
 *     caller.  Pointers documented as HOST are read during the call only.
 *   - The library never allocates or frees device memory and never
 *     synchronises.  Scratch memory is a caller-provided device workspace
 *     whose size is returned by the matching *_workspace_bytes query;
 *     256-byte alignment is required.  salad_forward alone creates, on its
 *     first call on each caller stream, two streams and three events of its
 *     own (kept until the process exits) to run independent steps side by
 *     side.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) in call order.  All argument checks run on the host before any
 *     launch: an invalid call returns an error and enqueues nothing.
 *   - Waits inside the kernels are bounded.  A wait that runs out sets a
 *     device-side error word instead of trapping; salad_check_error() reads
 *     it (and is the only call that synchronises).
 */
#ifndef SALAD_H_
#define SALAD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int salad_status;
#define SALAD_OK                0
#define SALAD_ERR_INVALID_ARG  (-1)   /* null pointer, bad size, misaligned */
#define SALAD_ERR_UNSUPPORTED  (-2)   /* d not in {64,128}, block != 64, no sm_100 device */
#define SALAD_ERR_CUDA         (-3)   /* a CUDA runtime call or launch failed */
#define SALAD_ERR_TIMEOUT      (-4)   /* a bounded device-side wait ran out */
#define SALAD_ERR_WORKSPACE    (-5)   /* workspace missing, too small or misaligned */

/* Sparse-branch patterns. */
#define SALAD_MODE_TOPK   0   /* Top-K block-sparse (ijyty.com 1.2) */
#define SALAD_MODE_SWA    1   /* spatio-temporal sliding window (ijyty.com 1.1) */
#define SALAD_MODE_DENSE  2   /* every key (the full-attention special case) */

typedef void* salad_stream;   /* cudaStream_t */

/* Human-readable text of a status code; never NULL. */
const char* salad_status_string(salad_status status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int salad_version(void);

/*
 * Gate (paper.rainbus.top 方法步骤详情 step 5; ijyty.com 2.3):
 *   s[b] = sigmoid( sum_c w[c] * (1/N) sum_n x[b,n,c] + bias ).
 * x: bf16 [B, N, D] device; w: bf16 [D] device; s: float32 [B] device (out).
 * D must be a multiple of 8.  Workspace: salad_gate_workspace_bytes(B, N, D).
 */
size_t salad_gate_workspace_bytes(int B, int N, int D);
salad_status salad_gate(const void* x, const void* w, float bias, int B, int N, int D,
                        float* s, void* workspace, size_t workspace_bytes,
                        salad_stream stream);

/*
 * Gate with no scratch argument, for callers that cannot allocate device
 * memory at all (a plug-in that receives only its input and output buffers,
 * or code on a path where an allocator call is not permitted).  No passage of
 * the paper corresponds to it.  It keeps its per-CTA partial sums in a fixed
 * 64 KB array inside the library (present on every GPU that loads the
 * library, until the process exits) instead of a caller workspace.
 *   - Result: the value salad_gate computes, from the same kernels and the
 *     same partition of the tokens whenever that partition's B x parts
 *     partial sums fit the array's 16384 floats -- on a 148-SM B200 that
 *     holds for every accepted B, N and D, and the two results are then
 *     bit-identical.  (Were it not to fit, fewer parts per sample would be
 *     used, which changes only the float32 rounding of the partial sums.)
 *   - B may be at most 256; larger batches return SALAD_ERR_INVALID_ARG
 *     before any launch.  Other arguments as for salad_gate.
 *   - The first call on each device looks up the array's device address;
 *     make that first call before capturing the stream into a CUDA graph.
 *   - All calls share the one array, and each call overwrites the slots it
 *     reads, so no clearing is needed -- but two calls whose kernels overlap
 *     on the GPU (different streams without ordering) race on it.
 *   - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library.
 */
salad_status salad_gate_noalloc(const void* x, const void* w, float bias, int B, int N, int D,
                                float* s, salad_stream stream);

/*
 * Top-K block selection (ijyty.com 1.2): split tokens into blocks of `block`
 * rows, average each block over its valid rows (float64), score every
 * query-block mean against every key-block mean (float64 dot product), keep
 * the `topk` largest per query block (ties: lower block index first).
 * q, k: bf16 [B, H, N, d] device.  idx: int32 [B, H, nb, topk] device (out),
 * nb = ceil(N/block), each row in ascending block order.  1 <= topk <= nb.
 * The float64 decision is reached by tensor-core scores of a two-term bf16
 * split of the means with a certified error bound, and a float64 rescoring
 * of the blocks the bound leaves undecided (the bound assumes float32
 * accumulation in the tensor core no worse than float32 additions).
 * Workspace: salad_select_workspace_bytes(B, H, N, d, block); it holds the
 * float32 score matrix [B, H, nb, ceil(nb/128)*128] among others.
 */
size_t salad_select_workspace_bytes(int B, int H, int N, int d, int block);
salad_status salad_select_blocks(const void* q, const void* k, int B, int H, int N, int d,
                                 int block, int topk, int32_t* idx,
                                 void* workspace, size_t workspace_bytes,
                                 salad_stream stream);

/*
 * Linear-attention state (paper.rainbus.top 前置知识 Linear Attention):
 *   Hst[b,h] = relu(K[b,h])^T V[b,h]   float32 [B, H, d, d] device (out)
 *   Z[b,h]   = relu(K[b,h])^T 1        float32 [B, H, d]    device (out)
 * Hst is row-major: Hst[b,h][c][j] = sum_n relu(k[n][c]) v[n][j].
 * Workspace: salad_linear_state_workspace_bytes(B, H, N, d).
 */
size_t salad_linear_state_workspace_bytes(int B, int H, int N, int d);
salad_status salad_linear_state(const void* k, const void* v, int B, int H, int N, int d,
                                float* Hst, float* Z, void* workspace, size_t workspace_bytes,
                                salad_stream stream);

/*
 * Linear-attention output (paper.rainbus.top 前置知识 Linear Attention, the
 * output phi(Q) H / (phi(Q) Z) of the state above; 方法步骤详情 step 3, the
 * linear branch on the layer's own Q):
 *   o_lin[b,h,n,:] = relu(q) Hst / (relu(q) . Z + eps).
 * eps (>= 0, finite) keeps a row with relu(q) = 0 at zero instead of 0/0.
 * q: bf16 [B,H,N,d] device; Hst, Z: float32 device, as produced by
 * salad_linear_state; o_lin: bf16 [B,H,N,d] device (out), must not overlap q.
 * Needs no workspace.  Errors: SALAD_ERR_INVALID_ARG for a null or
 * misaligned pointer, a bad size or eps; nothing is enqueued then.
 */
salad_status salad_linear_apply(const void* q, const float* Hst, const float* Z, float eps,
                                int B, int H, int N, int d, void* o_lin, salad_stream stream);

/*
 * Token permutation of the ST-SWA heads (ijyty.com 1.1).  The latent grid
 * F x Hh x Wh (N = F*Hh*Wh) is flattened frame-major, t = (f*Hh + y)*Wh + x;
 * the space-major order is r = (y*Wh + x)*F + f.
 * src, dst: bf16 [S, N, d] device, S = number of (batch, head) slabs,
 * 1 <= S <= 65535.
 * inverse = 0: dst[s][r] = src[s][t(r)] (frame-major -> space-major);
 * inverse = 1: dst[s][t(r)] = src[s][r] (space-major -> frame-major).
 * src and dst must not overlap.
 */
salad_status salad_permute_tokens(const void* src, void* dst, int S, int N, int d,
                                  int F, int Hh, int Wh, int inverse, salad_stream stream);

/*
 * Sparse branch alone: normalised softmax attention over the pattern,
 * o_sparse = softmax(Q K^T / sqrt(d) + M) V, bf16 [B,H,N,d] (out).
 *   mode SALAD_MODE_TOPK : M keeps, for query block i, the key blocks
 *                          idx[b,h,i,0..topk) (device int32, ascending).
 *   mode SALAD_MODE_SWA  : M keeps |r - c| <= window in each head's order;
 *                          heads with space_major_heads[h] != 0 (HOST uint8
 *                          [H], may be NULL = none) are regrouped
 *                          space-major with the (F, Hh, Wh) grid and their
 *                          output rows are returned in frame-major order.
 *   mode SALAD_MODE_DENSE: every key.
 * Workspace: salad_sparse_attn_workspace_bytes(...).
 */
size_t salad_sparse_attn_workspace_bytes(int B, int H, int N, int d, int mode, int topk,
                                         const uint8_t* space_major_heads);
salad_status salad_sparse_attn(const void* q, const void* k, const void* v,
                               int B, int H, int N, int d, int mode, int block, int topk,
                               const int32_t* idx, int window,
                               const uint8_t* space_major_heads, int F, int Hh, int Wh,
                               void* o_sparse, void* workspace, size_t workspace_bytes,
                               salad_stream stream);

/*
 * Dense flash attention on the same shapes (the comparator the method is
 * measured against): o = softmax(Q K^T / sqrt(d)) V, bf16 [B,H,N,d] (out).
 * Needs no workspace.
 */
salad_status salad_dense_attn(const void* q, const void* k, const void* v,
                              int B, int H, int N, int d, void* o, salad_stream stream);

/*
 * Full-width projection of concatenated heads with a gated residual
 * (paper.rainbus.top 方法步骤详情 step 4, the linear branch's projection read
 * as one layer over all heads, and step 7, the output projection):
 *   out[b,n,:] = resid[b,n,:] + s_b * (A_cat[b,n,:] W)
 * A: bf16 [B,H,N,d] device; A_cat[b,n, h*d + c] = A[b,h,n,c] (the heads of a
 * token concatenated, head-major; no copy is made).  W: bf16 row-major
 * [H*d, n_out] device, n_out a positive multiple of 64.
 * out_per_head = 1: out (and resid) are bf16 [B,H,N,d] (n_out must equal
 *   H*d; column h*d + c of a token is out[b,h,n,c]).
 * out_per_head = 0: out (and resid) are bf16 [B,N,n_out], token-major.
 * resid: device, same layout as out, or NULL (no residual).  It may be the
 *   same pointer as out (in place); otherwise it must not overlap out.
 * s: device float32 [B] or NULL (s_b = 1).  Samples with s_b < drop_threshold
 *   are skipped: their out is not written (0 or NaN never skips).
 * out must not overlap A or W.  Needs no workspace.  tcgen05 GEMM with fp32
 * accumulation; the result is rounded once to bf16.
 */
salad_status salad_project(const void* a, int B, int H, int N, int d, const void* w, int n_out,
                           void* out, int out_per_head, const void* resid, const float* s,
                           float drop_threshold, salad_stream stream);

/*
 * The whole hybrid layer (paper.rainbus.top 方法步骤详情 steps 2-6, 8):
 * gate, sparse branch, linear branch, per-head projection W_lin (d x d,
 * right-multiplying row vectors: O_l' = O_l W_lin[h]), gated residual sum.
 * The sparse pattern runs on `stream`; the gate and the linear branch run on
 * two streams of the library forked from `stream` by an event and joined
 * back to it before the attention kernel, so all work is ordered after the
 * caller's earlier work on `stream` and before its later work.
 * Reentrant: each caller stream gets its own two side streams and fork/join
 * events (created by the first call on that stream -- make it before the
 * stream is captured into a CUDA graph -- and kept until the process exits;
 * up to 32 caller streams per device, after which a call enqueues every step
 * on `stream` itself, in order).  So calls from several threads on different
 * streams neither wait for one another on the host nor depend on one another
 * on the GPU; calls on the same stream are serialised while they enqueue.
 * Concurrent calls must not share a workspace or an output buffer.
 */
typedef struct salad_forward_args {
    const void* q;              /* bf16 [B,H,N,d] device */
    const void* k;              /* bf16 [B,H,N,d] device */
    const void* v;              /* bf16 [B,H,N,d] device */
    const void* x;              /* bf16 [B,N,D] device: gate input (time-modulated hidden state) */
    const void* w_gate;         /* bf16 [D] device */
    float gate_bias;
    const void* w_lin;          /* bf16 [H,d,d] device */
    void* o;                    /* bf16 [B,H,N,d] device (out) */
    int B, H, N, d, D;
    int mode;                   /* SALAD_MODE_* */
    int block;                  /* must be 64 */
    int topk;                   /* TOPK mode: key blocks per query block, 1..nb */
    int window;                 /* SWA mode: half-width, >= 0 */
    const uint8_t* space_major_heads;  /* SWA mode: HOST uint8 [H] or NULL */
    int F, Hh, Wh;              /* SWA mode: latent grid, F*Hh*Wh == N */
    float eps;                  /* linear-attention denominator eps (1e-6) */
    float gate_override;        /* NaN: use the gate; otherwise s_b = this value */
    /* Post-training branch dropping ("SALAD ... (paper.rainbus.top)" 方法步骤详情
     * step 8; "视频扩散模型中的稀疏注意力机制解析" 3.1-3.2): the linear branch
     * of sample b (state, fold and linear term) is skipped, on the device,
     * when s_b < drop_threshold; that sample's output is then O_sparse.  The
     * threshold is calibrated offline (a percentile of gate values).  0 or
     * NaN: never drop.  +-inf is rejected. */
    float drop_threshold;
    /* 3-D rotary position encoding in the linear branch ("SALAD ...
     * (paper.rainbus.top)" 方法步骤详情 step 3): 1 = on, 0 = off.  Adjacent
     * channel pairs of phi(q) and phi(k) turn by the token's frame, row and
     * column positions on the F x Hh x Wh grid (F*Hh*Wh == N required; the
     * tokens are frame-major) over three channel groups of d - 4*floor(d/6),
     * 2*floor(d/6), 2*floor(d/6) channels, pair i of a g-channel group at
     * rate rope_base^(-2i/g).  The rotation enters the numerator only:
     * O_l = (R phi(q)) H_R / (phi(q) Z + eps) with H_R = sum_j R_j phi(k_j) v_j^T
     * and Z = sum_j phi(k_j). */
    int rope3d;
    float rope_base;            /* > 1, usually 10000 */
    /* Full-width projection of the linear branch (paper.rainbus.top 方法步骤详情
     * step 4 read as one layer over all heads): bf16 [H*d, H*d] device, or
     * NULL for the per-head w_lin.  When set, w_lin is not read and
     *   O[b,:,n,:] = O_sparse + s_b * split_heads(cat_heads(O_l[b,:,n,:]) w_lin_full)
     * with cat_heads putting column h*d + c = O_l[b,h,n,c] (see
     * salad_project).  With rope3d, O_l carries the rotation as above. */
    const void* w_lin_full;
    /* Output projection (step 7): bf16 [H*d, d_out] device, or NULL.  When
     * set, out[b,n,:] = cat_heads(O[b,:,n,:]) w_out is written too; o still
     * receives O. */
    const void* w_out;
    int d_out;                  /* multiple of 64 when w_out is set */
    void* out;                  /* bf16 [B,N,d_out] device (out) when w_out is set */
    float* s_out;               /* optional device float32 [B] (out), may be NULL */
    int32_t* idx_out;           /* optional device int32 [B,H,nb,topk] (out), may be NULL */
    void* workspace;            /* device scratch, >= salad_forward_workspace_bytes() */
    size_t workspace_bytes;
    /* Optional profiling hook: NULL, or a HOST array of 5 cudaEvent_t,
     * recorded at the start (on `stream`), when the gate ends, when the
     * sparse-pattern step (selection or regrouping) ends, when the attention
     * kernel starts (every input ready), and when it ends (the full-width
     * projections, if any, follow that last event).  The gate and the
     * linear branch run on two library-owned streams forked from `stream`
     * and joined back before the attention, so only the last two events
     * bound one kernel. */
    void* const* phase_events;
    /* SWA mode, heads regrouped space-major ("视频扩散模型中的稀疏注意力机制解析
     * (ijyty.com)" 1.1): 0 (default) copies their Q, K, V space-major into
     * the workspace first; 1 regroups them inside the attention's TMA loads
     * instead (no copy): their work items and key tiles are floor(128/F)
     * whole spatial positions, floor(128/F)*F of the 128 MMA rows (requires
     * F <= 128, else SALAD_ERR_UNSUPPORTED).  Same results within rounding
     * (frame-major heads bit-identical); no copy workspace.  On a B200 the
     * copy is faster (480p ST-SWA layer: 1.02 ms with the copy, 1.63 ms in
     * the loads), so 1 exists for memory-tight callers. */
    int regroup_in_load;
} salad_forward_args;

size_t salad_forward_workspace_bytes(const salad_forward_args* args);
salad_status salad_forward(const salad_forward_args* args, salad_stream stream);

/*
 * Reads and clears the device-side error word after synchronising `stream`.
 * Returns SALAD_ERR_TIMEOUT if any kernel gave up a bounded wait since the
 * last check; SALAD_ERR_CUDA if the stream reports an error or a kernel
 * refused to run (the attention kernel does when its dynamic shared memory
 * is not 1024-byte aligned); else SALAD_OK.
 */
salad_status salad_check_error(salad_stream stream);

/*
 * Test hook for the bounded-wait machinery: launches one CTA that waits on
 * an mbarrier nothing will ever arrive on, with a limit of `timeout_ns`
 * nanoseconds, then records SALAD_ERR_TIMEOUT in the device error word and
 * exits.  Used to check that a wait which runs out surfaces as an error
 * status rather than a hang or a trap.
 */
salad_status salad_debug_wait_timeout(unsigned long long timeout_ns, salad_stream stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* SALAD_H_ */
