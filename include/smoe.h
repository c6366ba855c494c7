/*
 * smoe.h -- C ABI of libsmoe.so: a sparse Mixture-of-Experts (SMoE) MLP and its
 * building block ParallelLinear for NVIDIA B200 (sm_100a).
 *
 * The method is ScatterMoE ("Scattered Mixture-of-Experts Implementation",
 * arXiv 2403.08245).  Its pages define the operations only in prose:
 *   [abs]  arXiv abstract: an SMoE implementation built on ParallelLinear that
 *          avoids padding and excessive copies of the input; extended to Mixture
 *          of Attention.
 *   [rev1] library page of arXiv 2403.08245, review 1 summary: ParallelLinear lets
 *          the input and the output each be grouped or scattered, and serves both
 *          the forward and the backward pass, without copying or padding.
 *   [rev2] same page, review 2 summary: the scatter2scatter kernel covers
 *          group-to-group, group-to-scatter, scatter-to-scatter and
 *          scatter-to-group, fusing grouped GEMMs with scattered reads and writes.
 *   [art]  tradepoint.io article "This Machine Learning Research Presents
 *          ScatterMoE", method paragraphs: grouped matrix operations on scattered
 *          groups; prior work needs a scatter-to-group copy of the input and pads
 *          it; the backward pass computes the gradient of each expert.
 *   [src]  sourcepulse.org project summary, "How It Works": expert linear
 *          transforms are fused with the reordering operations.
 *
 * Conventions (all entry points):
 *   - Row-major tensors.  Weights are [E, K, N] (K input features, N output
 *     features): y = x W[e].  Indices are int32, gates fp32.
 *   - dtype SMOE_BF16: x, W, activations and outputs in bf16, fp32 accumulation,
 *     weight gradients in fp32.  SMOE_F32: everything fp32.
 *   - Slots: token t's j-th selected expert is slot p = t*k + j.  "Scattered"
 *     rows are in token/slot order; "grouped" rows are in expert-sorted order:
 *     grouped row i holds slot sorted_slot[i], and expert e owns grouped rows
 *     [expert_offsets[e], expert_offsets[e+1]).
 *   - Pointers are device pointers unless stated otherwise; the caller owns all
 *     memory.  The library never allocates device memory: scratch space is the
 *     caller's workspace, sized by the *_workspace_size queries (256-byte aligned
 *     start required).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream)
 *     and never synchronised, except by smoe_check.
 *   - Return value: SMOE_OK or a negative smoe_status.  Argument errors are found
 *     on the host before any launch and leave outputs untouched; the message is
 *     available from smoe_last_error() (thread-local).  T == 0 is a no-op.
 *   - Data errors found on the device (an expert id outside [0, E), inconsistent
 *     offsets) never trap: the kernel skips the bad element and records the error
 *     in a per-device error word that smoe_check reports.
 *   - Alignment: d, f, K and N must be multiples of 8 (16-byte rows for the
 *     tensor-memory-accelerator copies); every tensor start 16-byte aligned.
 *   - Several calls may run concurrently on different streams as long as they
 *     do not share workspaces or outputs.
 *   - Size limits (checked on the host, SMOE_ERR_INVALID_ARG beyond them):
 *       routed entry points (smoe_route, smoe_route_bwd, smoe_mlp_*):
 *         1 <= k <= min(E, SMOE_MAX_TOPK), E <= SMOE_MAX_ROUTED_EXPERTS;
 *       sort and ParallelLinear (smoe_sort, smoe_sort_static,
 *         parallel_linear_*): E <= SMOE_MAX_EXPERTS;
 *       everywhere: T * k (the slot count) <= INT32_MAX, and every [rows, cols]
 *         tensor the call touches has fewer than 2^31 elements.
 */
#ifndef SMOE_H_
#define SMOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SMOE_OK = 0,
  SMOE_ERR_INVALID_ARG = -1, /* bad pointer, size, alignment or flag combination */
  SMOE_ERR_UNSUPPORTED = -2, /* valid request this build does not implement (e.g. no sm_100 GPU) */
  SMOE_ERR_CUDA = -3,        /* a CUDA runtime/driver call failed (message has the CUDA error) */
  SMOE_ERR_DATA = -4,        /* device-detected bad index data (reported by smoe_check) */
  SMOE_ERR_TIMEOUT = -5      /* a bounded device-side wait gave up (reported by smoe_check) */
} smoe_status;

typedef enum { SMOE_F32 = 0, SMOE_BF16 = 1 } smoe_dtype;

#define SMOE_MAX_ROUTED_EXPERTS 128 /* E for the router and the MLP */
#define SMOE_MAX_TOPK 16            /* k for the router and the MLP */
#define SMOE_MAX_EXPERTS 1024       /* E for the sort and ParallelLinear */

typedef enum {
  SMOE_ACT_GELU_TANH = 0, /* a = 0.5 h (1 + tanh(sqrt(2/pi) (h + 0.044715 h^3))) */
  SMOE_ACT_SWIGLU = 1,    /* a = silu(h_gate) * h_up, silu(z) = z / (1 + exp(-z)) */
  SMOE_ACT_NONE = 2
} smoe_act;

/* ---------------------------------------------------------------------------
 * Status
 * ------------------------------------------------------------------------ */

/* Message of the last failing call on this host thread ("" if none). */
const char* smoe_last_error(void);

/* Synchronises `stream`, then reads and clears the calling device's error word.
 * Returns SMOE_OK, SMOE_ERR_DATA, SMOE_ERR_TIMEOUT or SMOE_ERR_CUDA. */
int smoe_check(void* stream);

/* Library version string. */
const char* smoe_version(void);

/* ---------------------------------------------------------------------------
 * Workspace queries (bytes; 0 means no workspace needed)
 * ------------------------------------------------------------------------ */
typedef enum {
  SMOE_OP_SORT = 0,
  SMOE_OP_PL_FWD = 1,
  SMOE_OP_PL_BWD = 2,
  SMOE_OP_MLP_FWD = 3,
  SMOE_OP_MLP_BWD = 4,
  SMOE_OP_ROUTE_BWD = 5
} smoe_op;

/* Upper bound of the workspace for `op` on an SMoE layer of T tokens, width d,
 * expert width f, E experts, top-k.  For the ParallelLinear ops it bounds every
 * flag combination with num_slots = T*k, K and N in {d, f, 2f}. */
size_t smoe_workspace_size(int op, int T, int k, int E, int d, int f, smoe_dtype dt);

/* ---------------------------------------------------------------------------
 * Routing [abs, art: top-k SMoE layer; router definition: softmax, top-k,
 * renormalised gates]
 *
 * smoe_route: logits l[t,e] = sum_i x[t,i] W_r[i,e] (+ b_r[e]) in fp32 in this
 * documented order: lane L of a 32-lane group accumulates, in ascending i, the
 * products for every i with i % 32 == L as acc = fmaf(x, w, acc) from +0;
 * the 32 lane sums are combined by an xor butterfly with offsets 16, 8, 4, 2, 1;
 * then b_r[e] is added.  The k largest logits are selected (descending; equal
 * logits go to the lower expert id) and gates[t,j] = softmax over the k
 * selected logits (this equals softmax over all E, top-k, renormalise).
 *   x        [T, d] dtype          w_r [d, E] dtype        b_r [E] fp32 or NULL
 *   topk_idx [T, k] int32 (out)    gates [T, k] fp32 (out)
 * Requires 1 <= k <= min(E, 16), E <= 128, d % 8 == 0.
 * ------------------------------------------------------------------------ */
int smoe_route(const void* x, const void* w_r, const float* b_r, int T, int d, int E, int k,
               smoe_dtype dt, int32_t* topk_idx, float* gates, void* stream);

/* smoe_route_bwd: gradient through the renormalised softmax of smoe_route.
 *   dl[t,j] = gates[t,j] (dgates[t,j] - sum_i gates[t,i] dgates[t,i]) for the
 *   selected expert e = topk_idx[t,j], 0 for unselected experts;
 *   dw_r[i,e] = sum_t x[t,i] dl[t,e]  (fp32, overwritten; summed in token order in
 *                                      runs of 32-128 expert-sorted slots, the runs
 *                                      then in order: fixed by T, k, d, E, routing)
 *   db_r[e]   = sum_t dl[t,e]         (fp32, overwritten; NULL to skip)
 *   dx[t,i]  += sum_j dl[t,j] W_r[i, topk_idx[t,j]]  (dtype, accumulated into dx;
 *                                                     NULL to skip)
 * workspace: smoe_workspace_size(SMOE_OP_ROUTE_BWD, ...) bytes (no more than the
 * SMOE_OP_MLP_BWD size of the same shape).
 * Requires 1 <= k <= min(E, 16), E <= 128, d % 8 == 0 (as smoe_route).       */
int smoe_route_bwd(const void* x, const void* w_r, const int32_t* topk_idx, const float* gates,
                   const float* dgates, int T, int d, int E, int k, smoe_dtype dt, void* dx,
                   float* dw_r, float* db_r, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Reordering [src: "reordering operations"; rev1: grouped = expert-sorted]
 *
 * smoe_sort: stable sort of the T*k slots by expert id (ties by slot index) and
 * the exclusive prefix sum of per-expert counts.
 *   topk_idx [T, k] int32   sorted_slot [T*k] int32 (out)
 *   expert_offsets [E+1] int32 (out; offsets[0] = 0, offsets[E] = T*k)
 * Ids outside [0, E) are reported through smoe_check (SMOE_ERR_DATA) and their
 * slots are left out (the outputs are then incomplete).  Requires 1 <= E <= 1024.
 * ------------------------------------------------------------------------ */
int smoe_sort(const int32_t* topk_idx, int T, int k, int E, int32_t* sorted_slot,
              int32_t* expert_offsets, void* workspace, size_t ws_bytes, void* stream);

/* smoe_sort_static: the same stable sort and offsets as smoe_sort, for callers
 * that cannot allocate device memory for a workspace -- for example a runtime
 * that plans all device memory up front and gives its kernels only their inputs
 * and outputs, or code running while a CUDA graph is being captured, where a
 * cudaMalloc would synchronise the device or escape the graph.  This entry point
 * calls no allocator.  (The paper has no counterpart; it is a calling
 * convention of this library.)
 *   Scratch: a fixed 256 KB device array inside the library (held by every GPU
 *   that loads the library until the process exits) stores the per-block expert
 *   counts, so ceil(T*k / 4096) * E must be <= 65536; larger problems are
 *   rejected with SMOE_ERR_INVALID_ARG and a message (use smoe_sort).
 *   The first call on a device looks up the array's device address with that
 *   device current; make that first call before any stream capture begins.
 *   The address is kept for the life of the process, so the library must not
 *   be used across a cudaDeviceReset (or any other teardown of the device's
 *   primary context) that unloads and reloads its module.
 *   Every call rewrites all the counts it uses, so nothing has to be cleared
 *   between calls; but all calls share the one array, so calls whose work
 *   overlaps on the GPU (different streams without ordering) race and give
 *   wrong results.  Serialise them (one stream, or events).
 * Arguments, outputs and data-error reporting are those of smoe_sort.          */
int smoe_sort_static(const int32_t* topk_idx, int T, int k, int E, int32_t* sorted_slot,
                     int32_t* expert_offsets, void* stream);

/* smoe_selftest_wait_timeout: a check of the failure path (no counterpart on the
 * pages).  Launches one small kernel whose thread waits, through the same bounded
 * wait that every pipeline barrier of the GEMM kernels uses, on a barrier that
 * nothing completes.  After limit_us microseconds (0 < limit_us <= 1e6) the wait
 * gives up and records the timeout in the device error word, exactly as a stalled
 * GEMM pipeline would; the next smoe_check on the stream returns SMOE_ERR_TIMEOUT
 * and clears the word.  Nothing faults and nothing hangs: a caller or a test can
 * confirm that a device-side stall becomes an error status on the host.
 * Returns SMOE_OK once the kernel is launched, SMOE_ERR_INVALID_ARG for a limit
 * out of range, SMOE_ERR_CUDA for a launch error. */
int smoe_selftest_wait_timeout(int limit_us, void* stream);

/* ---------------------------------------------------------------------------
 * ParallelLinear [rev1, rev2, art]
 *
 * For every grouped row i of expert e, with p = sorted_slot[i]:
 *   input row   : x[i]                 if grouped_in
 *                 x[p / fan_out]       otherwise (fan_out = k for token-shaped
 *                                      x [T, K]; 1 for slot-shaped x [T*k, K])
 *   v           = g * x_row W[e]       g = gates[p] if gates != NULL, else 1
 *   output      : y[i] = v             if grouped_out           (y [num_slots, N])
 *                 y[p] = v             if scattered, combine_k == 0 (y [num_slots, N])
 *                 y[p / combine_k] = sum of the combine_k slots' v, in slot
 *                                      order (combine_k > 0, scattered only;
 *                                      y [num_slots / combine_k, N])
 * No grouped or padded copy of a scattered input is made.  The k-way combine is
 * deterministic (no atomics): this library rounds each slot's (gated) v to dtype
 * (its own choice: the pages do not say how per-slot outputs are held), then sums
 * the combine_k values in fp32 in slot order.
 *   x [x_rows, K] dtype, w [E, K, N] dtype, y dtype.  Requires 1 <= E <= 1024.
 * ------------------------------------------------------------------------ */
size_t parallel_linear_fwd_workspace_size(int num_slots, int K, int N, int E, int combine_k,
                                          smoe_dtype dt);
int parallel_linear_fwd(const void* x, int x_rows, int K, const void* w, int N, int E,
                        const int32_t* sorted_slot, const int32_t* expert_offsets, int num_slots,
                        int fan_out, int grouped_in, int grouped_out, const float* gates,
                        int combine_k, void* y, smoe_dtype dt, void* workspace, size_t ws_bytes,
                        void* stream);

/* Backward of parallel_linear_fwd against dy (shaped like its y).  With
 * G_i = dy[p / combine_k] (combine) or dy[output row of i]:
 *   dx[input row of i] += g G_i W[e]^T   (dx [x_rows, K] dtype, overwritten; NULL to skip)
 *   dw[e] = sum_i x_row(i)^T (g G_i)     (dw [E, K, N] fp32, overwritten, zero for an
 *                                         empty expert; NULL to skip)
 *   dgates[p] = <G_i, x_row(i) W[e]>     (fp32 [num_slots]; only with gates; NULL to skip)
 * `gates` must be the forward's gates (NULL if the forward had none).         */
size_t parallel_linear_bwd_workspace_size(int x_rows, int num_slots, int K, int N, int E,
                                          int fan_out, int grouped_in, int grouped_out,
                                          int has_gates, int combine_k, smoe_dtype dt);
int parallel_linear_bwd(const void* dy, const void* x, const void* w, int x_rows, int K, int N,
                        int E, const int32_t* sorted_slot, const int32_t* expert_offsets,
                        int num_slots, int fan_out, int grouped_in, int grouped_out,
                        const float* gates, int combine_k, void* dx, float* dw, float* dgates,
                        smoe_dtype dt, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Mixture-of-Attention core [abs: ParallelLinear extended to Mixture of
 * Attention; art, method paragraph: MoA without additional memory costs]
 *
 * The attention between the per-expert query projection (ParallelLinear,
 * scatter->group, fan_out kslots) and the per-expert output projection
 * (group->scatter with the gated k-way combine).  The pages give no formula; this
 * library's reading: the T tokens form sequences of L consecutive tokens (the
 * last may be shorter); keys and values are shared by all experts; slot
 * p = t*kslots + j holds token t's query for its j-th selected expert, in grouped
 * order (row i with sorted_slot[i] = p); for every head h of width head_dim:
 *   o[i, h] = sum_u softmax_u(<q[i, h], k[u, h]> / sqrt(head_dim)) v[u, h]
 * over u from the first token of t's sequence to t (causal), and
 *   lse[i, h] = log sum_u exp(<q[i, h], k[u, h]> / sqrt(head_dim)).
 *   q, o [T*kslots, heads*head_dim] dtype, grouped rows;  k, v [T, heads*head_dim]
 *   dtype, token order;  lse [T*kslots, heads] fp32.  Columns of head h are
 *   [h*head_dim, (h+1)*head_dim).
 * No grouped copy is made: the kernels gather query rows through sorted_slot.
 * Requires dt == SMOE_BF16 and head_dim == 128 (else SMOE_ERR_UNSUPPORTED);
 * 1 <= kslots <= 128; L >= 1.  workspace: smoe_moa_attn_workspace_size(T, kslots,
 * heads, backward) bytes, 256-byte aligned (the inverse of sorted_slot, and for
 * the backward D = <dO, O> per row and head).
 * Backward of L = <o, dout>: dq (grouped, like q), dk and dv (token order, like
 * k and v), all overwritten, dtype; summed in a fixed order (no atomics).
 * ------------------------------------------------------------------------ */
size_t smoe_moa_attn_workspace_size(int T, int kslots, int heads, int backward);
int smoe_moa_attn_fwd(const void* q, const void* k, const void* v, const int32_t* sorted_slot, int T,
                      int L, int kslots, int heads, int head_dim, smoe_dtype dt, void* o, float* lse,
                      void* workspace, size_t ws_bytes, void* stream);
int smoe_moa_attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                      const void* dout, const int32_t* sorted_slot, int T, int L, int kslots, int heads,
                      int head_dim, smoe_dtype dt, void* dq, void* dk, void* dv, void* workspace,
                      size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * SMoE MLP [abs, art: SMoE layer = top-k routing + weighted sum of expert MLPs]
 *
 * Forward: route, sort, H = ParallelLinear(x, W1; scatter->group, fan_out k),
 * A = act(H), y = ParallelLinear(A, W2; group->scatter, gated k-way combine).
 * Backward of L = <y, dy>: expert weight gradients, gate gradients, the router
 * gradient (smoe_route_bwd) and dx.
 * ------------------------------------------------------------------------ */
typedef struct {
  int T, d, f, E, k;
  int act;   /* SMOE_ACT_GELU_TANH or SMOE_ACT_SWIGLU */
  int dtype; /* smoe_dtype */
} smoe_mlp_desc;

typedef struct {
  const void* x;    /* [T, d] */
  const void* w_r;  /* [d, E] dtype (router weight) */
  const float* b_r; /* [E] or NULL */
  const void* w1;   /* [E, d, m*f]; SwiGLU (m = 2): columns [0,f) gate, [f,2f) up */
  const void* w2;   /* [E, f, d] */
  /* forward outputs, kept for the backward */
  void* y;                 /* [T, d] */
  int32_t* topk_idx;       /* [T, k] */
  float* gates;            /* [T, k] */
  int32_t* sorted_slot;    /* [T*k] */
  int32_t* expert_offsets; /* [E+1] */
  void* h;                 /* [T*k, m*f] grouped pre-activation */
  void* a;                 /* [T*k, f] grouped activation */
  /* backward inputs / outputs */
  const void* dy; /* [T, d] */
  void* dx;       /* [T, d] (overwritten) */
  float* dw1;     /* [E, d, m*f] fp32 */
  float* dw2;     /* [E, f, d] fp32 */
  float* dw_r;    /* [d, E] fp32 */
  float* db_r;    /* [E] fp32 or NULL */
  float* dgates;  /* [T, k] fp32 or NULL */
  void* workspace;
  size_t workspace_bytes;
} smoe_mlp_tensors;

size_t smoe_mlp_workspace_size(const smoe_mlp_desc* desc, int backward);
int smoe_mlp_fwd(const smoe_mlp_desc* desc, const smoe_mlp_tensors* t, void* stream);
int smoe_mlp_bwd(const smoe_mlp_desc* desc, const smoe_mlp_tensors* t, void* stream);

/* ---------------------------------------------------------------------------
 * FP8 inference forward [src: inference speed as a target of the method]
 *
 * The pages name inference speed but no number format; this library's FP8 path
 * stores expert weights as e4m3 codes (OCP 8-bit float: 4 exponent bits, bias 7,
 * 3 mantissa bits, largest value 448) and runs both expert products on
 * tcgen05.mma kind::f8f6f4 with fp32 accumulation.  Scales are fp32: one per
 * (expert, output column) for the weights, one per row for the activations
 * (x per token, A per slot row after it is stored in bf16); a scale maps its
 * row's or column's largest magnitude to 448 (scale = amax / 448 in fp32, 1 for an
 * all-zero row), and a code is e4m3(fl32(v / scale)), rounded to nearest even.
 *
 * smoe_quantize_weights_fp8: W [E, K, N] bf16 -> codes [E, N, K] uint8 (K-major:
 * row n of expert e holds column n of W[e]) and scales [E, N] fp32.  K % 16 == 0.
 * For the MLP: W1 [E, d, m*f] -> w1q [E, m*f, d], s1 [E, m*f];
 * W2 [E, f, d] -> w2q [E, d, f], s2 [E, d].
 *
 * smoe_mlp_fwd_fp8: the forward of smoe_mlp_fwd with those weights:
 *   h = (x8 . w1q[e]) sx s1[e]  (bf16, grouped, as smoe_mlp_fwd's h),
 *   a = act(h) (bf16), a8 = the row quantisation of a,
 *   y_t = sum_j gates[t,j] (a8 . w2q[e]) sa s2[e].
 * Routing, sort and the deterministic k-way combine are those of smoe_mlp_fwd.
 * Uses desc (dtype must be SMOE_BF16; d % 16 == 0, f % 16 == 0), the routing and
 * activation buffers of t (x, w_r, b_r, y, topk_idx, gates, sorted_slot,
 * expert_offsets, h, a, workspace of smoe_mlp_fp8_workspace_size bytes); t->w1
 * and t->w2 are not read.
 * ------------------------------------------------------------------------ */
typedef struct {
  const uint8_t* w1q; /* [E, m*f, d] e4m3 codes */
  const float* s1;    /* [E, m*f] */
  const uint8_t* w2q; /* [E, d, f] e4m3 codes */
  const float* s2;    /* [E, d] */
} smoe_fp8_weights;

int smoe_quantize_weights_fp8(const void* w, int E, int K, int N, smoe_dtype dt, uint8_t* codes,
                              float* scales, void* stream);
size_t smoe_mlp_fp8_workspace_size(const smoe_mlp_desc* desc);
int smoe_mlp_fwd_fp8(const smoe_mlp_desc* desc, const smoe_mlp_tensors* t, const smoe_fp8_weights* w8,
                     void* stream);

/* smoe_set_gemm_policy: how the tensor-core GEMMs of every later call in this
 * process choose their kernel variant (no counterpart on the pages; every policy
 * computes the same products, bit for bit on the same GPU).
 *   0 (default): one CTA per 128-row tile, 8 gather warps, tiles of an expert in
 *     panels of 16 M tiles.  Measured fastest per step over 20 steps of the
 *     Mixtral-shaped layer under the B200's 1 kW power cap.
 *   1: long-K products (K >= 4096) over large expert slices (at least 2048 rows per
 *     expert on average): TMA-fed ones on 2-CTA pairs sharing M = 256 MMAs,
 *     gathered ones with 4 gather warps, and ungated weight gradients on pairs.
 *     More MMAs per cycle (about 90% against 78% of the tensor pipe on the
 *     TMA-fed products) and about 2.5% less time per step in short runs below the
 *     power cap, but more DRAM traffic: over sustained steps under the cap it
 *     measured equal or slower.
 * Set it between calls, not while a call of this library is in flight.
 * Returns SMOE_OK, or SMOE_ERR_INVALID_ARG for another value. */
int smoe_set_gemm_policy(int policy);

/* ---------------------------------------------------------------------------
 * Instrumentation (the pages have no counterpart; used by the benchmark).
 *
 * smoe_profile_begin: from now on, every kernel launch this library makes from
 * the calling process is bracketed by a pair of CUDA events recorded on the
 * launching stream (at most max_launches brackets; later ones are not timed
 * but still counted).  Events are created here, not per launch.
 * smoe_profile_end: synchronises the recorded events, aggregates per kernel
 * name, stops recording.  smoe_profile_entry then returns, for entry i < the
 * returned count, the kernel name, its launch count and total milliseconds.
 * ------------------------------------------------------------------------ */
int smoe_profile_begin(int max_launches);
int smoe_profile_end(void);
int smoe_profile_entry(int i, const char** name, int* launches, double* total_ms);

#ifdef __cplusplus
}
#endif
#endif /* SMOE_H_ */
