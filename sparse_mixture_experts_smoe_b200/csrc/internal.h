// internal.h -- host-side declarations shared by the translation units of
// libsmoe.so: argument blocks of the grouped GEMMs and the kernel launchers.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "smoe.h"

namespace smoe {

// Bits of the per-device error word (see smoe_check).
enum : unsigned { ERRBIT_DATA = 1u, ERRBIT_TIMEOUT = 2u };

// How grouped row i finds its source row in a row-indexed operand:
//   ROWS_GROUPED: row i;  ROWS_GATHER: row sorted_slot[i] / fan_out.
enum RowMode : int { ROWS_GROUPED = 0, ROWS_GATHER = 1 };

// Epilogues of the grouped-M GEMM.
enum EpiMode : int {
  EPI_STORE = 0,    // out[row] = g * acc                       (g = gates[p] or 1)
  EPI_ACT_FWD = 1,  // out = H = acc (pre-activation), out2 = A = act(H)
  EPI_ACT_BWD = 2   // acc = dA'; dg partial <dA', aux_a>; out2 = g * aux_a; out = g dA' act'(H)
};

// Grouped-M GEMM: for every expert e and grouped row i in [offsets[e], offsets[e+1]):
//   acc[i, n] = sum_k A[src(i), k] * B_e[k, n]
// B_e is W[e] ([K, NW], b_kn = 1) or W[e]^T (W[e] is [NW, K], b_kn = 0).
// For SwiGLU EPI_ACT_FWD the logical output column c uses B columns c (gate) and
// n_out + c (up).
struct GroupedGemm {
  int E = 0;
  int num_rows = 0;
  const int32_t* offsets = nullptr;      // [E+1]
  const int32_t* sorted_slot = nullptr;  // [num_rows]
  int K = 0;
  const void* a = nullptr;
  int lda = 0, a_rows = 0, a_mode = ROWS_GROUPED, a_fan_out = 1;
  const void* b = nullptr;
  int b_kn = 1, NW = 0;
  int epi = EPI_STORE, act = SMOE_ACT_NONE;
  int n_out = 0;
  int out_mode = ROWS_GROUPED;  // ROWS_GROUPED: row i; ROWS_GATHER: row p (fan-out 1)
  void* out = nullptr;
  int ldo = 0, out_f32 = 0;
  void* out2 = nullptr;  // ACT_FWD: A [rows, n_out]; ACT_BWD: g*aux_a grouped (nullable)
  int ldo2 = 0;
  const float* gates = nullptr;  // per slot, nullable
  const void* aux_a = nullptr;   // ACT_BWD: rows dotted with dA' (A, or the forward input)
  int ld_aux_a = 0, aux_a_mode = ROWS_GROUPED, aux_a_fan_out = 1;
  const void* aux_h = nullptr;  // ACT_BWD: H grouped
  int ld_aux_h = 0;
  float* dg_partial = nullptr;  // ACT_BWD: [num_rows, dg_ld], column = N tile index
  int dg_ld = 0;
  // split K (EPI_STORE, grouped A, tensor-core path): ksplit > 1 writes each split's
  // raw fp32 sums to partial [ksplit, num_rows, n_out]; launch_splitk_reduce then
  // applies the gates and stores out
  int ksplit = 1;
  int panel_m = 1 << 30;  // M tiles per raster panel of an expert's tile list (the tensor-core path)
  float* partial = nullptr;
  // fp8 = 1: a and b hold e4m3 codes (b K-major, b_kn = 0); the fp32 sums are
  // multiplied by row_scale[source row of A] and col_scale[e * NW + column]
  int fp8 = 0;
  const float* row_scale = nullptr;
  const float* col_scale = nullptr;
  unsigned* err = nullptr;
};

// Per-expert weight gradient: dW[e][m, n] = sum_{i in slice(e)} A[src_a(i), m] * B[src_b(i), n]
struct DwGemm {
  int E = 0;
  int num_rows = 0;
  const int32_t* offsets = nullptr;
  const int32_t* sorted_slot = nullptr;
  int M = 0, N = 0;
  const void* a = nullptr;
  int lda = 0, a_rows = 0, a_mode = ROWS_GROUPED, a_fan_out = 1;
  const void* b = nullptr;
  int ldb = 0, b_rows = 0, b_mode = ROWS_GROUPED, b_fan_out = 1;
  float* dw = nullptr;  // [E, M, N]
  // Per-slot gates multiplying each reduction row's product (row i by
  // gates[sorted_slot[i]]), nullable: the gated ParallelLinear's
  // dW = sum_i (g_i x_i)^T G_i without a gated copy of x.  The kernels apply the
  // gate to whichever operand they gather.
  const float* row_gates = nullptr;
  unsigned* err = nullptr;
};

// ---- launchers (return a cudaError_t from the launch) ----------------------
cudaError_t launch_route(const void* x, const void* w_r, const float* b_r, int T, int d, int E,
                         int k, smoe_dtype dt, int32_t* idx, float* gates, unsigned* err,
                         cudaStream_t s);
cudaError_t launch_route_dl(const float* gates, const float* dgates, int T, int k, float* dl,
                            cudaStream_t s);
// Router weight gradient from the slots in grouped order (sorted_slot, offsets of
// the expert sort of idx).  partial: route_dw_runs(T*k, E, d) * (d + 1) floats.
cudaError_t launch_route_dw(const void* x, const int32_t* idx, const int32_t* sorted_slot,
                            const int32_t* offsets, const float* dl, int T, int d, int E, int k,
                            smoe_dtype dt, float* partial, float* dw_r, float* db_r,
                            cudaStream_t s);
// Rows of the router weight gradient's partial sums (sizes its workspace).
int route_dw_runs(int S, int E, int d);
cudaError_t launch_route_dx(const float* dl, const int32_t* idx, const void* w_r, int T, int d,
                            int E, int k, smoe_dtype dt, void* dx, cudaStream_t s);

size_t sort_workspace_bytes(int T, int k, int E);
// kernel launches of launch_sort for this shape (1 for a single-block sort, else 3)
int sort_launches(int T, int k, int E);
// inv (nullable): also write inv[sorted_slot[i]] = i
cudaError_t launch_sort(const int32_t* idx, int T, int k, int E, int32_t* sorted_slot,
                        int32_t* offsets, void* ws, unsigned* err, cudaStream_t s,
                        int32_t* inv = nullptr);

// out[t] = sum_{j<ck} ws[row(t*ck + j)] (+ sum_j dl[t*ck+j] * w_rt[idx[t*ck+j], :] if dl),
// summed in fp32; ws, out and w_rt (the router weight transposed to [E, N]) in dtype
// dt; row(p) = inv[p] (the slot's grouped row) or p when inv is null
cudaError_t launch_combine(const void* ws, const int32_t* inv, int T, int ck, int N, void* out,
                           smoe_dtype dt, const float* dl, const int32_t* idx, const void* w_rt,
                           int E, cudaStream_t s);
// inv[sorted_slot[i]] = i for i < num_rows
cudaError_t launch_invert(const int32_t* sorted_slot, int num_rows, int32_t* inv, cudaStream_t s);
// w_rt[e][i] = w_r[i][e]
cudaError_t launch_transpose_wr(const void* w_r, int d, int E, smoe_dtype dt, void* w_rt,
                                cudaStream_t s);
// dg[sorted_slot[i]] = sum_{c < n_tiles} partial[i*ld + c]; inv (nullable) as launch_invert
cudaError_t launch_dg_reduce(const float* partial, int ld, int n_tiles, const int32_t* sorted_slot,
                             int num_rows, float* dg, cudaStream_t s, int32_t* inv = nullptr);
// out[i, :] = gates[sorted_slot[i]] * sum_{s < ksplit} partial[s, i, :] (ascending s),
// grouped rows, bf16; the epilogue of a split-K grouped product
cudaError_t launch_splitk_reduce(const float* partial, int ksplit, int num_rows, int n_out,
                                 const int32_t* sorted_slot, const float* gates, void* out,
                                 int ldo, cudaStream_t s);
// Splits of K for a grouped product of num_rows rows over E experts with n_out
// output columns and K-dimension K: > 1 only when even the most tiles it can have
// would leave most SMs idle (decode-sized batches).
int grouped_ksplit(int num_rows, int E, int n_out, int K, int fp8 = 0);

cudaError_t launch_grouped_gemm_simt(const GroupedGemm& g, smoe_dtype dt, cudaStream_t s);
cudaError_t launch_dw_gemm_simt(const DwGemm& g, smoe_dtype dt, cudaStream_t s);

// Mixture-of-Attention core (attn_tc.cu, bf16, head width attn_head_dim()):
// q/o/dout grouped [T*kslots, heads*128], k/v [T, heads*128], inv the grouped row
// of each slot; lse [T*kslots, heads] fp32; dsum scratch [T*kslots, heads] fp32.
int attn_head_dim();
cudaError_t launch_moa_attn_fwd(const void* q, const void* k, const void* v, const int32_t* inv, int T,
                                int L, int kslots, int heads, void* o, float* lse, unsigned* err,
                                cudaStream_t s);
// backward: dsum = <dO, O> first, then dq and (dk, dv) from it
cudaError_t launch_attn_dsum(const void* dout, const void* o, int S, int heads, float* dsum, cudaStream_t s);
cudaError_t launch_attn_dq(const void* q, const void* k, const void* v, const float* lse,
                           const void* dout, const int32_t* inv, int T, int L, int kslots, int heads,
                           void* dq, const float* dsum, unsigned* err, cudaStream_t s);
cudaError_t launch_attn_dkv(const void* q, const void* k, const void* v, const float* lse,
                            const void* dout, const int32_t* inv, int T, int L, int kslots, int heads,
                            void* dk, void* dv, const float* dsum, unsigned* err, cudaStream_t s);

// e4m3 quantisation (fp8.cu): rows of a bf16 [rows, cols] matrix with one scale per
// row; weights [E, K, N] bf16 -> codes [E, N, K] with one scale per (e, column)
cudaError_t launch_quantize_rows_fp8(const void* x, int rows, int cols, uint8_t* codes, float* scales,
                                     cudaStream_t s);
cudaError_t launch_quantize_weights_fp8(const void* w, int E, int K, int N, uint8_t* codes, float* scales,
                                        cudaStream_t s);

// tcgen05 / TMEM path (bf16 only); *_supported() checks the device once.
bool tc_supported();
// Kernel-selection policy of the tensor-core GEMMs (smoe_set_gemm_policy).
void set_gemm_policy(int policy);
cudaError_t launch_grouped_gemm_tc(const GroupedGemm& g, cudaStream_t s);
cudaError_t launch_dw_gemm_tc(const DwGemm& g, cudaStream_t s);

// Error reporting shared with entry points defined outside api.cu: sets the
// thread-local message returned by smoe_last_error and returns `code`.
int api_fail(int code, const char* fmt, ...);
// This device's error word (resolved once per device), or null with *status set.
unsigned* api_error_word(cudaError_t* status);

}  // namespace smoe
