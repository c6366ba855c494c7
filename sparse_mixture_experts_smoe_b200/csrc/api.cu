// api.cu -- the extern "C" entry points of libsmoe.so (declared in smoe.h):
// argument validation (host side, before any launch), workspace layout, and the
// composition of the kernels into ParallelLinear and the SMoE MLP.
//
// ParallelLinear (library page of arXiv 2403.08245, review 1 summary: input and
// output each grouped or scattered, used for forward and backward; review 2
// summary: group-to-group, group-to-scatter, scatter-to-scatter, scatter-to-group)
// maps onto one grouped-M GEMM whose A rows are read grouped or gathered through
// sorted_slot and whose output rows are written grouped or scattered; a k-way
// combine goes through a grouped-order buffer of gated slot rows in the layer's
// dtype and a fixed-order fp32 sum per token.  The
// backward (tradepoint.io article, method paragraphs: the gradient of each
// expert) swaps the roles of the row maps for dx and runs a per-expert dW GEMM.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"

namespace smoe {

// NVTX range around each entry point (a no-op unless a tool is attached).
struct NvtxScope {
  explicit NvtxScope(const char* name) { nvtxRangePushA(name); }
  ~NvtxScope() { nvtxRangePop(); }
};
int simt_tile_cols();
int tc_tile_cols();
}  // namespace smoe

using namespace smoe;

// Per-device error word of the data/timeout checks (one per device that loads
// the library; read and cleared by smoe_check).
__device__ unsigned g_smoe_error_word;

namespace {

thread_local char g_msg[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* where) {
  return fail(SMOE_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

#define SMOE_TRY(expr, where)                      \
  do {                                             \
    cudaError_t e_ = (expr);                       \
    if (e_ != cudaSuccess) return cuda_fail(e_, where); \
  } while (0)

// ---------------------------------------------------------------------------
// Launch instrumentation (smoe_profile_*): CUDA event pairs around each launch.
// ---------------------------------------------------------------------------
struct Profiler {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> ev;                   // 2 per bracket
  std::vector<std::pair<const char*, int>> rec;  // name, kernels in the bracket
  int used = 0;
  std::map<std::string, int> untimed;            // launches past max_launches
  std::vector<std::string> names;
  std::vector<int> counts;
  std::vector<double> ms;
};
Profiler& profiler() {
  static Profiler p;
  return p;
}

struct ProfScope {
  int slot = -1;
  cudaStream_t s;
  ProfScope(const char* name, int nk, cudaStream_t st) : s(st) {
    Profiler& p = profiler();
    if (!p.on) return;
    std::lock_guard<std::mutex> lock(p.mu);
    if (p.used < (int)p.rec.size()) {
      slot = p.used++;
      p.rec[slot] = {name, nk};
      cudaEventRecord(p.ev[2 * slot], s);
    } else {
      p.untimed[name] += nk;
    }
  }
  ~ProfScope() {
    if (slot >= 0) cudaEventRecord(profiler().ev[2 * slot + 1], s);
  }
};
#define SMOE_PROF_CAT2(a, b) a##b
#define SMOE_PROF_CAT(a, b) SMOE_PROF_CAT2(a, b)
#define PROF(name, nk) ProfScope SMOE_PROF_CAT(prof_scope_, __LINE__)(name, nk, s)

unsigned* error_word(cudaError_t* status) {
  static std::mutex mu;
  static unsigned* ptrs[128] = {};
  int dev = 0;
  *status = cudaGetDevice(&dev);
  if (*status != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr) {
    *status = cudaGetSymbolAddress((void**)&ptrs[dev], g_smoe_error_word);
    if (*status != cudaSuccess) return nullptr;
  }
  return ptrs[dev];
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
// The slot count T*k (and every slot index) fits an int32.
bool slots_fit(int T, int k) { return (long long)T * k <= 0x7fffffffLL; }
size_t align256(size_t n) { return (n + 255) & ~(size_t)255; }
size_t esize(smoe_dtype dt) { return dt == SMOE_BF16 ? 2 : 4; }
bool valid_dtype(int dt) { return dt == SMOE_F32 || dt == SMOE_BF16; }

// Bump allocator over the caller's workspace.
struct Carve {
  char* base;
  size_t off = 0;
  explicit Carve(void* b) : base((char*)b) {}
  void* take(size_t bytes) {
    void* p = base ? base + off : nullptr;
    off += align256(bytes);
    return p;
  }
};

int act_tile_cols(smoe_dtype dt) { return dt == SMOE_BF16 ? tc_tile_cols() : simt_tile_cols(); }

cudaError_t run_grouped(const GroupedGemm& g, smoe_dtype dt, cudaStream_t s) {
  if (dt == SMOE_BF16) return launch_grouped_gemm_tc(g, s);
  return launch_grouped_gemm_simt(g, dt, s);
}
cudaError_t run_dw(const DwGemm& g, smoe_dtype dt, cudaStream_t s) {
  if (dt == SMOE_BF16) return launch_dw_gemm_tc(g, s);
  return launch_dw_gemm_simt(g, dt, s);
}

int check_tc(smoe_dtype dt) {
  if (dt == SMOE_BF16 && !tc_supported())
    return fail(SMOE_ERR_UNSUPPORTED, "bf16 path needs an sm_100 (B200) device");
  return SMOE_OK;
}

// ---------------------------------------------------------------------------
// ParallelLinear workspace layout
// ---------------------------------------------------------------------------
struct PLFwdWs {
  void* comb = nullptr;    // [num_slots, N] slot rows (dtype), grouped order
  int32_t* inv = nullptr;  // [num_slots] grouped row of each slot
  size_t bytes = 0;
};
PLFwdWs pl_fwd_layout(void* ws, int num_slots, int N, int combine_k, smoe_dtype dt) {
  Carve c(ws);
  PLFwdWs l;
  if (combine_k > 0) {
    l.comb = c.take((size_t)num_slots * N * esize(dt));
    l.inv = (int32_t*)c.take((size_t)num_slots * sizeof(int32_t));
  }
  l.bytes = c.off;
  return l;
}

struct PLBwdWs {
  void* dx_comb = nullptr;   // [num_slots, K] dtype when dx needs a fan-out combine (grouped order)
  int32_t* inv = nullptr;    // [num_slots] grouped row of each slot, with dx_comb
  float* dg_part = nullptr;  // [num_slots, dg_ld]
  int dg_ld = 0;
  size_t bytes = 0;
};
// No term here holds x: with gates, dW's gate multiplies x's rows inside the dW
// kernel as they are gathered.
PLBwdWs pl_bwd_layout(void* ws, int num_slots, int K, int grouped_in, int fan_out, int has_gates,
                      int want_dx, int want_dg, smoe_dtype dt) {
  Carve c(ws);
  PLBwdWs l;
  if (want_dx && !grouped_in && fan_out > 1) {
    l.dx_comb = c.take((size_t)num_slots * K * esize(dt));
    l.inv = (int32_t*)c.take((size_t)num_slots * sizeof(int32_t));
  }
  if (has_gates && want_dg) {
    l.dg_ld = cdiv(K, act_tile_cols(dt));
    l.dg_part = (float*)c.take((size_t)num_slots * l.dg_ld * sizeof(float));
  }
  l.bytes = c.off;
  return l;
}

// ---------------------------------------------------------------------------
// Router backward workspace layout
// ---------------------------------------------------------------------------
struct RouteBwdWs {
  float* dl = nullptr;           // [T, k]
  void* sort = nullptr;          // the expert sort's scratch
  int32_t* sorted_slot = nullptr;  // [T * k]
  int32_t* offsets = nullptr;    // [E + 1]
  float* part = nullptr;         // route_dw_runs * (d + 1)
  size_t bytes = 0;
};
RouteBwdWs route_bwd_layout(void* ws, int T, int d, int E, int k) {
  Carve c(ws);
  RouteBwdWs l;
  const size_t S = (size_t)T * k;
  l.dl = (float*)c.take(S * sizeof(float));
  l.sort = c.take(sort_workspace_bytes(T, k, E));
  l.sorted_slot = (int32_t*)c.take(S * sizeof(int32_t));
  l.offsets = (int32_t*)c.take((size_t)(E + 1) * sizeof(int32_t));
  l.part = (float*)c.take((size_t)route_dw_runs((int)S, E, d) * (d + 1) * sizeof(float));
  l.bytes = c.off;
  return l;
}

// ---------------------------------------------------------------------------
// SMoE MLP workspace layout
// ---------------------------------------------------------------------------
struct MlpWs {
  void* sort = nullptr;
  void* ycomb = nullptr;    // fwd: [S, d] slot rows (dtype), grouped order
  float* kpart = nullptr;   // fwd: [ksplit, S, d] fp32 split-K partials of the down projection
  int ksplit = 1;
  float* dg_part = nullptr; // bwd: [S, dg_ld]
  void* dh = nullptr;       // bwd: [S, m*f] dtype (grouped dH)
  void* ga = nullptr;       // bwd: [S, f] dtype (gates * A), written by the dA' epilogue for dW2
  void* dxcomb = nullptr;   // bwd: [S, d] slot rows (dtype), grouped order
  int32_t* inv = nullptr;   // fwd and bwd: [S] grouped row of each slot
  float* dl = nullptr;      // bwd: [T, k]
  float* dg = nullptr;      // bwd: [T, k] when the caller passes no dgates
  float* rpart = nullptr;   // bwd: router dW partials
  void* wrt = nullptr;      // bwd: router weight transposed [E, d] dtype
  int dg_ld = 0, r_runs = 0;
  size_t bytes = 0;
};
MlpWs mlp_layout(void* ws, const smoe_mlp_desc& m, int backward) {
  Carve c(ws);
  MlpWs l;
  const size_t S = (size_t)m.T * m.k;
  const smoe_dtype dt = (smoe_dtype)m.dtype;
  l.sort = c.take(sort_workspace_bytes(m.T, m.k, m.E));
  l.inv = (int32_t*)c.take(S * sizeof(int32_t));
  if (!backward) {
    l.ycomb = c.take(S * m.d * esize(dt));
    // a decode-sized batch splits the down projection's K (tensor-core path only)
    l.ksplit = dt == SMOE_BF16 ? grouped_ksplit((int)S, m.E, m.d, m.f) : 1;
    if (l.ksplit > 1) l.kpart = (float*)c.take((size_t)l.ksplit * S * m.d * sizeof(float));
  } else {
    l.dg_ld = cdiv(m.f, act_tile_cols(dt));
    l.dg_part = (float*)c.take(S * l.dg_ld * sizeof(float));
    l.dh = c.take(S * (size_t)(m.act == SMOE_ACT_SWIGLU ? 2 * m.f : m.f) * esize(dt));
    l.ga = c.take(S * m.f * esize(dt));
    l.dxcomb = c.take(S * m.d * esize(dt));
    l.dl = (float*)c.take(S * sizeof(float));
    l.dg = (float*)c.take(S * sizeof(float));
    l.r_runs = route_dw_runs((int)S, m.E, m.d);
    l.rpart = (float*)c.take((size_t)l.r_runs * (m.d + 1) * sizeof(float));
    l.wrt = c.take((size_t)m.E * m.d * esize(dt));
  }
  l.bytes = c.off;
  return l;
}

int validate_mlp_desc(const smoe_mlp_desc* m) {
  if (!m) return fail(SMOE_ERR_INVALID_ARG, "desc is NULL");
  if (m->T < 0 || m->d <= 0 || m->f <= 0 || m->E <= 0 || m->k <= 0)
    return fail(SMOE_ERR_INVALID_ARG, "bad sizes T=%d d=%d f=%d E=%d k=%d", m->T, m->d, m->f, m->E, m->k);
  if (m->k > m->E || m->k > SMOE_MAX_TOPK || m->E > SMOE_MAX_ROUTED_EXPERTS)
    return fail(SMOE_ERR_INVALID_ARG, "need 1 <= k <= min(E, %d) and E <= %d (k=%d E=%d)",
                SMOE_MAX_TOPK, SMOE_MAX_ROUTED_EXPERTS, m->k, m->E);
  if (m->d % 8 || m->f % 8) return fail(SMOE_ERR_INVALID_ARG, "d and f must be multiples of 8");
  if (!valid_dtype(m->dtype)) return fail(SMOE_ERR_INVALID_ARG, "bad dtype %d", m->dtype);
  if (m->act != SMOE_ACT_GELU_TANH && m->act != SMOE_ACT_SWIGLU)
    return fail(SMOE_ERR_INVALID_ARG, "act must be GELU_TANH or SWIGLU");
  if ((long long)m->T * m->k * 2LL * m->f >= (1LL << 31) || (long long)m->T * m->d >= (1LL << 31))
    return fail(SMOE_ERR_INVALID_ARG, "tensor too large for 32-bit row indexing");
  return SMOE_OK;
}

#define NEED(p, name) \
  if (!(p)) return fail(SMOE_ERR_INVALID_ARG, "%s is NULL", name)
#define ALIGNED(p, name) \
  if (!aligned16(p)) return fail(SMOE_ERR_INVALID_ARG, "%s is not 16-byte aligned", name)

}  // namespace

namespace smoe {
int api_fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return code;
}
unsigned* api_error_word(cudaError_t* status) { return error_word(status); }
}  // namespace smoe

extern "C" {

const char* smoe_last_error(void) { return g_msg; }

const char* smoe_version(void) { return "smoe-b200 0.1 (sm_100a)"; }

int smoe_check(void* stream) {
  cudaError_t st;
  SMOE_TRY(cudaStreamSynchronize((cudaStream_t)stream), "smoe_check sync");
  unsigned* w = error_word(&st);
  if (!w) return cuda_fail(st, "smoe_check error word");
  unsigned v = 0;
  SMOE_TRY(cudaMemcpy(&v, w, sizeof(v), cudaMemcpyDeviceToHost), "smoe_check read");
  if (v != 0) {
    const unsigned zero = 0;
    SMOE_TRY(cudaMemcpy(w, &zero, sizeof(zero), cudaMemcpyHostToDevice), "smoe_check clear");
  }
  if (v & ERRBIT_TIMEOUT) return fail(SMOE_ERR_TIMEOUT, "a bounded device wait gave up");
  if (v & ERRBIT_DATA) return fail(SMOE_ERR_DATA, "device found an index outside its range");
  return SMOE_OK;
}

int smoe_profile_begin(int max_launches) {
  Profiler& p = profiler();
  std::lock_guard<std::mutex> lock(p.mu);
  if (max_launches < 0) return fail(SMOE_ERR_INVALID_ARG, "max_launches < 0");
  for (cudaEvent_t e : p.ev) cudaEventDestroy(e);
  p.ev.assign(2 * (size_t)max_launches, nullptr);
  for (auto& e : p.ev) SMOE_TRY(cudaEventCreate(&e), "smoe_profile_begin");
  p.rec.assign(max_launches, {nullptr, 0});
  p.used = 0;
  p.untimed.clear();
  p.names.clear(); p.counts.clear(); p.ms.clear();
  p.on = true;
  return SMOE_OK;
}

int smoe_profile_end(void) {
  Profiler& p = profiler();
  std::lock_guard<std::mutex> lock(p.mu);
  p.on = false;
  std::map<std::string, std::pair<int, double>> agg;
  for (int i = 0; i < p.used; ++i) {
    SMOE_TRY(cudaEventSynchronize(p.ev[2 * i + 1]), "smoe_profile_end");
    float t = 0.0f;
    SMOE_TRY(cudaEventElapsedTime(&t, p.ev[2 * i], p.ev[2 * i + 1]), "smoe_profile_end");
    auto& a = agg[p.rec[i].first];
    a.first += p.rec[i].second;
    a.second += t;
  }
  for (auto& kv : p.untimed) agg[kv.first].first += kv.second;
  p.names.clear(); p.counts.clear(); p.ms.clear();
  for (auto& kv : agg) {
    p.names.push_back(kv.first);
    p.counts.push_back(kv.second.first);
    p.ms.push_back(kv.second.second);
  }
  return (int)p.names.size();
}

int smoe_profile_entry(int i, const char** name, int* launches, double* total_ms) {
  Profiler& p = profiler();
  std::lock_guard<std::mutex> lock(p.mu);
  if (i < 0 || i >= (int)p.names.size()) return fail(SMOE_ERR_INVALID_ARG, "no entry %d", i);
  if (name) *name = p.names[i].c_str();
  if (launches) *launches = p.counts[i];
  if (total_ms) *total_ms = p.ms[i];
  return SMOE_OK;
}

size_t smoe_workspace_size(int op, int T, int k, int E, int d, int f, smoe_dtype dt) {
  if (T < 0 || k <= 0 || E <= 0 || d <= 0 || f <= 0 || !slots_fit(T, k)) return 0;
  const int S = T * k;
  const int wide = (d > 2 * f ? d : 2 * f);
  switch (op) {
    case SMOE_OP_SORT: return sort_workspace_bytes(T, k, E);
    case SMOE_OP_PL_FWD: return pl_fwd_layout(nullptr, S, wide, k, dt).bytes;
    case SMOE_OP_PL_BWD: return pl_bwd_layout(nullptr, S, wide, 0, k, 1, 1, 1, dt).bytes;
    case SMOE_OP_ROUTE_BWD: return route_bwd_layout(nullptr, T, d, E, k).bytes;
    case SMOE_OP_MLP_FWD:
    case SMOE_OP_MLP_BWD: {
      smoe_mlp_desc m{T, d, f, E, k, SMOE_ACT_SWIGLU, dt};
      size_t b = mlp_layout(nullptr, m, op == SMOE_OP_MLP_BWD).bytes;
      return b;
    }
    default: return 0;
  }
}

int smoe_route(const void* x, const void* w_r, const float* b_r, int T, int d, int E, int k,
               smoe_dtype dt, int32_t* topk_idx, float* gates, void* stream) {
  smoe::NvtxScope nvtx_scope("smoe_route");
  if (T < 0 || d <= 0 || E <= 0 || k <= 0) return fail(SMOE_ERR_INVALID_ARG, "bad sizes");
  if (k > E || k > SMOE_MAX_TOPK || E > SMOE_MAX_ROUTED_EXPERTS)
    return fail(SMOE_ERR_INVALID_ARG, "need 1 <= k <= min(E, %d), E <= %d", SMOE_MAX_TOPK,
                SMOE_MAX_ROUTED_EXPERTS);
  if (d % 8) return fail(SMOE_ERR_INVALID_ARG, "d must be a multiple of 8");
  if (!slots_fit(T, k) || (long long)T * d >= (1LL << 31))
    return fail(SMOE_ERR_INVALID_ARG, "T*k or T*d too large for 32-bit indexing");
  if (!valid_dtype(dt)) return fail(SMOE_ERR_INVALID_ARG, "bad dtype");
  if (T == 0) return SMOE_OK;
  NEED(x, "x"); NEED(w_r, "w_r"); NEED(topk_idx, "topk_idx"); NEED(gates, "gates");
  ALIGNED(x, "x"); ALIGNED(w_r, "w_r");
  cudaError_t st;
  unsigned* err = error_word(&st);
  if (!err) return cuda_fail(st, "smoe_route");
  cudaStream_t s = (cudaStream_t)stream;
  { PROF("route", 1);
  SMOE_TRY(launch_route(x, w_r, b_r, T, d, E, k, dt, topk_idx, gates, err, s), "smoe_route launch"); }
  return SMOE_OK;
}

int smoe_route_bwd(const void* x, const void* w_r, const int32_t* topk_idx, const float* gates,
                   const float* dgates, int T, int d, int E, int k, smoe_dtype dt, void* dx,
                   float* dw_r, float* db_r, void* workspace, size_t ws_bytes, void* stream) {
  smoe::NvtxScope nvtx_scope("smoe_route_bwd");
  if (T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E || k > SMOE_MAX_TOPK ||
      E > SMOE_MAX_ROUTED_EXPERTS)
    return fail(SMOE_ERR_INVALID_ARG, "bad sizes (need 1 <= k <= min(E, %d), E <= %d)",
                SMOE_MAX_TOPK, SMOE_MAX_ROUTED_EXPERTS);
  if (d % 8) return fail(SMOE_ERR_INVALID_ARG, "d must be a multiple of 8");
  if (!slots_fit(T, k) || (long long)T * d >= (1LL << 31))
    return fail(SMOE_ERR_INVALID_ARG, "T*k or T*d too large for 32-bit indexing");
  if (!valid_dtype(dt)) return fail(SMOE_ERR_INVALID_ARG, "bad dtype");
  NEED(x, "x"); NEED(w_r, "w_r"); NEED(topk_idx, "topk_idx"); NEED(gates, "gates");
  NEED(dgates, "dgates"); NEED(dw_r, "dw_r");
  const RouteBwdWs l = route_bwd_layout(workspace, T, d, E, k);
  if (T > 0 && (!workspace || ws_bytes < l.bytes))
    return fail(SMOE_ERR_INVALID_ARG, "workspace too small (%zu < %zu)", ws_bytes, l.bytes);
  if (T == 0) {
    cudaStream_t s = (cudaStream_t)stream;
    SMOE_TRY(cudaMemsetAsync(dw_r, 0, (size_t)d * E * sizeof(float), s), "route_bwd zero");
    if (db_r) SMOE_TRY(cudaMemsetAsync(db_r, 0, (size_t)E * sizeof(float), s), "route_bwd zero");
    return SMOE_OK;
  }
  cudaError_t st;
  unsigned* err = error_word(&st);
  if (!err) return cuda_fail(st, "smoe_route_bwd");
  cudaStream_t s = (cudaStream_t)stream;
  { PROF("route_dl", 1); SMOE_TRY(launch_route_dl(gates, dgates, T, k, l.dl, s), "route_dl"); }
  // the weight gradient walks the slots in grouped order
  { PROF("sort", sort_launches(T, k, E)); SMOE_TRY(launch_sort(topk_idx, T, k, E, l.sorted_slot, l.offsets, l.sort, err, s), "route_bwd sort"); }
  { PROF("route_dw", 2); SMOE_TRY(launch_route_dw(x, topk_idx, l.sorted_slot, l.offsets, l.dl, T, d, E, k, dt, l.part, dw_r, db_r, s), "route_dw"); }
  if (dx) { PROF("route_dx", 1); SMOE_TRY(launch_route_dx(l.dl, topk_idx, w_r, T, d, E, k, dt, dx, s), "route_dx"); }
  return SMOE_OK;
}

int smoe_sort(const int32_t* topk_idx, int T, int k, int E, int32_t* sorted_slot,
              int32_t* expert_offsets, void* workspace, size_t ws_bytes, void* stream) {
  smoe::NvtxScope nvtx_scope("smoe_sort");
  if (T < 0 || k <= 0 || E <= 0 || E > SMOE_MAX_EXPERTS)
    return fail(SMOE_ERR_INVALID_ARG, "bad sizes (E <= %d)", SMOE_MAX_EXPERTS);
  if (!slots_fit(T, k)) return fail(SMOE_ERR_INVALID_ARG, "T*k too large for 32-bit indexing");
  NEED(expert_offsets, "expert_offsets");
  cudaStream_t s = (cudaStream_t)stream;
  if (T == 0) {
    SMOE_TRY(cudaMemsetAsync(expert_offsets, 0, (size_t)(E + 1) * sizeof(int32_t), s), "sort zero");
    return SMOE_OK;
  }
  NEED(topk_idx, "topk_idx"); NEED(sorted_slot, "sorted_slot");
  const size_t need = sort_workspace_bytes(T, k, E);
  if (!workspace || ws_bytes < need)
    return fail(SMOE_ERR_INVALID_ARG, "workspace too small (%zu < %zu)", ws_bytes, need);
  cudaError_t st;
  unsigned* err = error_word(&st);
  if (!err) return cuda_fail(st, "smoe_sort");
  { PROF("sort", sort_launches(T, k, E)); SMOE_TRY(launch_sort(topk_idx, T, k, E, sorted_slot, expert_offsets, workspace, err, s), "smoe_sort"); }
  return SMOE_OK;
}

// ---------------------------------------------------------------------------
// ParallelLinear
// ---------------------------------------------------------------------------
static int validate_pl(const void* x, int x_rows, int K, const void* w, int N, int E,
                       const int32_t* sorted_slot, const int32_t* offsets, int num_slots,
                       int fan_out, int grouped_in, int grouped_out, int combine_k, int dt) {
  if (num_slots < 0 || x_rows < 0 || K <= 0 || N <= 0 || E <= 0)
    return fail(SMOE_ERR_INVALID_ARG, "bad sizes");
  if (E > SMOE_MAX_EXPERTS) return fail(SMOE_ERR_INVALID_ARG, "E <= %d", SMOE_MAX_EXPERTS);
  if (K % 8 || N % 8) return fail(SMOE_ERR_INVALID_ARG, "K and N must be multiples of 8");
  if (!valid_dtype(dt)) return fail(SMOE_ERR_INVALID_ARG, "bad dtype");
  if (fan_out < 1 || combine_k < 0) return fail(SMOE_ERR_INVALID_ARG, "fan_out >= 1, combine_k >= 0");
  if (combine_k > 0 && (grouped_out || num_slots % combine_k))
    return fail(SMOE_ERR_INVALID_ARG, "combine needs a scattered output and num_slots %% combine_k == 0");
  if (grouped_in && x_rows != num_slots)
    return fail(SMOE_ERR_INVALID_ARG, "grouped input needs x_rows == num_slots");
  if (!grouped_in && (long long)x_rows * fan_out < num_slots)
    return fail(SMOE_ERR_INVALID_ARG, "x_rows * fan_out < num_slots");
  if ((long long)num_slots * (K > N ? K : N) >= (1LL << 31) ||
      (long long)x_rows * K >= (1LL << 31))
    return fail(SMOE_ERR_INVALID_ARG, "tensor too large for 32-bit row indexing");
  if (num_slots == 0) return SMOE_OK;
  NEED(x, "x"); NEED(w, "w"); NEED(sorted_slot, "sorted_slot"); NEED(offsets, "expert_offsets");
  ALIGNED(x, "x"); ALIGNED(w, "w");
  return SMOE_OK;
}

size_t parallel_linear_fwd_workspace_size(int num_slots, int K, int N, int E, int combine_k,
                                          smoe_dtype dt) {
  (void)K; (void)E;
  if (num_slots <= 0 || N <= 0) return 0;
  return pl_fwd_layout(nullptr, num_slots, N, combine_k, dt).bytes;
}

int parallel_linear_fwd(const void* x, int x_rows, int K, const void* w, int N, int E,
                        const int32_t* sorted_slot, const int32_t* expert_offsets, int num_slots,
                        int fan_out, int grouped_in, int grouped_out, const float* gates,
                        int combine_k, void* y, smoe_dtype dt, void* workspace, size_t ws_bytes,
                        void* stream) {
  smoe::NvtxScope nvtx_scope("parallel_linear_fwd");
  int rc = validate_pl(x, x_rows, K, w, N, E, sorted_slot, expert_offsets, num_slots, fan_out,
                       grouped_in, grouped_out, combine_k, dt);
  if (rc != SMOE_OK) return rc;
  if (num_slots == 0) return SMOE_OK;
  NEED(y, "y"); ALIGNED(y, "y");
  PLFwdWs l = pl_fwd_layout(workspace, num_slots, N, combine_k, dt);
  if (l.bytes > 0 && (!workspace || ws_bytes < l.bytes))
    return fail(SMOE_ERR_INVALID_ARG, "workspace too small (%zu < %zu)", ws_bytes, l.bytes);
  if ((rc = check_tc(dt)) != SMOE_OK) return rc;
  cudaError_t st;
  unsigned* err = error_word(&st);
  if (!err) return cuda_fail(st, "parallel_linear_fwd");
  cudaStream_t s = (cudaStream_t)stream;
  GroupedGemm g;
  g.E = E; g.num_rows = num_slots; g.offsets = expert_offsets; g.sorted_slot = sorted_slot;
  g.K = K; g.a = x; g.lda = K; g.a_rows = x_rows;
  g.a_mode = grouped_in ? ROWS_GROUPED : ROWS_GATHER; g.a_fan_out = fan_out;
  g.b = w; g.b_kn = 1; g.NW = N; g.n_out = N;
  g.epi = EPI_STORE; g.gates = gates; g.err = err;
  if (combine_k > 0) {
    g.out_mode = ROWS_GROUPED; g.out = l.comb; g.ldo = N; g.out_f32 = dt == SMOE_F32;
  } else {
    g.out_mode = grouped_out ? ROWS_GROUPED : ROWS_GATHER; g.out = y; g.ldo = N;
    g.out_f32 = dt == SMOE_F32;
  }
  { PROF("pl.gemm_fwd", 1); SMOE_TRY(run_grouped(g, dt, s), "parallel_linear_fwd gemm"); }
  if (combine_k > 0) {
    { PROF("pl.invert", 1); SMOE_TRY(launch_invert(sorted_slot, num_slots, l.inv, s), "parallel_linear_fwd invert"); }
    PROF("pl.combine", 1);
    SMOE_TRY(launch_combine(l.comb, l.inv, num_slots / combine_k, combine_k, N, y, dt, nullptr,
                            nullptr, nullptr, 0, s), "parallel_linear_fwd combine");
  }
  return SMOE_OK;
}

size_t parallel_linear_bwd_workspace_size(int x_rows, int num_slots, int K, int N, int E,
                                          int fan_out, int grouped_in, int grouped_out,
                                          int has_gates, int combine_k, smoe_dtype dt) {
  (void)x_rows; (void)N; (void)E; (void)grouped_out; (void)combine_k;
  if (num_slots <= 0 || K <= 0) return 0;
  return pl_bwd_layout(nullptr, num_slots, K, grouped_in, fan_out, has_gates, 1, 1, dt).bytes;
}

int parallel_linear_bwd(const void* dy, const void* x, const void* w, int x_rows, int K, int N,
                        int E, const int32_t* sorted_slot, const int32_t* expert_offsets,
                        int num_slots, int fan_out, int grouped_in, int grouped_out,
                        const float* gates, int combine_k, void* dx, float* dw, float* dgates,
                        smoe_dtype dt, void* workspace, size_t ws_bytes, void* stream) {
  smoe::NvtxScope nvtx_scope("parallel_linear_bwd");
  int rc = validate_pl(x, x_rows, K, w, N, E, sorted_slot, expert_offsets, num_slots, fan_out,
                       grouped_in, grouped_out, combine_k, dt);
  if (rc != SMOE_OK) return rc;
  if (dgates && !gates) return fail(SMOE_ERR_INVALID_ARG, "dgates needs the forward's gates");
  cudaStream_t s = (cudaStream_t)stream;
  if (num_slots == 0) {
    if (dw) SMOE_TRY(cudaMemsetAsync(dw, 0, (size_t)E * K * N * sizeof(float), s), "pl_bwd zero dw");
    if (dx && x_rows > 0) SMOE_TRY(cudaMemsetAsync(dx, 0, (size_t)x_rows * K * esize(dt), s), "pl_bwd zero dx");
    return SMOE_OK;
  }
  NEED(dy, "dy"); ALIGNED(dy, "dy");
  if (dx) ALIGNED(dx, "dx");
  const int has_g = gates != nullptr;
  PLBwdWs l = pl_bwd_layout(workspace, num_slots, K, grouped_in, fan_out, has_g, dx != nullptr,
                            dgates != nullptr, dt);
  if (l.bytes > 0 && (!workspace || ws_bytes < l.bytes))
    return fail(SMOE_ERR_INVALID_ARG, "workspace too small (%zu < %zu)", ws_bytes, l.bytes);
  if ((rc = check_tc(dt)) != SMOE_OK) return rc;
  cudaError_t st;
  unsigned* err = error_word(&st);
  if (!err) return cuda_fail(st, "parallel_linear_bwd");

  // rows of dy feeding grouped row i
  const int g_mode = combine_k > 0 ? ROWS_GATHER : (grouped_out ? ROWS_GROUPED : ROWS_GATHER);
  const int g_fan = combine_k > 0 ? combine_k : 1;
  const int x_mode = grouped_in ? ROWS_GROUPED : ROWS_GATHER;
  // where dx rows go
  const bool dx_comb = !grouped_in && fan_out > 1;

  const bool need_gemm = dx != nullptr || dgates != nullptr;
  if (need_gemm) {
    GroupedGemm g;
    g.E = E; g.num_rows = num_slots; g.offsets = expert_offsets; g.sorted_slot = sorted_slot;
    g.K = N; g.a = dy; g.lda = N; g.a_mode = g_mode; g.a_fan_out = g_fan;
    g.a_rows = combine_k > 0 ? num_slots / combine_k : num_slots;
    g.b = w; g.b_kn = 0; g.NW = K; g.n_out = K;
    g.gates = gates; g.err = err;
    g.out_mode = grouped_in ? ROWS_GROUPED : ROWS_GATHER;
    if (dx_comb) { g.out_mode = ROWS_GROUPED; g.out = l.dx_comb; g.ldo = K; g.out_f32 = dt == SMOE_F32; }
    else { g.out = dx; g.ldo = K; g.out_f32 = dt == SMOE_F32; }
    if (has_g) {  // dx rows g * dA'; gate-gradient partials <dA', x row>
      g.epi = EPI_ACT_BWD; g.act = SMOE_ACT_NONE;
      g.aux_a = x; g.ld_aux_a = K; g.aux_a_mode = x_mode; g.aux_a_fan_out = fan_out;
      g.out2 = nullptr;
      g.dg_partial = l.dg_part; g.dg_ld = l.dg_ld;
      if (!dgates) { g.dg_partial = nullptr; }
    } else {
      g.epi = EPI_STORE;
    }
    if (!dx) g.out = nullptr;
    { PROF("pl.gemm_dx", 1); SMOE_TRY(run_grouped(g, dt, s), "parallel_linear_bwd dx gemm"); }
    if (dgates) {
      PROF("pl.dg_reduce", 1);
      SMOE_TRY(launch_dg_reduce(l.dg_part, l.dg_ld, cdiv(K, act_tile_cols(dt)), sorted_slot,
                                num_slots, dgates, s, dx && dx_comb ? l.inv : nullptr),
               "parallel_linear_bwd dg");
    }
    if (dx && dx_comb) {
      if (!dgates) { PROF("pl.invert", 1); SMOE_TRY(launch_invert(sorted_slot, num_slots, l.inv, s), "parallel_linear_bwd invert"); }
      PROF("pl.combine_dx", 1);
      SMOE_TRY(launch_combine(l.dx_comb, l.inv, x_rows, fan_out, K, dx, dt, nullptr, nullptr,
                              nullptr, 0, s), "parallel_linear_bwd dx combine");
    }
  }
  if (dw) {  // dW[e] = sum_i (g x_row(i))^T G_i: the gate is applied inside the dW kernel
    DwGemm g;
    g.E = E; g.num_rows = num_slots; g.offsets = expert_offsets; g.sorted_slot = sorted_slot;
    g.M = K; g.N = N;
    g.a = x; g.lda = K; g.a_mode = x_mode; g.a_fan_out = fan_out; g.a_rows = x_rows;
    g.b = dy; g.ldb = N; g.b_mode = g_mode; g.b_fan_out = g_fan;
    g.b_rows = combine_k > 0 ? num_slots / combine_k : num_slots;
    g.row_gates = gates;
    g.dw = dw; g.err = err;
    { PROF("pl.gemm_dw", 1); SMOE_TRY(run_dw(g, dt, s), "parallel_linear_bwd dw gemm"); }
  }
  return SMOE_OK;
}

// ---------------------------------------------------------------------------
// FP8 inference forward
// ---------------------------------------------------------------------------
struct Fp8Ws {
  void* sort = nullptr;
  int32_t* inv = nullptr;
  void* ycomb = nullptr;    // [S, d] bf16 slot rows, grouped order
  float* kpart = nullptr;   // split-K partials of the down projection
  int ksplit = 1;
  uint8_t* x8 = nullptr;    // [T, d] codes
  float* sx = nullptr;      // [T]
  uint8_t* a8 = nullptr;    // [S, f] codes (grouped rows)
  float* sa = nullptr;      // [S]
  size_t bytes = 0;
};
static Fp8Ws fp8_layout(void* ws, const smoe_mlp_desc& m) {
  Carve c(ws);
  Fp8Ws l;
  const size_t S = (size_t)m.T * m.k;
  l.sort = c.take(sort_workspace_bytes(m.T, m.k, m.E));
  l.inv = (int32_t*)c.take(S * sizeof(int32_t));
  l.ycomb = c.take(S * m.d * 2);
  l.ksplit = grouped_ksplit((int)S, m.E, m.d, m.f, 1);
  if (l.ksplit > 1) l.kpart = (float*)c.take((size_t)l.ksplit * S * m.d * sizeof(float));
  l.x8 = (uint8_t*)c.take((size_t)m.T * m.d);
  l.sx = (float*)c.take((size_t)m.T * sizeof(float));
  l.a8 = (uint8_t*)c.take(S * m.f);
  l.sa = (float*)c.take(S * sizeof(float));
  l.bytes = c.off;
  return l;
}

static int validate_fp8_desc(const smoe_mlp_desc* m) {
  int rc = validate_mlp_desc(m);
  if (rc != SMOE_OK) return rc;
  if (m->dtype != SMOE_BF16) return fail(SMOE_ERR_UNSUPPORTED, "the FP8 forward takes bf16 activations");
  if (m->d % 16 || m->f % 16) return fail(SMOE_ERR_INVALID_ARG, "FP8: d and f must be multiples of 16");
  return SMOE_OK;
}

// ---------------------------------------------------------------------------
// Mixture-of-Attention core
// ---------------------------------------------------------------------------
static size_t moa_ws_bytes(int T, int kslots, int heads, int backward) {
  const size_t S = (size_t)T * kslots;
  return align256(S * sizeof(int32_t)) + (backward ? align256(S * heads * sizeof(float)) : 0);
}

static int validate_moa(int T, int L, int kslots, int heads, int head_dim, int dt) {
  if (T < 0 || L < 1 || kslots < 1 || kslots > 128 || heads < 1)
    return fail(SMOE_ERR_INVALID_ARG, "bad sizes (T >= 0, L >= 1, 1 <= kslots <= 128, heads >= 1)");
  if (!slots_fit(T, kslots) || (long long)T * kslots * heads * head_dim >= (1LL << 31))
    return fail(SMOE_ERR_INVALID_ARG, "tensor too large for 32-bit row indexing");
  if (!valid_dtype(dt)) return fail(SMOE_ERR_INVALID_ARG, "bad dtype");
  if (dt != SMOE_BF16) return fail(SMOE_ERR_UNSUPPORTED, "the attention core is bf16 only");
  if (head_dim != attn_head_dim())
    return fail(SMOE_ERR_UNSUPPORTED, "head_dim must be %d", attn_head_dim());
  return SMOE_OK;
}

size_t smoe_moa_attn_workspace_size(int T, int kslots, int heads, int backward) {
  if (T < 0 || kslots < 1 || heads < 1 || !slots_fit(T, kslots)) return 0;
  return moa_ws_bytes(T, kslots, heads, backward);
}

int smoe_moa_attn_fwd(const void* q, const void* k, const void* v, const int32_t* sorted_slot, int T,
                      int L, int kslots, int heads, int head_dim, smoe_dtype dt, void* o, float* lse,
                      void* workspace, size_t ws_bytes, void* stream) {
  smoe::NvtxScope nvtx_scope("smoe_moa_attn_fwd");
  int rc = validate_moa(T, L, kslots, heads, head_dim, dt);
  if (rc != SMOE_OK) return rc;
  if (T == 0) return SMOE_OK;
  NEED(q, "q"); NEED(k, "k"); NEED(v, "v"); NEED(sorted_slot, "sorted_slot"); NEED(o, "o");
  NEED(lse, "lse");
  ALIGNED(q, "q"); ALIGNED(k, "k"); ALIGNED(v, "v"); ALIGNED(o, "o");
  const size_t need = moa_ws_bytes(T, kslots, heads, 0);
  if (!workspace || ws_bytes < need)
    return fail(SMOE_ERR_INVALID_ARG, "workspace too small (%zu < %zu)", ws_bytes, need);
  if ((rc = check_tc(dt)) != SMOE_OK) return rc;
  cudaError_t st;
  unsigned* err = error_word(&st);
  if (!err) return cuda_fail(st, "smoe_moa_attn_fwd");
  cudaStream_t s = (cudaStream_t)stream;
  int32_t* inv = (int32_t*)workspace;
  { PROF("moa.invert", 1); SMOE_TRY(launch_invert(sorted_slot, T * kslots, inv, s), "moa invert"); }
  { PROF("moa.attn_fwd", 1);
    SMOE_TRY(launch_moa_attn_fwd(q, k, v, inv, T, L, kslots, heads, o, lse, err, s), "moa attn fwd"); }
  return SMOE_OK;
}

int smoe_moa_attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                      const void* dout, const int32_t* sorted_slot, int T, int L, int kslots, int heads,
                      int head_dim, smoe_dtype dt, void* dq, void* dk, void* dv, void* workspace,
                      size_t ws_bytes, void* stream) {
  smoe::NvtxScope nvtx_scope("smoe_moa_attn_bwd");
  int rc = validate_moa(T, L, kslots, heads, head_dim, dt);
  if (rc != SMOE_OK) return rc;
  if (T == 0) return SMOE_OK;
  NEED(q, "q"); NEED(k, "k"); NEED(v, "v"); NEED(o, "o"); NEED(lse, "lse"); NEED(dout, "dout");
  NEED(sorted_slot, "sorted_slot"); NEED(dq, "dq"); NEED(dk, "dk"); NEED(dv, "dv");
  ALIGNED(q, "q"); ALIGNED(k, "k"); ALIGNED(v, "v"); ALIGNED(o, "o"); ALIGNED(dout, "dout");
  ALIGNED(dq, "dq"); ALIGNED(dk, "dk"); ALIGNED(dv, "dv");
  const size_t need = moa_ws_bytes(T, kslots, heads, 1);
  if (!workspace || ws_bytes < need)
    return fail(SMOE_ERR_INVALID_ARG, "workspace too small (%zu < %zu)", ws_bytes, need);
  if (((uintptr_t)workspace & 255u) != 0) return fail(SMOE_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  if ((rc = check_tc(dt)) != SMOE_OK) return rc;
  cudaError_t st;
  unsigned* err = error_word(&st);
  if (!err) return cuda_fail(st, "smoe_moa_attn_bwd");
  cudaStream_t s = (cudaStream_t)stream;
  const size_t S = (size_t)T * kslots;
  int32_t* inv = (int32_t*)workspace;
  float* dsum = (float*)((char*)workspace + align256(S * sizeof(int32_t)));
  { PROF("moa.invert", 1); SMOE_TRY(launch_invert(sorted_slot, (int)S, inv, s), "moa invert"); }
  { PROF("moa.attn_dsum", 1);
    SMOE_TRY(launch_attn_dsum(dout, o, (int)S, heads, dsum, s), "moa attn dsum"); }
  { PROF("moa.attn_dq", 1);
    SMOE_TRY(launch_attn_dq(q, k, v, lse, dout, inv, T, L, kslots, heads, dq, dsum, err, s), "moa attn dq"); }
  { PROF("moa.attn_dkv", 1);
    SMOE_TRY(launch_attn_dkv(q, k, v, lse, dout, inv, T, L, kslots, heads, dk, dv, dsum, err, s),
             "moa attn dkv"); }
  return SMOE_OK;
}

int smoe_quantize_weights_fp8(const void* w, int E, int K, int N, smoe_dtype dt, uint8_t* codes,
                              float* scales, void* stream) {
  smoe::NvtxScope nvtx_scope("smoe_quantize_weights_fp8");
  if (E <= 0 || K <= 0 || N <= 0) return fail(SMOE_ERR_INVALID_ARG, "bad sizes");
  if (K % 16) return fail(SMOE_ERR_INVALID_ARG, "K must be a multiple of 16");
  if (dt != SMOE_BF16) return fail(SMOE_ERR_UNSUPPORTED, "FP8 weights are quantised from bf16");
  if ((long long)E * K * N >= (1LL << 40)) return fail(SMOE_ERR_INVALID_ARG, "tensor too large");
  NEED(w, "w"); NEED(codes, "codes"); NEED(scales, "scales");
  cudaStream_t s = (cudaStream_t)stream;
  { PROF("fp8.quantize_w", 1);
    SMOE_TRY(launch_quantize_weights_fp8(w, E, K, N, codes, scales, s), "quantize weights"); }
  return SMOE_OK;
}

size_t smoe_mlp_fp8_workspace_size(const smoe_mlp_desc* desc) {
  if (validate_fp8_desc(desc) != SMOE_OK) return 0;
  return fp8_layout(nullptr, *desc).bytes;
}

int smoe_mlp_fwd_fp8(const smoe_mlp_desc* desc, const smoe_mlp_tensors* t, const smoe_fp8_weights* w8,
                     void* stream) {
  smoe::NvtxScope nvtx_scope("smoe_mlp_fwd_fp8");
  int rc = validate_fp8_desc(desc);
  if (rc != SMOE_OK) return rc;
  NEED(t, "tensors"); NEED(w8, "fp8 weights");
  const smoe_mlp_desc& m = *desc;
  if (m.T == 0) return SMOE_OK;
  NEED(t->x, "x"); NEED(t->w_r, "w_r"); NEED(t->y, "y"); NEED(t->topk_idx, "topk_idx");
  NEED(t->gates, "gates"); NEED(t->sorted_slot, "sorted_slot"); NEED(t->expert_offsets, "expert_offsets");
  NEED(t->h, "h"); NEED(t->a, "a");
  NEED(w8->w1q, "w1q"); NEED(w8->s1, "s1"); NEED(w8->w2q, "w2q"); NEED(w8->s2, "s2");
  ALIGNED(t->x, "x"); ALIGNED(t->w_r, "w_r"); ALIGNED(t->y, "y"); ALIGNED(t->h, "h"); ALIGNED(t->a, "a");
  ALIGNED(w8->w1q, "w1q"); ALIGNED(w8->w2q, "w2q"); ALIGNED(w8->s1, "s1"); ALIGNED(w8->s2, "s2");
  Fp8Ws l = fp8_layout(t->workspace, m);
  if (!t->workspace || t->workspace_bytes < l.bytes)
    return fail(SMOE_ERR_INVALID_ARG, "workspace too small (%zu < %zu)", t->workspace_bytes, l.bytes);
  if (((uintptr_t)t->workspace & 255u) != 0) return fail(SMOE_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  if ((rc = check_tc(SMOE_BF16)) != SMOE_OK) return rc;
  cudaError_t st;
  unsigned* err = error_word(&st);
  if (!err) return cuda_fail(st, "smoe_mlp_fwd_fp8");
  cudaStream_t s = (cudaStream_t)stream;
  const int S = m.T * m.k;
  const int mf = m.act == SMOE_ACT_SWIGLU ? 2 * m.f : m.f;
  { PROF("route", 1); SMOE_TRY(launch_route(t->x, t->w_r, t->b_r, m.T, m.d, m.E, m.k, SMOE_BF16, t->topk_idx, t->gates, err, s), "route"); }
  { PROF("sort", sort_launches(m.T, m.k, m.E)); SMOE_TRY(launch_sort(t->topk_idx, m.T, m.k, m.E, t->sorted_slot, t->expert_offsets, l.sort, err, s, l.inv), "sort"); }
  { PROF("fp8.quantize_x", 1); SMOE_TRY(launch_quantize_rows_fp8(t->x, m.T, m.d, l.x8, l.sx, s), "quantize x"); }
  {  // H = (x8 W1_8[e]) sx s1, A = act(H)   (scatter -> group, fan-out k)
    GroupedGemm g;
    g.E = m.E; g.num_rows = S; g.offsets = t->expert_offsets; g.sorted_slot = t->sorted_slot;
    g.K = m.d; g.a = l.x8; g.lda = m.d; g.a_rows = m.T; g.a_mode = ROWS_GATHER; g.a_fan_out = m.k;
    g.b = w8->w1q; g.b_kn = 0; g.NW = mf; g.n_out = m.f;
    g.epi = EPI_ACT_FWD; g.act = m.act;
    g.out_mode = ROWS_GROUPED; g.out = t->h; g.ldo = mf; g.out2 = t->a; g.ldo2 = m.f;
    g.fp8 = 1; g.row_scale = l.sx; g.col_scale = w8->s1; g.err = err;
    { PROF("gemm.fwd_up_fp8", 1); SMOE_TRY(launch_grouped_gemm_tc(g, s), "fp8 gemm1"); }
  }
  { PROF("fp8.quantize_a", 1); SMOE_TRY(launch_quantize_rows_fp8(t->a, S, m.f, l.a8, l.sa, s), "quantize a"); }
  {  // slot rows g (a8 W2_8[e]) sa s2   (group -> group; the k-way combine scatters)
    GroupedGemm g;
    g.E = m.E; g.num_rows = S; g.offsets = t->expert_offsets; g.sorted_slot = t->sorted_slot;
    g.K = m.f; g.a = l.a8; g.lda = m.f; g.a_rows = S; g.a_mode = ROWS_GROUPED;
    g.b = w8->w2q; g.b_kn = 0; g.NW = m.d; g.n_out = m.d;
    g.epi = EPI_STORE; g.gates = t->gates;
    g.out_mode = ROWS_GROUPED; g.out = l.ycomb; g.ldo = m.d;
    g.ksplit = l.ksplit; g.partial = l.kpart;
    g.fp8 = 1; g.row_scale = l.sa; g.col_scale = w8->s2; g.err = err;
    { PROF("gemm.fwd_down_fp8", 1); SMOE_TRY(launch_grouped_gemm_tc(g, s), "fp8 gemm2"); }
    if (l.ksplit > 1) {
      PROF("splitk_reduce", 1);
      SMOE_TRY(launch_splitk_reduce(l.kpart, l.ksplit, S, m.d, t->sorted_slot, t->gates, l.ycomb, m.d, s),
               "fp8 split-K reduce");
    }
  }
  { PROF("combine.y", 1); SMOE_TRY(launch_combine(l.ycomb, l.inv, m.T, m.k, m.d, t->y, SMOE_BF16, nullptr, nullptr, nullptr, 0, s), "fp8 combine"); }
  return SMOE_OK;
}

// ---------------------------------------------------------------------------
// SMoE MLP
// ---------------------------------------------------------------------------
size_t smoe_mlp_workspace_size(const smoe_mlp_desc* desc, int backward) {
  if (validate_mlp_desc(desc) != SMOE_OK) return 0;
  return mlp_layout(nullptr, *desc, backward).bytes;
}

int smoe_mlp_fwd(const smoe_mlp_desc* desc, const smoe_mlp_tensors* t, void* stream) {
  smoe::NvtxScope nvtx_scope("smoe_mlp_fwd");
  int rc = validate_mlp_desc(desc);
  if (rc != SMOE_OK) return rc;
  NEED(t, "tensors");
  const smoe_mlp_desc& m = *desc;
  if (m.T == 0) return SMOE_OK;
  NEED(t->x, "x"); NEED(t->w_r, "w_r"); NEED(t->w1, "w1"); NEED(t->w2, "w2"); NEED(t->y, "y");
  NEED(t->topk_idx, "topk_idx"); NEED(t->gates, "gates"); NEED(t->sorted_slot, "sorted_slot");
  NEED(t->expert_offsets, "expert_offsets"); NEED(t->h, "h"); NEED(t->a, "a");
  ALIGNED(t->x, "x"); ALIGNED(t->w_r, "w_r"); ALIGNED(t->w1, "w1"); ALIGNED(t->w2, "w2");
  ALIGNED(t->y, "y"); ALIGNED(t->h, "h"); ALIGNED(t->a, "a");
  MlpWs l = mlp_layout(t->workspace, m, 0);
  if (!t->workspace || t->workspace_bytes < l.bytes)
    return fail(SMOE_ERR_INVALID_ARG, "workspace too small (%zu < %zu)", t->workspace_bytes, l.bytes);
  if (((uintptr_t)t->workspace & 255u) != 0) return fail(SMOE_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  const smoe_dtype dt = (smoe_dtype)m.dtype;
  if ((rc = check_tc(dt)) != SMOE_OK) return rc;
  cudaError_t st;
  unsigned* err = error_word(&st);
  if (!err) return cuda_fail(st, "smoe_mlp_fwd");
  cudaStream_t s = (cudaStream_t)stream;
  const int S = m.T * m.k;
  const int mf = m.act == SMOE_ACT_SWIGLU ? 2 * m.f : m.f;

  { PROF("route", 1); SMOE_TRY(launch_route(t->x, t->w_r, t->b_r, m.T, m.d, m.E, m.k, dt, t->topk_idx, t->gates, err, s), "route"); }
  { PROF("sort", sort_launches(m.T, m.k, m.E)); SMOE_TRY(launch_sort(t->topk_idx, m.T, m.k, m.E, t->sorted_slot, t->expert_offsets, l.sort, err, s, l.inv), "sort"); }
  {  // H = x[gathered] W1, A = act(H)   (scatter -> group, fan-out k)
    GroupedGemm g;
    g.E = m.E; g.num_rows = S; g.offsets = t->expert_offsets; g.sorted_slot = t->sorted_slot;
    g.K = m.d; g.a = t->x; g.lda = m.d; g.a_rows = m.T; g.a_mode = ROWS_GATHER; g.a_fan_out = m.k;
    g.b = t->w1; g.b_kn = 1; g.NW = mf; g.n_out = m.f;
    g.epi = EPI_ACT_FWD; g.act = m.act;
    g.out_mode = ROWS_GROUPED; g.out = t->h; g.ldo = mf; g.out_f32 = 0;
    g.out2 = t->a; g.ldo2 = m.f; g.err = err;
    { PROF("gemm.fwd_up", 1); SMOE_TRY(run_grouped(g, dt, s), "mlp fwd gemm1"); }
  }
  {  // y = sum_j g * (A W2)   (group -> group in fp32, gated; the k-way combine scatters)
    GroupedGemm g;
    g.E = m.E; g.num_rows = S; g.offsets = t->expert_offsets; g.sorted_slot = t->sorted_slot;
    g.K = m.f; g.a = t->a; g.lda = m.f; g.a_rows = S; g.a_mode = ROWS_GROUPED;
    g.b = t->w2; g.b_kn = 1; g.NW = m.d; g.n_out = m.d;
    g.epi = EPI_STORE; g.gates = t->gates;
    g.out_mode = ROWS_GROUPED; g.out = l.ycomb; g.ldo = m.d; g.out_f32 = dt == SMOE_F32; g.err = err;
    g.ksplit = l.ksplit; g.partial = l.kpart;
    { PROF("gemm.fwd_down", 1); SMOE_TRY(run_grouped(g, dt, s), "mlp fwd gemm2"); }
    if (l.ksplit > 1) {
      PROF("splitk_reduce", 1);
      SMOE_TRY(launch_splitk_reduce(l.kpart, l.ksplit, S, m.d, t->sorted_slot, t->gates, l.ycomb,
                                    m.d, s), "mlp fwd split-K reduce");
    }
  }
  { PROF("combine.y", 1); SMOE_TRY(launch_combine(l.ycomb, l.inv, m.T, m.k, m.d, t->y, dt, nullptr, nullptr, nullptr, 0, s), "mlp fwd combine"); }
  return SMOE_OK;
}

int smoe_mlp_bwd(const smoe_mlp_desc* desc, const smoe_mlp_tensors* t, void* stream) {
  smoe::NvtxScope nvtx_scope("smoe_mlp_bwd");
  int rc = validate_mlp_desc(desc);
  if (rc != SMOE_OK) return rc;
  NEED(t, "tensors");
  const smoe_mlp_desc& m = *desc;
  const smoe_dtype dt = (smoe_dtype)m.dtype;
  const int mf = m.act == SMOE_ACT_SWIGLU ? 2 * m.f : m.f;
  NEED(t->dw1, "dw1"); NEED(t->dw2, "dw2"); NEED(t->dw_r, "dw_r");
  cudaStream_t s = (cudaStream_t)stream;
  if (m.T == 0) {
    SMOE_TRY(cudaMemsetAsync(t->dw1, 0, (size_t)m.E * m.d * mf * 4, s), "zero");
    SMOE_TRY(cudaMemsetAsync(t->dw2, 0, (size_t)m.E * m.f * m.d * 4, s), "zero");
    SMOE_TRY(cudaMemsetAsync(t->dw_r, 0, (size_t)m.d * m.E * 4, s), "zero");
    if (t->db_r) SMOE_TRY(cudaMemsetAsync(t->db_r, 0, (size_t)m.E * 4, s), "zero");
    return SMOE_OK;
  }
  NEED(t->x, "x"); NEED(t->w_r, "w_r"); NEED(t->w1, "w1"); NEED(t->w2, "w2");
  NEED(t->topk_idx, "topk_idx"); NEED(t->gates, "gates"); NEED(t->sorted_slot, "sorted_slot");
  NEED(t->expert_offsets, "expert_offsets"); NEED(t->h, "h"); NEED(t->a, "a");
  NEED(t->dy, "dy"); NEED(t->dx, "dx");
  ALIGNED(t->dy, "dy"); ALIGNED(t->dx, "dx"); ALIGNED(t->h, "h"); ALIGNED(t->a, "a");
  MlpWs l = mlp_layout(t->workspace, m, 1);
  if (!t->workspace || t->workspace_bytes < l.bytes)
    return fail(SMOE_ERR_INVALID_ARG, "workspace too small (%zu < %zu)", t->workspace_bytes, l.bytes);
  if (((uintptr_t)t->workspace & 255u) != 0) return fail(SMOE_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  if ((rc = check_tc(dt)) != SMOE_OK) return rc;
  cudaError_t st;
  unsigned* err = error_word(&st);
  if (!err) return cuda_fail(st, "smoe_mlp_bwd");
  const int S = m.T * m.k;
  float* dg = t->dgates ? t->dgates : l.dg;

  {  // dA' = dy[gathered] W2^T; fused: dg partials, gA = g A, dH = g dA' act'(H)
    GroupedGemm g;
    g.E = m.E; g.num_rows = S; g.offsets = t->expert_offsets; g.sorted_slot = t->sorted_slot;
    g.K = m.d; g.a = t->dy; g.lda = m.d; g.a_rows = m.T; g.a_mode = ROWS_GATHER; g.a_fan_out = m.k;
    g.b = t->w2; g.b_kn = 0; g.NW = m.f; g.n_out = m.f;
    g.epi = EPI_ACT_BWD; g.act = m.act; g.gates = t->gates;
    g.aux_a = t->a; g.ld_aux_a = m.f; g.aux_a_mode = ROWS_GROUPED; g.aux_a_fan_out = 1;
    g.aux_h = t->h; g.ld_aux_h = mf;
    g.out_mode = ROWS_GROUPED; g.out = l.dh; g.ldo = mf; g.out_f32 = dt == SMOE_F32;
    g.out2 = l.ga; g.ldo2 = m.f;
    g.dg_partial = l.dg_part; g.dg_ld = l.dg_ld; g.err = err;
    { PROF("gemm.bwd_dA", 1); SMOE_TRY(run_grouped(g, dt, s), "mlp bwd gemm dA"); }
  }
  { PROF("dg_reduce", 1); SMOE_TRY(launch_dg_reduce(l.dg_part, l.dg_ld, l.dg_ld, t->sorted_slot, S, dg, s, l.inv), "mlp bwd dg"); }
  { PROF("route_dl", 1); SMOE_TRY(launch_route_dl(t->gates, dg, m.T, m.k, l.dl, s), "mlp bwd dl"); }
  {  // dW2[e] = sum_i (g A)_i^T dy[t_i].  g A comes from the dA' epilogue: measured
     // faster than multiplying dY's gathered rows by g inside the dW kernel
     // (Mixtral-shaped step: dW2 4.5 ms against 7.6 ms, the epilogue's extra
     // store 0.4 ms), since a gated stage can only be handed to the tensor core
     // after its copies land, which shortens the gather's look-ahead.
    DwGemm g;
    g.E = m.E; g.num_rows = S; g.offsets = t->expert_offsets; g.sorted_slot = t->sorted_slot;
    g.M = m.f; g.N = m.d;
    g.a = l.ga; g.lda = m.f; g.a_rows = S; g.a_mode = ROWS_GROUPED; g.a_fan_out = 1;
    g.b = t->dy; g.ldb = m.d; g.b_rows = m.T; g.b_mode = ROWS_GATHER; g.b_fan_out = m.k;
    g.dw = t->dw2; g.err = err;
    { PROF("gemm.bwd_dW2", 1); SMOE_TRY(run_dw(g, dt, s), "mlp bwd dW2"); }
  }
  {  // dW1[e] = sum_i x[t_i]^T dH_i
    DwGemm g;
    g.E = m.E; g.num_rows = S; g.offsets = t->expert_offsets; g.sorted_slot = t->sorted_slot;
    g.M = m.d; g.N = mf;
    g.a = t->x; g.lda = m.d; g.a_rows = m.T; g.a_mode = ROWS_GATHER; g.a_fan_out = m.k;
    g.b = l.dh; g.ldb = mf; g.b_rows = S; g.b_mode = ROWS_GROUPED; g.b_fan_out = 1;
    g.dw = t->dw1; g.err = err;
    { PROF("gemm.bwd_dW1", 1); SMOE_TRY(run_dw(g, dt, s), "mlp bwd dW1"); }
  }
  {  // per-slot dx rows: dH_i W1[e]^T  (group -> group, fp32; the combine scatters)
    GroupedGemm g;
    g.E = m.E; g.num_rows = S; g.offsets = t->expert_offsets; g.sorted_slot = t->sorted_slot;
    g.K = mf; g.a = l.dh; g.lda = mf; g.a_rows = S; g.a_mode = ROWS_GROUPED;
    g.b = t->w1; g.b_kn = 0; g.NW = m.d; g.n_out = m.d;
    g.epi = EPI_STORE;
    g.out_mode = ROWS_GROUPED; g.out = l.dxcomb; g.ldo = m.d; g.out_f32 = dt == SMOE_F32; g.err = err;
    { PROF("gemm.bwd_dx", 1); SMOE_TRY(run_grouped(g, dt, s), "mlp bwd gemm dx"); }
  }
  // dx[t] = sum_j rows + router term sum_j dl W_r[:, e_j]
  { PROF("transpose_wr", 1);
  SMOE_TRY(launch_transpose_wr(t->w_r, m.d, m.E, dt, l.wrt, s), "mlp bwd router transpose"); }
  { PROF("combine.dx", 1);
  SMOE_TRY(launch_combine(l.dxcomb, l.inv, m.T, m.k, m.d, t->dx, dt, l.dl, t->topk_idx, l.wrt, m.E, s),
           "mlp bwd dx combine"); }
  { PROF("route_dw", 2);
  SMOE_TRY(launch_route_dw(t->x, t->topk_idx, t->sorted_slot, t->expert_offsets, l.dl, m.T, m.d,
                           m.E, m.k, dt, l.rpart,
                           t->dw_r, t->db_r, s), "mlp bwd router dW"); }
  return SMOE_OK;
}

int smoe_set_gemm_policy(int policy) {
  if (policy != 0 && policy != 1) return api_fail(SMOE_ERR_INVALID_ARG, "gemm policy must be 0 or 1");
  set_gemm_policy(policy);
  return SMOE_OK;
}

}  // extern "C"
