/*
 * smoe_oracle.cpp -- plain, slow fp64 CPU oracle of the sparse Mixture-of-Experts
 * (SMoE) MLP and of ParallelLinear, written from the ScatterMoE pages:
 *   - "Scattered Mixture-of-Experts Implementation" (arXiv 2403.08245), abstract:
 *     an SMoE layer built from ParallelLinear, extended to Mixture of Attention.
 *   - library page of arXiv 2403.08245, review 1 summary: ParallelLinear's input
 *     and output may each be grouped (expert-sorted) or scattered (token order),
 *     and it serves forward and backward.
 *   - library page of arXiv 2403.08245, review 2 summary: one kernel covering
 *     group-to-group, group-to-scatter, scatter-to-scatter and scatter-to-group.
 *   - tradepoint.io article "This Machine Learning Research Presents ScatterMoE",
 *     method paragraph: grouped matrix operations on scattered groups; the backward
 *     pass computes the gradient of each expert.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
 * this file.  Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline
 * and reference legs use it.  It shares no code, header or table with the CUDA
 * library.
 *
 * Readings (the pages print no equations; each plain reading is listed here):
 *   R1 router: logits l = x W_r + b; the k largest logits (descending, ties to
 *      the lower expert id) are selected; gates are the softmax over the selected
 *      logits, which equals softmax-then-top-k-then-renormalise.
 *   R2 the top-k decision is taken in fp32 on logits accumulated in the order the
 *      CUDA route kernel documents (see oracle_router_logits_f32), so that the
 *      integer outputs can be compared bit for bit.  Gates are computed in fp64
 *      from those fp32 logits.
 *   R3 slots p = t*k + j; the reorder is a stable sort of slots by expert id;
 *      expert_offsets[e] = number of slots whose expert is < e.
 *   R4 expert MLP: GELU(tanh): a = gelu(x W1[e]); SwiGLU: W1[e] holds the gate
 *      columns [0,f) and the up columns [f,2f), a = silu(x Wg) * (x Wu);
 *      o = a W2[e]; y_t = sum_j g[t,j] o_{t*k+j}.
 *   R5 backward of L = <y, dY> by plain reverse mode; router gradient through
 *      the renormalised softmax only (top-k selection is piecewise constant).
 *   R6 ParallelLinear: for grouped row i (expert e = expert owning i,
 *      p = sorted_slot[i]) the input row is x[i] (grouped) or x[p / fan_out]
 *      (scattered); the product v = x_row W[e] goes to row i (grouped), row p
 *      (scattered), or is summed into row p / combine_k (k-way combine),
 *      multiplied by gates[p] when gates are given.
 *   R7 Mixture-of-Attention core (see oracle_moa_attn): per-expert queries in
 *      grouped order attend causally, within each sequence of L tokens, to keys
 *      and values shared by all experts, head by head.
 *   R8 FP8 inference forward (see oracle_mlp_fwd_fp8): e4m3 codes with one fp32
 *      scale per expert output column (weights) and per row (x, and A stored in
 *      bf16 first); the quantisation decisions are taken in fp32, the products in
 *      fp64 from the decoded codes.
 *
 * Every input array is passed as its stored values (fp32, or bf16 bit patterns)
 * and upcast exactly to fp64.  All arithmetic below is fp64 except the fp32
 * router logits of R2.
 */
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

/* ---- stored element types ---------------------------------------------- */
struct bf16s { uint16_t bits; };

inline float to_float(float v) { return v; }
inline double to_float(double v) { return v; }
inline float to_float(bf16s v) {
  uint32_t u = (uint32_t)v.bits << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

/* element i of an array stored as dtype code dt (0 fp32, 1 bf16, 2 fp64) */
inline double load_any(const void* p, int dt, size_t i) {
  if (dt == 0) return ((const float*)p)[i];
  if (dt == 1) return to_float(((const bf16s*)p)[i]);
  return ((const double*)p)[i];
}

/* ---- activations (R4) -------------------------------------------------- */
const double kSqrt2OverPi = 0.79788456080286535588;  /* sqrt(2/pi) */
const double kGeluC = 0.044715;

double gelu_tanh(double h) {
  double u = kSqrt2OverPi * (h + kGeluC * h * h * h);
  return 0.5 * h * (1.0 + std::tanh(u));
}
double gelu_tanh_grad(double h) {
  double u = kSqrt2OverPi * (h + kGeluC * h * h * h);
  double th = std::tanh(u);
  double du = kSqrt2OverPi * (1.0 + 3.0 * kGeluC * h * h);
  return 0.5 * (1.0 + th) + 0.5 * h * (1.0 - th * th) * du;
}
double sigmoid(double z) { return 1.0 / (1.0 + std::exp(-z)); }
double silu(double z) { return z * sigmoid(z); }
double silu_grad(double z) {
  double s = sigmoid(z);
  return s * (1.0 + z * (1.0 - s));
}

enum { ACT_GELU_TANH = 0, ACT_SWIGLU = 1, ACT_NONE = 2 };

/* ---- the expert MLP of one slot (R4) -----------------------------------
 * h[mf] = x_t W1[e];  a[f] = act(h);  o[d] = a W2[e].                        */
template <typename TX, typename TW>
void expert_forward(const TX* x_t, const TW* W1e, const TW* W2e, int d, int f, int act,
                    std::vector<double>& h, std::vector<double>& a, std::vector<double>& o) {
  const int mf = (act == ACT_SWIGLU) ? 2 * f : f;
  h.assign(mf, 0.0);
  for (int i = 0; i < d; ++i) {
    const double xi = to_float(x_t[i]);
    const TW* row = W1e + (size_t)i * mf;
    for (int n = 0; n < mf; ++n) h[n] += xi * (double)to_float(row[n]);
  }
  a.assign(f, 0.0);
  for (int c = 0; c < f; ++c)
    a[c] = (act == ACT_SWIGLU) ? silu(h[c]) * h[f + c] : gelu_tanh(h[c]);
  o.assign(d, 0.0);
  for (int c = 0; c < f; ++c) {
    const double ac = a[c];
    const TW* row = W2e + (size_t)c * d;
    for (int n = 0; n < d; ++n) o[n] += ac * (double)to_float(row[n]);
  }
}

/* ---- the expert MLP backward of one slot (R5) ----------------------------
 * Given the upstream row dy_t and gate g:
 *   dg   = <dy_t, o>                (gate gradient)
 *   da'  = dy_t W2[e]^T             (ungated)
 *   da   = g da'
 *   dh   = da * act'(h)             (GELU)   or  [da*hu*silu'(hg) | da*silu(hg)]
 *   dx  += dh W1[e]^T                                                        */
template <typename TX, typename TW>
void expert_backward(const TX* x_t, const TW* W1e, const TW* W2e, const double* dy_t, double g,
                     int d, int f, int act, const std::vector<double>& h,
                     const std::vector<double>& o, double* dg_out, std::vector<double>& dh,
                     double* dx_t /* accumulated, may be null */) {
  const int mf = (act == ACT_SWIGLU) ? 2 * f : f;
  double dg = 0.0;
  for (int n = 0; n < d; ++n) dg += dy_t[n] * o[n];
  *dg_out = dg;
  dh.assign(mf, 0.0);
  for (int c = 0; c < f; ++c) {
    const TW* row = W2e + (size_t)c * d;
    double dap = 0.0;
    for (int n = 0; n < d; ++n) dap += dy_t[n] * (double)to_float(row[n]);
    const double da = g * dap;
    if (act == ACT_SWIGLU) {
      dh[c] = da * h[f + c] * silu_grad(h[c]);
      dh[f + c] = da * silu(h[c]);
    } else {
      dh[c] = da * gelu_tanh_grad(h[c]);
    }
  }
  if (dx_t) {
    for (int i = 0; i < d; ++i) {
      const TW* row = W1e + (size_t)i * mf;
      double s = 0.0;
      for (int n = 0; n < mf; ++n) s += dh[n] * (double)to_float(row[n]);
      dx_t[i] += s;
    }
  }
  (void)x_t;
}

/* Router gradient of one token through the renormalised softmax (R5):
 * dl_j = g_j (dg_j - sum_i g_i dg_i); unselected experts get 0.             */
void router_dlogits(const double* g, const double* dg, int k, double* dl) {
  double s = 0.0;
  for (int j = 0; j < k; ++j) s += g[j] * dg[j];
  for (int j = 0; j < k; ++j) dl[j] = g[j] * (dg[j] - s);
}

/* expert owning grouped row i, from the exclusive offsets */
int expert_of_row(const int32_t* offsets, int E, int i) {
  int e = 0;
  while (e + 1 <= E && offsets[e + 1] <= i) ++e;
  return e;
}

/* ======================================================================= */
/* typed implementations                                                   */
/* ======================================================================= */

template <typename TX, typename TW>
void mlp_fwd_impl(const TX* x, const TW* w1, const TW* w2, int d, int f, int E, int k, int act,
                  const int32_t* idx, const double* gates, const int32_t* tokens, int n_tok,
                  double* y, double* h_out, double* a_out) {
  const int mf = (act == ACT_SWIGLU) ? 2 * f : f;
#pragma omp parallel for schedule(dynamic, 1)
  for (int q = 0; q < n_tok; ++q) {
    const int t = tokens[q];
    std::vector<double> h, a, o;
    double* yq = y + (size_t)q * d;
    for (int n = 0; n < d; ++n) yq[n] = 0.0;
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      expert_forward(x + (size_t)t * d, w1 + (size_t)e * d * mf, w2 + (size_t)e * f * d, d, f,
                     act, h, a, o);
      const double g = gates[(size_t)t * k + j];
      for (int n = 0; n < d; ++n) yq[n] += g * o[n];
      if (h_out) std::memcpy(h_out + ((size_t)q * k + j) * mf, h.data(), sizeof(double) * mf);
      if (a_out) std::memcpy(a_out + ((size_t)q * k + j) * f, a.data(), sizeof(double) * f);
    }
  }
  (void)E;
}

template <typename TX, typename TW>
void mlp_bwd_tokens_impl(const TX* x, const TX* w_r, const TW* w1, const TW* w2, int d, int f,
                         int E, int k, int act, const int32_t* idx, const double* gates,
                         const double* dy, const int32_t* tokens, int n_tok, double* dx,
                         double* dg, double* dl) {
  const int mf = (act == ACT_SWIGLU) ? 2 * f : f;
#pragma omp parallel for schedule(dynamic, 1)
  for (int q = 0; q < n_tok; ++q) {
    const int t = tokens[q];
    std::vector<double> h, a, o, dh;
    double* dxq = dx + (size_t)q * d;
    for (int i = 0; i < d; ++i) dxq[i] = 0.0;
    const double* dy_t = dy + (size_t)t * d;
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      const TW* W1e = w1 + (size_t)e * d * mf;
      const TW* W2e = w2 + (size_t)e * f * d;
      expert_forward(x + (size_t)t * d, W1e, W2e, d, f, act, h, a, o);
      expert_backward(x + (size_t)t * d, W1e, W2e, dy_t, gates[(size_t)t * k + j], d, f, act,
                      h, o, dg + (size_t)q * k + j, dh, dxq);
    }
    router_dlogits(gates + (size_t)t * k, dg + (size_t)q * k, k, dl + (size_t)q * k);
    /* dX += dl W_r^T over the k selected experts */
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      for (int i = 0; i < d; ++i) dxq[i] += dl[(size_t)q * k + j] * (double)to_float(w_r[(size_t)i * E + e]);
    }
  }
}

/* Full backward: every dW by per-slot outer products, accumulated per expert in
 * ascending slot order; router weight and bias gradients from all tokens.   */
template <typename TX, typename TW>
void mlp_bwd_full_impl(const TX* x, const TX* w_r, const TW* w1, const TW* w2, int T, int d, int f,
                       int E, int k, int act, const int32_t* idx, const double* gates,
                       const double* dy, double* dx, double* dg, double* dw1, double* dw2,
                       double* dw_r, double* db_r) {
  const int mf = (act == ACT_SWIGLU) ? 2 * f : f;
  std::vector<int32_t> all(T);
  for (int t = 0; t < T; ++t) all[t] = t;
  std::vector<double> dl((size_t)T * k);
  mlp_bwd_tokens_impl(x, w_r, w1, w2, d, f, E, k, act, idx, gates, dy, all.data(), T, dx, dg,
                      dl.data());
  /* per-expert weight gradients: one thread per expert, slots in ascending order */
#pragma omp parallel for schedule(dynamic, 1)
  for (int e = 0; e < E; ++e) {
    double* dW1 = dw1 + (size_t)e * d * mf;
    double* dW2 = dw2 + (size_t)e * f * d;
    std::fill(dW1, dW1 + (size_t)d * mf, 0.0);
    std::fill(dW2, dW2 + (size_t)f * d, 0.0);
    std::vector<double> h, a, o, dh;
    for (int p = 0; p < T * k; ++p) {
      if (idx[p] != e) continue;
      const int t = p / k;
      const double g = gates[p];
      const TW* W1e = w1 + (size_t)e * d * mf;
      const TW* W2e = w2 + (size_t)e * f * d;
      expert_forward(x + (size_t)t * d, W1e, W2e, d, f, act, h, a, o);
      double dg_unused;
      expert_backward(x + (size_t)t * d, W1e, W2e, dy + (size_t)t * d, g, d, f, act, h, o,
                      &dg_unused, dh, nullptr);
      for (int i = 0; i < d; ++i) {
        const double xi = to_float(x[(size_t)t * d + i]);
        double* row = dW1 + (size_t)i * mf;
        for (int n = 0; n < mf; ++n) row[n] += xi * dh[n];
      }
      for (int c = 0; c < f; ++c) {
        const double gac = g * a[c];
        double* row = dW2 + (size_t)c * d;
        for (int n = 0; n < d; ++n) row[n] += gac * dy[(size_t)t * d + n];
      }
    }
  }
  /* router: dW_r[i][e] = sum_t x[t,i] dl[t,e];  db[e] = sum_t dl[t,e] */
  std::fill(dw_r, dw_r + (size_t)d * E, 0.0);
  std::fill(db_r, db_r + E, 0.0);
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      const double v = dl[(size_t)t * k + j];
      db_r[e] += v;
      for (int i = 0; i < d; ++i) dw_r[(size_t)i * E + e] += (double)to_float(x[(size_t)t * d + i]) * v;
    }
}

/* Sampled weight gradients: columns cols1 of every dW1[e] and rows rows2 of
 * every dW2[e].  Each needed entry of h, a and da' is one dot product, so this
 * scales to the full-size workloads.  Same definitions as mlp_bwd_full_impl. */
template <typename TX, typename TW>
void mlp_dw_sampled_impl(const TX* x, const TW* w1, const TW* w2, int T, int d, int f, int E,
                         int k, int act, const int32_t* idx, const double* gates, const double* dy,
                         const int32_t* cols1, int n_c1, const int32_t* rows2, int n_r2,
                         double* dw1_cols /* [E][d][n_c1] */, double* dw2_rows /* [E][n_r2][d] */) {
  const int mf = (act == ACT_SWIGLU) ? 2 * f : f;
  /* h column n of slot p: dot(x_t, W1[e][:, n]) */
  auto hcol = [&](int t, int e, int n) {
    const TW* W1e = w1 + (size_t)e * d * mf;
    double s = 0.0;
    for (int i = 0; i < d; ++i) s += (double)to_float(x[(size_t)t * d + i]) * (double)to_float(W1e[(size_t)i * mf + n]);
    return s;
  };
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int e = 0; e < E; ++e) {
    for (int q = 0; q < n_c1 + n_r2; ++q) {
      const TW* W2e = w2 + (size_t)e * f * d;
      if (q < n_c1) {
        const int n = cols1[q];
        const int c = (act == ACT_SWIGLU) ? n % f : n;
        for (int i = 0; i < d; ++i) dw1_cols[((size_t)e * d + i) * n_c1 + q] = 0.0;
        for (int p = 0; p < T * k; ++p) {
          if (idx[p] != e) continue;
          const int t = p / k;
          double dap = 0.0;
          for (int m = 0; m < d; ++m) dap += dy[(size_t)t * d + m] * (double)to_float(W2e[(size_t)c * d + m]);
          const double da = gates[p] * dap;
          double dh;
          if (act == ACT_SWIGLU) {
            const double hg = hcol(t, e, c), hu = hcol(t, e, f + c);
            dh = (n < f) ? da * hu * silu_grad(hg) : da * silu(hg);
          } else {
            dh = da * gelu_tanh_grad(hcol(t, e, c));
          }
          for (int i = 0; i < d; ++i)
            dw1_cols[((size_t)e * d + i) * n_c1 + q] += (double)to_float(x[(size_t)t * d + i]) * dh;
        }
      } else {
        const int r = rows2[q - n_c1];
        double* out = dw2_rows + ((size_t)e * n_r2 + (q - n_c1)) * d;
        for (int m = 0; m < d; ++m) out[m] = 0.0;
        for (int p = 0; p < T * k; ++p) {
          if (idx[p] != e) continue;
          const int t = p / k;
          const double ar = (act == ACT_SWIGLU) ? silu(hcol(t, e, r)) * hcol(t, e, f + r)
                                                : gelu_tanh(hcol(t, e, r));
          const double gar = gates[p] * ar;
          for (int m = 0; m < d; ++m) out[m] += gar * dy[(size_t)t * d + m];
        }
      }
    }
  }
}

/* ---- ParallelLinear (R6) ------------------------------------------------ */
struct PLMaps {
  std::vector<int> inv;     /* inv[p] = grouped row i holding slot p */
  std::vector<int> expert;  /* expert owning grouped row i */
};
PLMaps pl_maps(const int32_t* sorted_slot, const int32_t* offsets, int num_slots, int E) {
  PLMaps m;
  m.inv.assign(num_slots, -1);
  m.expert.assign(num_slots, 0);
  for (int i = 0; i < num_slots; ++i) {
    m.inv[sorted_slot[i]] = i;
    m.expert[i] = expert_of_row(offsets, E, i);
  }
  return m;
}

/* rows of y computed: all of them (out_rows == null) or the listed ones */
template <typename TX, typename TW>
void pl_fwd_impl(const TX* x, const TW* w, int K, int N, int E, const int32_t* sorted_slot,
                 const int32_t* offsets, int num_slots, int fan_out, int grouped_in,
                 int grouped_out, const double* gates, int combine_k, const int32_t* out_rows,
                 int n_out, double* y) {
  PLMaps m = pl_maps(sorted_slot, offsets, num_slots, E);
#pragma omp parallel for schedule(dynamic, 4)
  for (int q = 0; q < n_out; ++q) {
    const int row = out_rows ? out_rows[q] : q;
    double* yq = y + (size_t)q * N;
    for (int n = 0; n < N; ++n) yq[n] = 0.0;
    /* the grouped rows i that write output row `row` */
    std::vector<int> contrib;
    if (combine_k > 0) {
      for (int j = 0; j < combine_k; ++j) contrib.push_back(m.inv[(size_t)row * combine_k + j]);
    } else {
      contrib.push_back(grouped_out ? row : m.inv[row]);
    }
    for (int i : contrib) {
      const int p = sorted_slot[i];
      const int e = m.expert[i];
      const int xr = grouped_in ? i : p / fan_out;
      const double g = gates ? gates[p] : 1.0;
      const TW* We = w + (size_t)e * K * N;
      for (int kk = 0; kk < K; ++kk) {
        const double xv = g * (double)to_float(x[(size_t)xr * K + kk]);
        const TW* wrow = We + (size_t)kk * N;
        for (int n = 0; n < N; ++n) yq[n] += xv * (double)to_float(wrow[n]);
      }
    }
  }
}

/* Backward of ParallelLinear against the upstream gradient dy (shaped like y).
 *   G_i       = dy[p / combine_k] (combine) or dy[out row of i]
 *   dx[in(i)] += g_p G_i W[e]^T      for the listed x rows (or all)
 *   dw[e][:, c] = sum_i x[in(i)] (g_p G_i[c])   for the listed columns (or all)
 *   dgates[p]   = <G_i, x[in(i)] W[e]>         for the listed slots (or all)  */
template <typename TX, typename TW, typename TD>
void pl_bwd_impl(const TD* dy, const TX* x, const TW* w, int x_rows, int K, int N, int E,
                 const int32_t* sorted_slot, const int32_t* offsets, int num_slots, int fan_out,
                 int grouped_in, int grouped_out, const double* gates, int combine_k,
                 const int32_t* dx_rows, int n_dx, double* dx, const int32_t* dw_cols, int n_dw,
                 double* dw, const int32_t* dg_slots, int n_dg, double* dgates) {
  PLMaps m = pl_maps(sorted_slot, offsets, num_slots, E);
  auto in_row = [&](int i) { return grouped_in ? i : sorted_slot[i] / fan_out; };
  auto g_row = [&](int i) {
    const int p = sorted_slot[i];
    return combine_k > 0 ? p / combine_k : (grouped_out ? i : p);
  };
  auto gate = [&](int i) { return gates ? gates[sorted_slot[i]] : 1.0; };
  /* dx: grouped rows contributing to x row r */
  if (dx) {
    std::vector<std::vector<int>> writers(x_rows);
    for (int i = 0; i < num_slots; ++i) writers[in_row(i)].push_back(i);
#pragma omp parallel for schedule(dynamic, 4)
    for (int q = 0; q < n_dx; ++q) {
      const int r = dx_rows ? dx_rows[q] : q;
      double* out = dx + (size_t)q * K;
      for (int kk = 0; kk < K; ++kk) out[kk] = 0.0;
      for (int i : writers[r]) {
        const int e = m.expert[i];
        const TW* We = w + (size_t)e * K * N;
        const TD* G = dy + (size_t)g_row(i) * N;
        const double g = gate(i);
        for (int kk = 0; kk < K; ++kk) {
          double s = 0.0;
          for (int n = 0; n < N; ++n) s += (double)to_float(G[n]) * (double)to_float(We[(size_t)kk * N + n]);
          out[kk] += g * s;
        }
      }
    }
  }
  if (dw) {
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int e = 0; e < E; ++e)
      for (int q = 0; q < n_dw; ++q) {
        const int c = dw_cols ? dw_cols[q] : q;
        for (int kk = 0; kk < K; ++kk) dw[((size_t)e * K + kk) * n_dw + q] = 0.0;
        for (int i = offsets[e]; i < offsets[e + 1]; ++i) {
          const double gv = gate(i) * (double)to_float(dy[(size_t)g_row(i) * N + c]);
          const TX* xr = x + (size_t)in_row(i) * K;
          for (int kk = 0; kk < K; ++kk) dw[((size_t)e * K + kk) * n_dw + q] += (double)to_float(xr[kk]) * gv;
        }
      }
  }
  if (dgates) {
#pragma omp parallel for schedule(dynamic, 4)
    for (int q = 0; q < n_dg; ++q) {
      const int p = dg_slots ? dg_slots[q] : q;
      const int i = m.inv[p];
      const int e = m.expert[i];
      const TW* We = w + (size_t)e * K * N;
      const TX* xr = x + (size_t)in_row(i) * K;
      const TD* G = dy + (size_t)g_row(i) * N;
      double s = 0.0;
      for (int n = 0; n < N; ++n) {
        double v = 0.0;
        for (int kk = 0; kk < K; ++kk) v += (double)to_float(xr[kk]) * (double)to_float(We[(size_t)kk * N + n]);
        s += (double)to_float(G[n]) * v;
      }
      dgates[q] = s;
    }
  }
}

/* dtype dispatch: 0 = fp32, 1 = bf16 bit patterns, 2 = fp64 (inputs and
 * weights share one dtype; fp64 serves the finite-difference pins). */
#define SMOE_ORACLE_DISPATCH2(dx_, dw_, CALL)                                  \
  do {                                                                        \
    if ((dx_) != (dw_)) break;                                                \
    if ((dx_) == 0) { typedef float TX; typedef float TW; CALL; }             \
    else if ((dx_) == 1) { typedef bf16s TX; typedef bf16s TW; CALL; }        \
    else { typedef double TX; typedef double TW; CALL; }                      \
  } while (0)

/* R8: FP8 (e4m3) inference forward (sourcepulse.org summary: inference speed).
 * e4m3 as the OCP 8-bit floating-point format defines it: 1 sign bit, 4 exponent
 * bits (bias 7), 3 mantissa bits; normal values (1 + m/8) 2^(e-7) for e = 1..15
 * (except e = 15, m = 7, which is NaN), subnormal values (m/8) 2^-6; largest 448.
 * e4m3_round: round to nearest, ties to even mantissa, saturating at +-448. */
double e4m3_round(double x) {
  if (x == 0.0 || std::isnan(x)) return x;
  const double a = std::fabs(x);
  double q;
  if (a >= 448.0) {
    q = 448.0;
  } else {
    int e = (int)std::floor(std::log2(a));
    if (std::ldexp(1.0, e) > a) --e;          /* guard log2 rounding */
    if (std::ldexp(1.0, e + 1) <= a) ++e;
    const double quantum = e < -6 ? std::ldexp(1.0, -9) : std::ldexp(1.0, e - 3);
    const double n = a / quantum;             /* exact: a power-of-two scaling */
    double r = std::floor(n);
    const double frac = n - r;
    if (frac > 0.5 || (frac == 0.5 && std::fmod(r, 2.0) != 0.0)) r += 1.0;
    q = std::min(r * quantum, 448.0);
  }
  return x < 0 ? -q : q;
}
/* bits of an e4m3 value produced by e4m3_round (finite, |v| <= 448) */
uint8_t e4m3_bits(double v) {
  const uint8_t s = (std::signbit(v) ? 0x80 : 0x00);
  const double a = std::fabs(v);
  if (a == 0.0) return s;
  if (a < std::ldexp(1.0, -6)) return (uint8_t)(s | (uint8_t)std::lround(a / std::ldexp(1.0, -9)));
  int e = (int)std::floor(std::log2(a));
  if (std::ldexp(1.0, e) > a) --e;
  if (std::ldexp(1.0, e + 1) <= a) ++e;
  const int m = (int)std::lround((a / std::ldexp(1.0, e) - 1.0) * 8.0);
  return (uint8_t)(s | (uint8_t)((e + 7) << 3) | (uint8_t)m);
}
double e4m3_value(uint8_t b) {
  const int s = b >> 7, e = (b >> 3) & 15, m = b & 7;
  const double v = e == 0 ? std::ldexp((double)m / 8.0, -6) : std::ldexp(1.0 + m / 8.0, e - 7);
  return s ? -v : v;
}
/* Row quantisation (the kernels' decision precision, fp32): scale = fl32(amax / 448)
 * (1 for an all-zero row), code = e4m3(fl32(v / scale)). */
void quantize_row_fp8(const double* v, int n, uint8_t* codes, float* scale) {
  float amax = 0.0f;
  for (int i = 0; i < n; ++i) amax = std::max(amax, (float)std::fabs(v[i]));
  const float s = amax > 0.0f ? amax / 448.0f : 1.0f;
  for (int i = 0; i < n; ++i) codes[i] = e4m3_bits(e4m3_round((double)((float)v[i] / s)));
  *scale = s;
}

/* bf16 storage of a value (round to nearest even from fp32), as the kernels store
 * activations */
bf16s bf16_round(double v) {
  const float f = (float)v;
  uint32_t u;
  std::memcpy(&u, &f, 4);
  const uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  bf16s r;
  r.bits = (uint16_t)(u >> 16);
  return r;
}

}  // namespace

extern "C" {

/* R2: fp32 router logits in the CUDA route kernel's documented order.
 * For token t and expert e, lane L (0..31) of a 32-lane group accumulates the
 * products x[t,i]*W_r[i,e] for every i with i % 32 == L, in ascending i,
 * as acc = fmaf(x, w, acc) from +0.  The 32 lane sums are then combined by an
 * xor butterfly: for off = 16, 8, 4, 2, 1: s[L] = s[L] + s[L ^ off].  The
 * logit is s[0] + b[e] (a single fp32 add; b == null means 0 and no add).     */
void oracle_router_logits_f32(const void* x, const void* w_r, int dt, const float* b_r, int T,
                              int d, int E, float* logits) {
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) {
      float s[32];
      for (int L = 0; L < 32; ++L) s[L] = 0.0f;
      for (int i = 0; i < d; ++i) {
        const int L = i % 32;
        float xv, wv;
        if (dt == 0) {
          xv = ((const float*)x)[(size_t)t * d + i];
          wv = ((const float*)w_r)[(size_t)i * E + e];
        } else {
          xv = to_float(((const bf16s*)x)[(size_t)t * d + i]);
          wv = to_float(((const bf16s*)w_r)[(size_t)i * E + e]);
        }
        s[L] = std::fmaf(xv, wv, s[L]);
      }
      for (int off = 16; off >= 1; off /= 2) {
        float nxt[32];
        for (int L = 0; L < 32; ++L) nxt[L] = s[L] + s[L ^ off];
        for (int L = 0; L < 32; ++L) s[L] = nxt[L];
      }
      logits[(size_t)t * E + e] = b_r ? s[0] + b_r[e] : s[0];
    }
  }
}

/* fp64 logits (no rounding order), used to report near-tie tokens and by the
 * finite-difference pins.  dt: 0 fp32, 1 bf16, 2 fp64. */
void oracle_router_logits_f64(const void* x, const void* w_r, int dt, const float* b_r, int T,
                              int d, int E, double* logits) {
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t)
    for (int e = 0; e < E; ++e) {
      double s = 0.0;
      for (int i = 0; i < d; ++i)
        s += load_any(x, dt, (size_t)t * d + i) * load_any(w_r, dt, (size_t)i * E + e);
      logits[(size_t)t * E + e] = s + (b_r ? (double)b_r[e] : 0.0);
    }
}

/* R1: top-k (descending, ties to the lower expert id) and gates = softmax over
 * the selected logits, computed in fp64 from the given fp32 logits.          */
void oracle_topk_gates(const float* logits, int T, int E, int k, int32_t* idx, double* gates) {
  for (int t = 0; t < T; ++t) {
    const float* l = logits + (size_t)t * E;
    std::vector<char> taken(E, 0);
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        if (best < 0 || l[e] > l[best]) best = e;
      }
      taken[best] = 1;
      idx[(size_t)t * k + j] = best;
    }
    const double mx = l[idx[(size_t)t * k]];
    double z = 0.0;
    for (int j = 0; j < k; ++j) z += std::exp((double)l[idx[(size_t)t * k + j]] - mx);
    for (int j = 0; j < k; ++j)
      gates[(size_t)t * k + j] = std::exp((double)l[idx[(size_t)t * k + j]] - mx) / z;
  }
}

/* R3: stable sort of slots by expert id and exclusive offsets. */
void oracle_sort(const int32_t* idx, int T, int k, int E, int32_t* sorted_slot, int32_t* offsets) {
  const int S = T * k;
  std::vector<int32_t> p(S);
  for (int i = 0; i < S; ++i) p[i] = i;
  std::stable_sort(p.begin(), p.end(), [&](int32_t a, int32_t b) { return idx[a] < idx[b]; });
  for (int i = 0; i < S; ++i) sorted_slot[i] = p[i];
  for (int e = 0; e <= E; ++e) offsets[e] = 0;
  for (int i = 0; i < S; ++i) offsets[idx[i] + 1] += 1;
  for (int e = 0; e < E; ++e) offsets[e + 1] += offsets[e];
}

/* Activation values and derivatives (for unit pins). act 0 = gelu(tanh), 1 = silu. */
void oracle_act(int act, const double* z, int n, double* val, double* grad) {
  for (int i = 0; i < n; ++i) {
    val[i] = act == 0 ? gelu_tanh(z[i]) : silu(z[i]);
    grad[i] = act == 0 ? gelu_tanh_grad(z[i]) : silu_grad(z[i]);
  }
}

/* R4: forward of the listed tokens.  y: [n_tok, d]; h (nullable): [n_tok*k, mf]
 * and a (nullable): [n_tok*k, f], slot-ordered within the listed tokens.     */
void oracle_mlp_fwd(const void* x, int dtx, const void* w1, const void* w2, int dtw, int d, int f,
                    int E, int k, int act, const int32_t* idx, const double* gates,
                    const int32_t* tokens, int n_tok, double* y, double* h, double* a) {
  SMOE_ORACLE_DISPATCH2(dtx, dtw,
      mlp_fwd_impl((const TX*)x, (const TW*)w1, (const TW*)w2, d, f, E, k, act, idx, gates,
                   tokens, n_tok, y, h, a));
}

/* R5: backward of the listed tokens: dx [n_tok, d] (expert and router paths),
 * dg [n_tok, k] (gate gradients), dl [n_tok, k] (router logit gradients of the
 * selected experts).  dy is fp64 [T, d].                                      */
void oracle_mlp_bwd_tokens(const void* x, int dtx, const void* w_r, const void* w1, const void* w2,
                           int dtw, int d, int f, int E, int k, int act, const int32_t* idx,
                           const double* gates, const double* dy, const int32_t* tokens, int n_tok,
                           double* dx, double* dg, double* dl) {
  SMOE_ORACLE_DISPATCH2(dtx, dtw,
      mlp_bwd_tokens_impl((const TX*)x, (const TX*)w_r, (const TW*)w1, (const TW*)w2, d, f, E, k,
                          act, idx, gates, dy, tokens, n_tok, dx, dg, dl));
}

/* R5: full backward.  dx [T,d], dg [T,k], dw1 [E,d,mf], dw2 [E,f,d], dw_r [d,E], db_r [E]. */
void oracle_mlp_bwd_full(const void* x, int dtx, const void* w_r, const void* w1, const void* w2,
                         int dtw, int T, int d, int f, int E, int k, int act, const int32_t* idx,
                         const double* gates, const double* dy, double* dx, double* dg,
                         double* dw1, double* dw2, double* dw_r, double* db_r) {
  SMOE_ORACLE_DISPATCH2(dtx, dtw,
      mlp_bwd_full_impl((const TX*)x, (const TX*)w_r, (const TW*)w1, (const TW*)w2, T, d, f, E, k,
                        act, idx, gates, dy, dx, dg, dw1, dw2, dw_r, db_r));
}

/* R5, sampled: columns cols1 of each dW1[e] -> [E, d, n_c1]; rows rows2 of each
 * dW2[e] -> [E, n_r2, d]. */
void oracle_mlp_dw_sampled(const void* x, int dtx, const void* w1, const void* w2, int dtw, int T,
                           int d, int f, int E, int k, int act, const int32_t* idx,
                           const double* gates, const double* dy, const int32_t* cols1, int n_c1,
                           const int32_t* rows2, int n_r2, double* dw1_cols, double* dw2_rows) {
  SMOE_ORACLE_DISPATCH2(dtx, dtw,
      mlp_dw_sampled_impl((const TX*)x, (const TW*)w1, (const TW*)w2, T, d, f, E, k, act, idx,
                          gates, dy, cols1, n_c1, rows2, n_r2, dw1_cols, dw2_rows));
}

/* R5, the router part alone (what smoe_route_bwd computes): given the routing
 * (idx, gates) and the gate gradients dg [T,k] (fp64), the logit gradients
 * dl [T,k] of the selected experts through the renormalised softmax, then
 *   dx_r[t,i]  = sum_j dl[t,j] W_r[i, idx[t,j]]        (the router's share of dx)
 *   dw_r[i,e]  = sum over slots (t,j) with idx = e of x[t,i] dl[t,j]
 *   db_r[e]    = sum over the same slots of dl[t,j]
 * Slots are taken in ascending order.  dx_r [T,d], dw_r [d,E], db_r [E], dl [T,k]. */
void oracle_route_bwd(const void* x, const void* w_r, int dt, int T, int d, int E, int k,
                      const int32_t* idx, const double* gates, const double* dg, double* dl,
                      double* dx_r, double* dw_r, double* db_r) {
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t) {
    router_dlogits(gates + (size_t)t * k, dg + (size_t)t * k, k, dl + (size_t)t * k);
    double* dxt = dx_r + (size_t)t * d;
    for (int i = 0; i < d; ++i) dxt[i] = 0.0;
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      const double v = dl[(size_t)t * k + j];
      for (int i = 0; i < d; ++i) dxt[i] += v * load_any(w_r, dt, (size_t)i * E + e);
    }
  }
  /* one thread per expert column: each sums its slots in ascending order */
#pragma omp parallel for schedule(dynamic, 1)
  for (int e = 0; e < E; ++e) {
    double b = 0.0;
    for (int i = 0; i < d; ++i) dw_r[(size_t)i * E + e] = 0.0;
    for (int p = 0; p < T * k; ++p) {
      if (idx[p] != e) continue;
      const int t = p / k;
      const double v = dl[p];
      b += v;
      for (int i = 0; i < d; ++i) dw_r[(size_t)i * E + e] += load_any(x, dt, (size_t)t * d + i) * v;
    }
    db_r[e] = b;
  }
}

/* R7: the Mixture-of-Attention core between the per-expert query projection and
 * the per-expert output projection (arXiv abstract: ParallelLinear extended to
 * Mixture of Attention; tradepoint.io article, method paragraph: MoA without
 * additional memory costs).  Reading: the T tokens form T / L sequences of L
 * consecutive tokens; slot p = t*kslots + j holds the query of token t for its
 * j-th selected expert, in grouped order (row inv[p] of q and o, inv the inverse
 * of sorted_slot); each of the `heads` heads of width dh attends causally, within
 * the token's sequence, to the shared keys and values of that head:
 *   s_u   = <q[inv[p], head a], k[u, head a]> / sqrt(dh)      for u in [t0, t]
 *   o[inv[p], head a] = sum_u softmax(s)_u v[u, head a],  lse = log sum_u exp(s_u)
 * (t0 = the first token of t's sequence).  Backward of L = <o, dout>:
 *   P_u = exp(s_u - lse), dP_u = <dout, v_u>, D = <dout, o> = sum_u P_u dP_u,
 *   dS_u = P_u (dP_u - D);  dq = sum_u dS_u k_u / sqrt(dh);
 *   dk_u += dS_u q / sqrt(dh);  dv_u += P_u dout      (summed over all queries).
 * q, dout: [T*kslots, heads*dh] grouped; k, v: [T, heads*dh] token order; all in
 * the stored dtype dt.  q_rows (nullable = all grouped rows): rows of o, lse, dq;
 * kv_tokens (nullable = all tokens, ignored when n_kv == 0): rows of dk, dv.
 * dout == null: forward only.                                                */
void oracle_moa_attn(const void* q, const void* k, const void* v, const void* dout, int dt,
                     const int32_t* sorted_slot, int T, int kslots, int L, int heads, int dh,
                     const int32_t* q_rows, int n_q, const int32_t* kv_tokens, int n_kv, double* o,
                     double* lse, double* dq, double* dk, double* dv) {
  const int S = T * kslots, W = heads * dh;
  const double scale = 1.0 / std::sqrt((double)dh);
  std::vector<int32_t> inv(S);
  for (int i = 0; i < S; ++i) inv[sorted_slot[i]] = i;
  auto Q = [&](int row, int a, int c) { return load_any(q, dt, (size_t)row * W + a * dh + c); };
  auto Kv = [&](int u, int a, int c) { return load_any(k, dt, (size_t)u * W + a * dh + c); };
  auto Vv = [&](int u, int a, int c) { return load_any(v, dt, (size_t)u * W + a * dh + c); };
  auto G = [&](int row, int a, int c) { return load_any(dout, dt, (size_t)row * W + a * dh + c); };
  /* scores of grouped row `row`, head a, over its causal window, into s; returns t0 */
  auto scores = [&](int row, int a, std::vector<double>& s, int& t_lo, int& t_hi) {
    const int t = sorted_slot[row] / kslots;
    t_lo = (t / L) * L;
    t_hi = t;
    s.assign(t_hi - t_lo + 1, 0.0);
    for (int u = t_lo; u <= t_hi; ++u) {
      double acc = 0.0;
      for (int c = 0; c < dh; ++c) acc += Q(row, a, c) * Kv(u, a, c);
      s[u - t_lo] = acc * scale;
    }
  };
  /* softmax of the window in place, returning lse */
  auto softmax = [&](std::vector<double>& s) {
    double m = s[0];
    for (double x : s) m = std::max(m, x);
    double z = 0.0;
    for (double& x : s) { x = std::exp(x - m); z += x; }
    for (double& x : s) x /= z;
    return m + std::log(z);
  };
  const bool all_q = q_rows == nullptr;
  const int nq = all_q ? S : n_q;
  /* forward rows and dq */
#pragma omp parallel for schedule(dynamic, 4)
  for (int qi = 0; qi < nq; ++qi) {
    const int row = all_q ? qi : q_rows[qi];
    std::vector<double> s;
    for (int a = 0; a < heads; ++a) {
      int t_lo, t_hi;
      scores(row, a, s, t_lo, t_hi);
      const double ls = softmax(s);
      if (lse) lse[(size_t)qi * heads + a] = ls;
      std::vector<double> orow(dh, 0.0);
      for (int u = t_lo; u <= t_hi; ++u)
        for (int c = 0; c < dh; ++c) orow[c] += s[u - t_lo] * Vv(u, a, c);
      if (o)
        for (int c = 0; c < dh; ++c) o[(size_t)qi * W + a * dh + c] = orow[c];
      if (dout && dq) {
        double D = 0.0;
        for (int c = 0; c < dh; ++c) D += G(row, a, c) * orow[c];
        double* dqr = dq + (size_t)qi * W + a * dh;
        for (int c = 0; c < dh; ++c) dqr[c] = 0.0;
        for (int u = t_lo; u <= t_hi; ++u) {
          double dP = 0.0;
          for (int c = 0; c < dh; ++c) dP += G(row, a, c) * Vv(u, a, c);
          const double dS = s[u - t_lo] * (dP - D);
          for (int c = 0; c < dh; ++c) dqr[c] += dS * Kv(u, a, c) * scale;
        }
      }
    }
  }
  if (!dout || n_kv == 0 || (!dk && !dv)) return;
  /* dk, dv: every query of the listed tokens' sequences contributes; its lse and
   * D = <dout, o> are computed once per (grouped row, head) */
  const bool all_kv = kv_tokens == nullptr;
  const int nkv = all_kv ? T : n_kv;
  std::vector<char> need_seq((T + L - 1) / L, 0);
  for (int ti = 0; ti < nkv; ++ti) need_seq[(all_kv ? ti : kv_tokens[ti]) / L] = 1;
  std::vector<double> lse_all((size_t)S * heads, 0.0), D_all((size_t)S * heads, 0.0);
#pragma omp parallel for schedule(dynamic, 4)
  for (int row = 0; row < S; ++row) {
    const int t = sorted_slot[row] / kslots;
    if (!need_seq[t / L]) continue;
    std::vector<double> s;
    for (int a = 0; a < heads; ++a) {
      int t_lo, t_hi;
      scores(row, a, s, t_lo, t_hi);
      lse_all[(size_t)row * heads + a] = softmax(s);
      double D = 0.0;
      for (int c = 0; c < dh; ++c) {
        double oc = 0.0;
        for (int u = t_lo; u <= t_hi; ++u) oc += s[u - t_lo] * Vv(u, a, c);
        D += G(row, a, c) * oc;
      }
      D_all[(size_t)row * heads + a] = D;
    }
  }
#pragma omp parallel for schedule(dynamic, 1)
  for (int ti = 0; ti < nkv; ++ti) {
    const int u = all_kv ? ti : kv_tokens[ti];
    const int seq_end = std::min(T, (u / L + 1) * L);
    for (int a = 0; a < heads; ++a) {
      std::vector<double> dkr(dh, 0.0), dvr(dh, 0.0);
      for (int t = u; t < seq_end; ++t)
        for (int j = 0; j < kslots; ++j) {
          const int row = inv[(size_t)t * kslots + j];
          double sc = 0.0, dP = 0.0;
          for (int c = 0; c < dh; ++c) {
            sc += Q(row, a, c) * Kv(u, a, c);
            dP += G(row, a, c) * Vv(u, a, c);
          }
          const double P = std::exp(sc * scale - lse_all[(size_t)row * heads + a]);
          const double dS = P * (dP - D_all[(size_t)row * heads + a]);
          for (int c = 0; c < dh; ++c) {
            dkr[c] += dS * Q(row, a, c) * scale;
            dvr[c] += P * G(row, a, c);
          }
        }
      for (int c = 0; c < dh; ++c) {
        if (dk) dk[(size_t)ti * W + a * dh + c] = dkr[c];
        if (dv) dv[(size_t)ti * W + a * dh + c] = dvr[c];
      }
    }
  }
}

/* e4m3 rounding of n values (for pins) */
void oracle_e4m3_round(const double* v, int n, double* out) {
  for (int i = 0; i < n; ++i) out[i] = e4m3_round(v[i]);
}
void oracle_e4m3_decode(const uint8_t* b, int n, double* out) {
  for (int i = 0; i < n; ++i) out[i] = e4m3_value(b[i]);
}
/* Weights W [E, K, N] (stored dtype dt) -> codes [E, N, K] (K-major) and one scale per
 * (expert, output column) [E, N], over that column's K values. */
void oracle_quantize_weights_fp8(const void* w, int dt, int E, int K, int N, uint8_t* codes,
                                 float* scales) {
#pragma omp parallel for schedule(static)
  for (int en = 0; en < E * N; ++en) {
    const int e = en / N, n = en % N;
    std::vector<double> col(K);
    for (int k = 0; k < K; ++k) col[k] = load_any(w, dt, ((size_t)e * K + k) * N + n);
    quantize_row_fp8(col.data(), K, codes + (size_t)en * K, scales + en);
  }
}
/* Rows of a matrix [rows, cols] (stored dtype dt) -> codes [rows, cols], scales [rows]. */
void oracle_quantize_rows_fp8(const void* x, int dt, int rows, int cols, uint8_t* codes,
                              float* scales) {
#pragma omp parallel for schedule(static)
  for (int r = 0; r < rows; ++r) {
    std::vector<double> v(cols);
    for (int c = 0; c < cols; ++c) v[c] = load_any(x, dt, (size_t)r * cols + c);
    quantize_row_fp8(v.data(), cols, codes + (size_t)r * cols, scales + r);
  }
}
/* FP8 forward of the listed tokens with quantised weights (codes K-major [E, N, K],
 * scales [E, N]) from oracle_quantize_weights_fp8:
 *   x8, sx = row quantisation of x[t];  H = (x8 . w1_8[e]) sx s1[e]  (fp64)
 *   A = act(H), stored in bf16;  a8, sa = row quantisation of A (its f values)
 *   o = (a8 . w2_8[e]) sa s2[e];  y_t = sum_j g[t,j] o_{t*k+j}.
 * y [n_tok, d]; a (nullable) [n_tok*k, f] = the bf16-rounded A. */
void oracle_mlp_fwd_fp8(const void* x, int dtx, const uint8_t* w1q, const float* s1,
                        const uint8_t* w2q, const float* s2, int d, int f, int E, int k, int act,
                        const int32_t* idx, const double* gates, const int32_t* tokens, int n_tok,
                        double* y, double* a_out) {
  const int mf = (act == ACT_SWIGLU) ? 2 * f : f;
#pragma omp parallel for schedule(dynamic, 1)
  for (int q = 0; q < n_tok; ++q) {
    const int t = tokens[q];
    std::vector<double> xv(d), h(mf), a(f);
    std::vector<uint8_t> x8(d), a8(f);
    float sx, sa;
    for (int i = 0; i < d; ++i) xv[i] = load_any(x, dtx, (size_t)t * d + i);
    quantize_row_fp8(xv.data(), d, x8.data(), &sx);
    double* yq = y + (size_t)q * d;
    for (int n = 0; n < d; ++n) yq[n] = 0.0;
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      for (int n = 0; n < mf; ++n) {
        const uint8_t* wr = w1q + ((size_t)e * mf + n) * d;
        double acc = 0.0;
        for (int i = 0; i < d; ++i) acc += e4m3_value(x8[i]) * e4m3_value(wr[i]);
        h[n] = acc * (double)sx * (double)s1[(size_t)e * mf + n];
      }
      for (int c = 0; c < f; ++c) {
        const double av = (act == ACT_SWIGLU) ? silu(h[c]) * h[f + c] : gelu_tanh(h[c]);
        a[c] = (double)to_float(bf16_round(av));
      }
      if (a_out) std::memcpy(a_out + ((size_t)q * k + j) * f, a.data(), sizeof(double) * f);
      quantize_row_fp8(a.data(), f, a8.data(), &sa);
      const double g = gates[(size_t)t * k + j];
      for (int n = 0; n < d; ++n) {
        const uint8_t* wr = w2q + ((size_t)e * d + n) * f;
        double acc = 0.0;
        for (int c = 0; c < f; ++c) acc += e4m3_value(a8[c]) * e4m3_value(wr[c]);
        yq[n] += g * acc * (double)sa * (double)s2[(size_t)e * d + n];
      }
    }
  }
  (void)E;
}

/* R6 forward.  gates: fp64 per slot (nullable).  out_rows (nullable): the rows
 * of y to compute (grouped row, slot or token, by mode); y: [n_out, N].      */
void oracle_pl_fwd(const void* x, int dtx, const void* w, int dtw, int K, int N, int E,
                   const int32_t* sorted_slot, const int32_t* offsets, int num_slots, int fan_out,
                   int grouped_in, int grouped_out, const double* gates, int combine_k,
                   const int32_t* out_rows, int n_out, double* y) {
  SMOE_ORACLE_DISPATCH2(dtx, dtw,
      pl_fwd_impl((const TX*)x, (const TW*)w, K, N, E, sorted_slot, offsets, num_slots, fan_out,
                  grouped_in, grouped_out, gates, combine_k, out_rows, n_out, y));
}

/* R6 backward; dy is in the dtype code dtd (0 fp32, 1 bf16, 2 fp64).  Each of
 * dx / dw / dgates is skipped when its output pointer is null; each row, column
 * or slot list may be null (= all).  dx: [n_dx, K]; dw: [E, K, n_dw];
 * dgates: [n_dg].                                                             */
void oracle_pl_bwd(const void* dy, int dtd, const void* x, int dtx, const void* w, int dtw,
                   int x_rows, int K, int N, int E, const int32_t* sorted_slot,
                   const int32_t* offsets, int num_slots, int fan_out, int grouped_in,
                   int grouped_out, const double* gates, int combine_k, const int32_t* dx_rows,
                   int n_dx, double* dx, const int32_t* dw_cols, int n_dw, double* dw,
                   const int32_t* dg_slots, int n_dg, double* dgates) {
#define SMOE_PL_BWD_CALL(TD_)                                                                 \
  SMOE_ORACLE_DISPATCH2(dtx, dtw,                                                             \
      (pl_bwd_impl<TX, TW, TD_>((const TD_*)dy, (const TX*)x, (const TW*)w, x_rows, K, N, E,  \
                                sorted_slot, offsets, num_slots, fan_out, grouped_in,         \
                                grouped_out, gates, combine_k, dx_rows, n_dx, dx, dw_cols,    \
                                n_dw, dw, dg_slots, n_dg, dgates)))
  if (dtd == 0) { SMOE_PL_BWD_CALL(float); }
  else if (dtd == 1) { SMOE_PL_BWD_CALL(bf16s); }
  else { SMOE_PL_BWD_CALL(double); }
#undef SMOE_PL_BWD_CALL
}

}  // extern "C"
