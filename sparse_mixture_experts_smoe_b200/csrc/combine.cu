// combine.cu -- bandwidth-bound helpers around the grouped GEMMs:
//   * the deterministic k-way combine of a slot-ordered fp32 buffer into token rows
//     (optionally adding the router's term dl W_r^T of the backward),
//   * the fixed-order reduction of per-column-tile gate-gradient partials,
//   * a gated gather of rows into grouped order.
//
// The k slots of a token are owned by k different experts, so their products
// come from different CTAs; summing them with atomics would make the result
// depend on scheduling.  Instead the GEMM epilogue stores each slot's row at
// row p = t*k + j of an fp32 buffer, and this pass sums the k rows of each token
// in ascending j (group-to-scatter with combine, library page of arXiv 2403.08245,
// review 2 summary).
#include "common.cuh"

namespace smoe {
namespace {

// One thread per 4 consecutive columns of one token.  The router term reads the
// transposed router weight w_rt [E, N] so each selected expert contributes one
// contiguous 4-element load.
template <typename TO, typename TW>
__global__ void combine_kernel(const float* __restrict__ ws, int T_, int ck, int N,
                               TO* __restrict__ out, const float* __restrict__ dl,
                               const int32_t* __restrict__ idx, const TW* __restrict__ w_rt,
                               int E) {
  const int n4 = N / 4;
  const size_t q = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= (size_t)T_ * n4) return;
  const int t = (int)(q / n4);
  const int c = (int)(q % n4) * 4;
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < ck; ++j) {
    const float4 v = *reinterpret_cast<const float4*>(ws + ((size_t)t * ck + j) * N + c);
    s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
  }
  if (dl != nullptr) {
    for (int j = 0; j < ck; ++j) {
      const int e = idx[(size_t)t * ck + j];
      if (e < 0 || e >= E) continue;
      const float g = dl[(size_t)t * ck + j];
      const TW* w = w_rt + (size_t)e * N + c;
      s.x = fmaf(g, to_f(w[0]), s.x);
      s.y = fmaf(g, to_f(w[1]), s.y);
      s.z = fmaf(g, to_f(w[2]), s.z);
      s.w = fmaf(g, to_f(w[3]), s.w);
    }
  }
  TO* o = out + (size_t)t * N + c;
  o[0] = from_f<TO>(s.x);
  o[1] = from_f<TO>(s.y);
  o[2] = from_f<TO>(s.z);
  o[3] = from_f<TO>(s.w);
}

// w_rt[e][i] = w_r[i][e]
template <typename T>
__global__ void transpose_kernel(const T* __restrict__ w_r, int d, int E, T* __restrict__ w_rt) {
  const int q = blockIdx.x * blockDim.x + threadIdx.x;  // q = e * d + i
  if (q >= d * E) return;
  const int e = q / d, i = q % d;
  w_rt[q] = w_r[(size_t)i * E + e];
}

__global__ void dg_reduce_kernel(const float* __restrict__ partial, int ld, int n_tiles,
                                 const int32_t* __restrict__ sorted_slot, int num_rows,
                                 float* __restrict__ dg) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= num_rows) return;
  float s = 0.0f;
  for (int c = 0; c < n_tiles; ++c) s += partial[(size_t)i * ld + c];
  dg[sorted_slot[i]] = s;
}

template <typename T>
__global__ void gather_scale_kernel(const T* __restrict__ src, int ld_src, int mode, int fan_out,
                                    const int32_t* __restrict__ sorted_slot,
                                    const float* __restrict__ gates, int num_rows, int cols,
                                    T* __restrict__ out) {
  const size_t q = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= (size_t)num_rows * cols) return;
  const int i = (int)(q / cols), c = (int)(q % cols);
  const int p = sorted_slot[i];
  const int r = mode == ROWS_GROUPED ? i : p / fan_out;
  const float g = gates ? gates[p] : 1.0f;
  out[q] = from_f<T>(g * to_f(src[(size_t)r * ld_src + c]));
}

}  // namespace

cudaError_t launch_transpose_wr(const void* w_r, int d, int E, smoe_dtype dt, void* w_rt,
                                cudaStream_t s) {
  const unsigned blocks = (unsigned)((d * E + 255) / 256);
  if (dt == SMOE_BF16)
    transpose_kernel<bf16><<<blocks, 256, 0, s>>>((const bf16*)w_r, d, E, (bf16*)w_rt);
  else
    transpose_kernel<float><<<blocks, 256, 0, s>>>((const float*)w_r, d, E, (float*)w_rt);
  return cudaGetLastError();
}

cudaError_t launch_combine(const float* ws, int T_, int ck, int N, void* out, smoe_dtype out_dt,
                           const float* dl, const int32_t* idx, const void* w_rt, int E,
                           cudaStream_t s) {
  const size_t n = (size_t)T_ * (N / 4);
  const unsigned blocks = (unsigned)((n + 255) / 256);
  if (out_dt == SMOE_BF16)
    combine_kernel<bf16, bf16><<<blocks, 256, 0, s>>>(ws, T_, ck, N, (bf16*)out, dl, idx,
                                                      (const bf16*)w_rt, E);
  else
    combine_kernel<float, float><<<blocks, 256, 0, s>>>(ws, T_, ck, N, (float*)out, dl, idx,
                                                        (const float*)w_rt, E);
  return cudaGetLastError();
}

cudaError_t launch_dg_reduce(const float* partial, int ld, int n_tiles, const int32_t* sorted_slot,
                             int num_rows, float* dg, cudaStream_t s) {
  dg_reduce_kernel<<<cdiv(num_rows, 256), 256, 0, s>>>(partial, ld, n_tiles, sorted_slot,
                                                       num_rows, dg);
  return cudaGetLastError();
}

cudaError_t launch_gather_scale(const void* src, int ld_src, int mode, int fan_out,
                                const int32_t* sorted_slot, const float* gates, int num_rows,
                                int cols, void* out, smoe_dtype dt, cudaStream_t s) {
  const size_t n = (size_t)num_rows * cols;
  const unsigned blocks = (unsigned)((n + 255) / 256);
  if (dt == SMOE_BF16)
    gather_scale_kernel<bf16><<<blocks, 256, 0, s>>>((const bf16*)src, ld_src, mode, fan_out,
                                                     sorted_slot, gates, num_rows, cols, (bf16*)out);
  else
    gather_scale_kernel<float><<<blocks, 256, 0, s>>>((const float*)src, ld_src, mode, fan_out,
                                                      sorted_slot, gates, num_rows, cols,
                                                      (float*)out);
  return cudaGetLastError();
}

}  // namespace smoe
