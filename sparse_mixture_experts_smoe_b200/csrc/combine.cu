// combine.cu -- bandwidth-bound helpers around the grouped GEMMs:
//   * the deterministic k-way combine of a slot-ordered fp32 buffer into token rows
//     (optionally adding the router's term dl W_r^T of the backward),
//   * the fixed-order reduction of per-column-tile gate-gradient partials,
//   * a gated gather of rows into grouped order.
//
// The k slots of a token are owned by k different experts, so their products
// come from different CTAs; summing them with atomics would make the result
// depend on scheduling.  Instead the GEMM epilogue stores each slot's row, already
// multiplied by its gate, in a buffer of the layer's dtype (the slot outputs are
// materialised in the compute type before the gate-weighted sum, as the library
// does it), in grouped order (row i of slot p = sorted_slot[i], so that whole warps
// of rows leave as TMA boxes); this pass sums the k rows of each token in fp32 in
// ascending j, finding slot p's row through the inverse permutation inv[p] = i
// (group-to-scatter with combine, library page of arXiv 2403.08245, review 2
// summary).
#include "common.cuh"

namespace smoe {
namespace {

// Each thread owns kCombV float4 columns of one token, u + v*U for v < kCombV
// (U threads per token, so every v is a coalesced sweep of the row).  The slot
// rows sit at grouped positions, so their indices come first; the thread then has
// kCombV independent 16-byte loads in flight per slot instead of one load behind
// a dependent index load.  The router term reads the transposed router weight
// w_rt [E, N] so each selected expert contributes contiguous loads.
constexpr int kCombV = 4;

// four consecutive elements as one 8- or 16-byte access
__device__ __forceinline__ float4 load4(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ float4 load4(const bf16* p) {
  const uint2 r = __ldg(reinterpret_cast<const uint2*>(p));
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void store4(bf16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  uint2 r;
  r.x = *reinterpret_cast<uint32_t*>(&a);
  r.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = r;
}

template <typename T>
__global__ void __launch_bounds__(256)
combine_kernel(const T* __restrict__ ws, const int32_t* __restrict__ inv, int T_, int ck,
               int N, T* __restrict__ out, const float* __restrict__ dl,
               const int32_t* __restrict__ idx, const T* __restrict__ w_rt, int E) {
  const int n4 = N / 4;
  const int U = (n4 + kCombV - 1) / kCombV;
  const size_t q = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= (size_t)T_ * U) return;
  const int t = (int)(q / U);
  const int u = (int)(q % U);
  const int S = T_ * ck;
  float4 acc[kCombV];
#pragma unroll
  for (int v = 0; v < kCombV; ++v) acc[v] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
  for (int j = 0; j < ck; ++j) {
    const int p = t * ck + j;
    const int row = inv ? __ldg(inv + p) : p;
    if (row < 0 || row >= S) continue;  // not a permutation: a data error flagged upstream
    const T* src = ws + (size_t)row * N;
    float4 x[kCombV];
#pragma unroll
    for (int v = 0; v < kCombV; ++v) {
      const int c4 = u + v * U;
      x[v] = c4 < n4 ? load4(src + 4 * c4) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int v = 0; v < kCombV; ++v) {
      acc[v].x += x[v].x; acc[v].y += x[v].y; acc[v].z += x[v].z; acc[v].w += x[v].w;
    }
  }
  if (dl != nullptr) {
    for (int j = 0; j < ck; ++j) {
      const int e = idx[(size_t)t * ck + j];
      if (e < 0 || e >= E) continue;
      const float g = dl[(size_t)t * ck + j];
#pragma unroll
      for (int v = 0; v < kCombV; ++v) {
        const int c4 = u + v * U;
        if (c4 >= n4) continue;
        const float4 w = load4(w_rt + (size_t)e * N + 4 * c4);
        acc[v].x = fmaf(g, w.x, acc[v].x);
        acc[v].y = fmaf(g, w.y, acc[v].y);
        acc[v].z = fmaf(g, w.z, acc[v].z);
        acc[v].w = fmaf(g, w.w, acc[v].w);
      }
    }
  }
#pragma unroll
  for (int v = 0; v < kCombV; ++v) {
    const int c4 = u + v * U;
    if (c4 >= n4) continue;
    store4(out + (size_t)t * N + 4 * c4, acc[v]);
  }
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
                                 float* __restrict__ dg, int32_t* __restrict__ inv) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= num_rows) return;
  float s = 0.0f;
  for (int c = 0; c < n_tiles; ++c) s += partial[(size_t)i * ld + c];
  const int p = sorted_slot[i];
  if (p < 0 || p >= num_rows) return;  // reported by the GEMM that read it
  dg[p] = s;
  if (inv) inv[p] = i;
}

__global__ void invert_kernel(const int32_t* __restrict__ sorted_slot, int num_rows,
                              int32_t* __restrict__ inv) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= num_rows) return;
  const int p = sorted_slot[i];
  if (p >= 0 && p < num_rows) inv[p] = i;
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

cudaError_t launch_combine(const void* ws, const int32_t* inv, int T_, int ck, int N, void* out,
                           smoe_dtype dt, const float* dl, const int32_t* idx, const void* w_rt,
                           int E, cudaStream_t s) {
  const size_t n = (size_t)T_ * cdiv(N / 4, kCombV);
  const unsigned blocks = (unsigned)((n + 255) / 256);
  if (dt == SMOE_BF16)
    combine_kernel<bf16><<<blocks, 256, 0, s>>>((const bf16*)ws, inv, T_, ck, N, (bf16*)out, dl,
                                                idx, (const bf16*)w_rt, E);
  else
    combine_kernel<float><<<blocks, 256, 0, s>>>((const float*)ws, inv, T_, ck, N, (float*)out, dl,
                                                 idx, (const float*)w_rt, E);
  return cudaGetLastError();
}

cudaError_t launch_invert(const int32_t* sorted_slot, int num_rows, int32_t* inv, cudaStream_t s) {
  invert_kernel<<<cdiv(num_rows, 256), 256, 0, s>>>(sorted_slot, num_rows, inv);
  return cudaGetLastError();
}

cudaError_t launch_dg_reduce(const float* partial, int ld, int n_tiles, const int32_t* sorted_slot,
                             int num_rows, float* dg, cudaStream_t s, int32_t* inv) {
  dg_reduce_kernel<<<cdiv(num_rows, 256), 256, 0, s>>>(partial, ld, n_tiles, sorted_slot,
                                                       num_rows, dg, inv);
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
