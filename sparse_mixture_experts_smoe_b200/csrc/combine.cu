// combine.cu -- bandwidth-bound helpers around the grouped GEMMs:
//   * the deterministic k-way combine of a grouped-order buffer of gated slot rows
//     (in the layer's dtype) into token rows, summed in fp32 (optionally adding the
//     router's term dl W_r^T of the backward),
//   * the fixed-order reduction of per-column-tile gate-gradient partials,
//   * the fixed-order reduction of split-K partials (decode-sized batches).
//
// The k slots of a token are owned by k different experts, so their products
// come from different CTAs; summing them with atomics would make the result
// depend on scheduling.  Instead the GEMM epilogue stores each slot's row, already
// multiplied by its gate, in a buffer of the layer's dtype (this library's choice:
// the pages do not say in what precision per-slot outputs are held before the
// gate-weighted sum), in grouped order (row i of slot p = sorted_slot[i], so that whole warps
// of rows leave as TMA boxes); this pass sums the k rows of each token in fp32 in
// ascending j, finding slot p's row through the inverse permutation inv[p] = i
// (group-to-scatter with combine, library page of arXiv 2403.08245, review 2
// summary).
#include "common.cuh"

namespace smoe {
namespace {

// Each thread owns kCombV 16-byte vectors of one token's row (VE = 8 bf16 or 4 fp32
// elements each), vector u + v*U for v < kCombV (U threads per token, so every v is
// a coalesced sweep of the row).  The slot rows sit at grouped positions, so their
// index comes first; the thread then has kCombV independent 16-byte loads in flight
// per slot instead of one load behind a dependent index load.  The router term
// reads the transposed router weight w_rt [E, N] so each selected expert
// contributes contiguous loads.
constexpr int kCombV = 4;

template <typename T>
struct Vec16 {
  static constexpr int VE = 16 / (int)sizeof(T);
  float f[VE];
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int i = 0; i < VE; ++i) f[i] = 0.f;
  }
  __device__ __forceinline__ void load(const T* p) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    if constexpr (sizeof(T) == 2) {
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 a = __bfloat1622float2(h[i]);
        f[2 * i] = a.x;
        f[2 * i + 1] = a.y;
      }
    } else {
      f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
      f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
    }
  }
  __device__ __forceinline__ void store(T* p) const {
    uint4 u;
    if constexpr (sizeof(T) == 2) {
      uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t*>(&h);
      }
    } else {
      u = make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                     __float_as_uint(f[3]));
    }
    *reinterpret_cast<uint4*>(p) = u;
  }
};

template <typename T>
__global__ void __launch_bounds__(256)
combine_kernel(const T* __restrict__ ws, const int32_t* __restrict__ inv, int T_, int ck,
               int N, T* __restrict__ out, const float* __restrict__ dl,
               const int32_t* __restrict__ idx, const T* __restrict__ w_rt, int E) {
  using V = Vec16<T>;
  constexpr int VE = V::VE;
  const int nv = N / VE;  // N % 8 == 0
  const int U = (nv + kCombV - 1) / kCombV;
  const size_t q = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= (size_t)T_ * U) return;
  const int t = (int)(q / U);
  const int u = (int)(q % U);
  const int S = T_ * ck;
  V acc[kCombV];
#pragma unroll
  for (int v = 0; v < kCombV; ++v) acc[v].zero();
#pragma unroll 2
  for (int j = 0; j < ck; ++j) {
    const int p = t * ck + j;
    const int row = inv ? __ldg(inv + p) : p;
    if (row < 0 || row >= S) continue;  // not a permutation: a data error flagged upstream
    const T* src = ws + (size_t)row * N;
    V x[kCombV];
#pragma unroll
    for (int v = 0; v < kCombV; ++v) {
      const int cv = u + v * U;
      if (cv < nv) x[v].load(src + VE * cv);
      else x[v].zero();
    }
#pragma unroll
    for (int v = 0; v < kCombV; ++v)
#pragma unroll
      for (int i = 0; i < VE; ++i) acc[v].f[i] += x[v].f[i];
  }
  if (dl != nullptr) {
    for (int j = 0; j < ck; ++j) {
      const int e = idx[(size_t)t * ck + j];
      if (e < 0 || e >= E) continue;
      const float g = dl[(size_t)t * ck + j];
#pragma unroll
      for (int v = 0; v < kCombV; ++v) {
        const int cv = u + v * U;
        if (cv >= nv) continue;
        V w;
        w.load(w_rt + (size_t)e * N + VE * cv);
#pragma unroll
        for (int i = 0; i < VE; ++i) acc[v].f[i] = fmaf(g, w.f[i], acc[v].f[i]);
      }
    }
  }
#pragma unroll
  for (int v = 0; v < kCombV; ++v) {
    const int cv = u + v * U;
    if (cv < nv) acc[v].store(out + (size_t)t * N + VE * cv);
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

// out[i, c..c+3] = g * sum_s partial[s, i, c..c+3], one thread per 4 columns of a row
__global__ void splitk_reduce_kernel(const float* __restrict__ partial, int ks, int num_rows,
                                     int n_out, const int32_t* __restrict__ sorted_slot,
                                     const float* __restrict__ gates, bf16* __restrict__ out,
                                     int ldo) {
  const int n4 = n_out / 4;
  const size_t q = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= (size_t)num_rows * n4) return;
  const int i = (int)(q / n4), c = (int)(q % n4) * 4;
  float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int sp = 0; sp < ks; ++sp) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(partial + ((size_t)sp * num_rows + i) * n_out + c));
    a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
  }
  const int p = sorted_slot[i];
  const float g = (gates != nullptr && p >= 0 && p < num_rows) ? gates[p] : 1.0f;
  __nv_bfloat162 lo = __floats2bfloat162_rn(g * a.x, g * a.y), hi = __floats2bfloat162_rn(g * a.z, g * a.w);
  uint2 r;
  r.x = *reinterpret_cast<uint32_t*>(&lo);
  r.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(out + (size_t)i * ldo + c) = r;
}

}  // namespace

cudaError_t launch_splitk_reduce(const float* partial, int ksplit, int num_rows, int n_out,
                                 const int32_t* sorted_slot, const float* gates, void* out,
                                 int ldo, cudaStream_t s) {
  const size_t n = (size_t)num_rows * (n_out / 4);
  splitk_reduce_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(partial, ksplit, num_rows, n_out,
                                                                    sorted_slot, gates, (bf16*)out, ldo);
  return cudaGetLastError();
}

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
  const int ve = dt == SMOE_BF16 ? 8 : 4;
  const size_t n = (size_t)T_ * cdiv(N / ve, kCombV);
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

}  // namespace smoe
