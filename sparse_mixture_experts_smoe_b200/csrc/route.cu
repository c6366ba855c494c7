// route.cu -- router of the SMoE layer: logits, top-k selection, renormalised
// gates (smoe_route), and the router backward (smoe_route_bwd).
//
// The pages define the layer as top-k routing with a gate-weighted sum of expert
// MLPs (arXiv abstract; tradepoint.io article, method paragraphs); the router
// itself is softmax, top-k, renormalise.  The top-k decision is an integer result
// taken from fp32 logits, so the logits are accumulated in one documented order
// (see smoe_route in smoe.h) that a CPU restatement can reproduce bit for bit:
// lane L of a warp owns every input feature i with i % 32 == L, accumulates its
// products in ascending i with fmaf, and the 32 lane sums meet in an xor
// butterfly (16, 8, 4, 2, 1) before the bias is added.
//
// Work split: a warp handles TM tokens; a block of 8 warps stages CH rows of W_r
// in shared memory as fp32 with a row stride = 4 (mod 32) words, so the eight
// lanes of a 128-bit shared load phase read eight different bank groups, and the
// block's CH-feature slice of x with 16-byte coalesced loads (lane L then reads
// its features L, L+32, ... from shared memory; the accumulation order above is
// unchanged).
#include "common.cuh"

namespace smoe {
namespace {

constexpr int kRouteWarps = 8;

__host__ __device__ constexpr int route_row_stride(int emax) {
  // smallest stride >= emax with stride % 32 == 4 (floats)
  return emax + ((4 - emax % 32) + 32) % 32;
}

// FULL: E == EMAX (the staged W_r rows need no padding and the index arithmetic
// of the staging divides by a constant).
template <typename T, int EMAX, int TM, int CH, bool FULL>
__global__ void __launch_bounds__(kRouteWarps * 32)
route_kernel(const T* __restrict__ x, const T* __restrict__ w_r, const float* __restrict__ b_r,
             int T_, int d, int E, int k, int32_t* __restrict__ idx, float* __restrict__ gates,
             unsigned* err) {
  constexpr int STRIDE = route_row_stride(EMAX);
  constexpr int BT = kRouteWarps * TM;  // tokens per block
  extern __shared__ float4 smem_f4[];
  float* ws = reinterpret_cast<float*>(smem_f4);  // [CH][STRIDE]
  float* xs = ws + CH * STRIDE;                   // [BT][CH]

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int tb = blockIdx.x * BT;
  const int t0 = tb + warp * TM;

  float acc[TM][EMAX];
#pragma unroll
  for (int m = 0; m < TM; ++m)
#pragma unroll
    for (int e = 0; e < EMAX; ++e) acc[m][e] = 0.0f;

  const int ecols = FULL ? EMAX : E;
  // padding columns [E, EMAX) of the staged W_r stay zero for every chunk
  if (!FULL && E < EMAX)
    for (int q = threadIdx.x; q < CH * (EMAX - E); q += blockDim.x)
      ws[(q / (EMAX - E)) * STRIDE + E + q % (EMAX - E)] = 0.0f;
  constexpr int VEC = 16 / (int)sizeof(T);  // elements per 16-byte load
  for (int i0 = 0; i0 < d; i0 += CH) {
    __syncthreads();
    // stage W_r[i0 : i0+CH, 0:E] as fp32: the rows are one contiguous span of
    // (rows * E) elements, a multiple of VEC because d % 8 == 0, read with 16-byte
    // loads several in flight per thread
    {
      const int rows = min(CH, d - i0);
      const int nvec = rows * ecols / VEC;
      const uint4* src = reinterpret_cast<const uint4*>(w_r + (size_t)i0 * E);
#pragma unroll 4
      for (int q = threadIdx.x; q < nvec; q += blockDim.x) {
        const uint4 u = __ldg(src + q);
        const T* vals = reinterpret_cast<const T*>(&u);
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
          const int flat = q * VEC + v;
          ws[(flat / ecols) * STRIDE + flat % ecols] = to_f(vals[v]);
        }
      }
    }
    // stage x[tb : tb+BT, i0 : i0+CH] as fp32 with 8-element (16-byte bf16) loads
    for (int q = threadIdx.x; q < BT * (CH / 8); q += blockDim.x) {
      const int m = q / (CH / 8), c8 = (q % (CH / 8)) * 8;
      const int t = tb + m, i = i0 + c8;
      float v[8];
      if (t < T_ && i < d) {  // d % 8 == 0, so the 8 features are all in range
        const T* src = x + (size_t)t * d + i;
        if (sizeof(T) == 2) {
          const uint4 u = *reinterpret_cast<const uint4*>(src);
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
          for (int h2 = 0; h2 < 4; ++h2) {
            const float2 f = __bfloat1622float2(h[h2]);
            v[2 * h2] = f.x;
            v[2 * h2 + 1] = f.y;
          }
        } else {
          const float4 a = *reinterpret_cast<const float4*>(src);
          const float4 b = *reinterpret_cast<const float4*>(src + 4);
          v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
          v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        }
      } else {
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = 0.0f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) xs[m * CH + c8 + u] = v[u];
    }
    __syncthreads();
#pragma unroll 2
    for (int r = lane; r < CH; r += 32) {
      if (i0 + r >= d) break;
      float xv[TM];
#pragma unroll
      for (int m = 0; m < TM; ++m) xv[m] = xs[(warp * TM + m) * CH + r];
      const float4* wrow = reinterpret_cast<const float4*>(ws + r * STRIDE);
#pragma unroll
      for (int e4 = 0; e4 < EMAX / 4; ++e4) {
        const float4 w4 = wrow[e4];
#pragma unroll
        for (int m = 0; m < TM; ++m) {
          acc[m][4 * e4 + 0] = fmaf(xv[m], w4.x, acc[m][4 * e4 + 0]);
          acc[m][4 * e4 + 1] = fmaf(xv[m], w4.y, acc[m][4 * e4 + 1]);
          acc[m][4 * e4 + 2] = fmaf(xv[m], w4.z, acc[m][4 * e4 + 2]);
          acc[m][4 * e4 + 3] = fmaf(xv[m], w4.w, acc[m][4 * e4 + 3]);
        }
      }
    }
  }
  // xor butterfly over the 32 lanes (every lane ends with the same sums)
#pragma unroll
  for (int m = 0; m < TM; ++m)
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
      float v = acc[m][e];
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) v = v + __shfl_xor_sync(0xffffffffu, v, off);
      acc[m][e] = v;
    }

  // Top-k per token, warp-parallel: lane L holds the logits of experts
  // e = L + 32 j (j < NC).  Each round reproduces the sequential scan "start at the
  // first free expert, replace on a strictly greater logit": if the first free
  // expert's logit is NaN it is taken, else the largest free non-NaN logit, the
  // lower expert id on ties.
  constexpr int NC = EMAX >= 32 ? EMAX / 32 : 1;
  constexpr int kNone = 0x7fffffff;
#pragma unroll
  for (int m = 0; m < TM; ++m) {
    const int t = t0 + m;
    if (t >= T_) break;
    float lv[NC];
    unsigned fr = 0u;  // bit j: expert lane + 32 j is free
#pragma unroll
    for (int j = 0; j < NC; ++j) {
      const int e = lane + 32 * j;
      float a = 0.0f;
#pragma unroll
      for (int ee = 0; ee < EMAX; ++ee)
        if (ee == e) a = acc[m][ee];
      lv[j] = (e < E && b_r != nullptr) ? a + b_r[e] : a;
      if (e < E && e < EMAX) fr |= 1u << j;
    }
    float sel[16];
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) {
      if (jj >= k) break;
      // first free expert and its logit
      int ff = kNone;
#pragma unroll
      for (int j = NC - 1; j >= 0; --j)
        if ((fr >> j) & 1u) ff = lane + 32 * j;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) ff = min(ff, __shfl_xor_sync(0xffffffffu, ff, off));
      float vff = 0.0f;
#pragma unroll
      for (int j = 0; j < NC; ++j)
        if (ff == lane + 32 * j) vff = lv[j];
      vff = __shfl_sync(0xffffffffu, vff, ff & 31);
      int win;
      float wv;
      if (vff != vff) {  // NaN at the first free expert: the scan keeps it
        win = ff;
        wv = vff;
      } else {
        float bv = 0.0f;
        int bi = kNone;
#pragma unroll
        for (int j = 0; j < NC; ++j) {
          const float v = lv[j];
          if (((fr >> j) & 1u) && v == v && (bi == kNone || v > bv)) {
            bv = v;
            bi = lane + 32 * j;
          }
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
          const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
          if (oi != kNone && (bi == kNone || ov > bv || (ov == bv && oi < bi))) {
            bv = ov;
            bi = oi;
          }
        }
        win = bi;  // a non-NaN free logit exists: the first free one is one
        wv = bv;
      }
#pragma unroll
      for (int j = 0; j < NC; ++j)
        if (win == lane + 32 * j) fr &= ~(1u << j);
      sel[jj] = wv;
      if (lane == 0) idx[(size_t)t * k + jj] = win;
    }
    // gates: softmax over the selected logits (sel[0] is the maximum)
    float z = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (j >= k) break;
      z += expf(sel[j] - sel[0]);
    }
    if (lane == 0) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (j >= k) break;
        gates[(size_t)t * k + j] = expf(sel[j] - sel[0]) / z;
      }
    }
  }
}

template <typename T, int EMAX, int TM>
cudaError_t launch_route_t(const void* x, const void* w_r, const float* b_r, int T_, int d, int E,
                           int k, int32_t* idx, float* gates, unsigned* err, cudaStream_t s) {
  constexpr int CH = EMAX <= 64 ? 256 : 128;
  const size_t smem = ((size_t)CH * route_row_stride(EMAX) + (size_t)kRouteWarps * TM * CH) * sizeof(float);
  auto kern = E == EMAX ? route_kernel<T, EMAX, TM, CH, true> : route_kernel<T, EMAX, TM, CH, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int blocks = cdiv(T_, kRouteWarps * TM);
  kern<<<blocks, kRouteWarps * 32, smem, s>>>((const T*)x, (const T*)w_r, b_r, T_, d, E, k, idx,
                                              gates, err);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_route_dt(const void* x, const void* w_r, const float* b_r, int T_, int d, int E,
                            int k, int32_t* idx, float* gates, unsigned* err, cudaStream_t s) {
  if (E <= 8) return launch_route_t<T, 8, 4>(x, w_r, b_r, T_, d, E, k, idx, gates, err, s);
  if (E <= 16) return launch_route_t<T, 16, 4>(x, w_r, b_r, T_, d, E, k, idx, gates, err, s);
  if (E <= 32) return launch_route_t<T, 32, 4>(x, w_r, b_r, T_, d, E, k, idx, gates, err, s);
  if (E <= 64) return launch_route_t<T, 64, 2>(x, w_r, b_r, T_, d, E, k, idx, gates, err, s);
  return launch_route_t<T, 128, 1>(x, w_r, b_r, T_, d, E, k, idx, gates, err, s);
}

// dl[t,j] = g_j (dg_j - sum_i g_i dg_i)
__global__ void route_dl_kernel(const float* __restrict__ gates, const float* __restrict__ dgates,
                                int T_, int k, float* __restrict__ dl) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T_) return;
  float s = 0.0f;
  for (int j = 0; j < k; ++j) s = fmaf(gates[(size_t)t * k + j], dgates[(size_t)t * k + j], s);
  for (int j = 0; j < k; ++j)
    dl[(size_t)t * k + j] = gates[(size_t)t * k + j] * (dgates[(size_t)t * k + j] - s);
}

// Router weight gradient in two passes with a fixed summation order: tokens are
// split into chunks of `chunk` consecutive tokens; pass 1 sums each chunk in
// ascending token order (per feature column and expert), pass 2 sums the chunk
// partials in ascending chunk order.  The chunk length and the columns per block
// depend only on (T, d, E, k) (route_dw_plan), so results do not depend on the GPU.
//
// Pass 1 per block (chunk c, 8 feature columns per thread): the chunk's routing
// goes to shared memory as one compact list per expert, in token order (one
// thread per expert builds its list); then each thread sums, expert by expert,
// x[t, i:i+8] * dl over the expert's list in registers, reading the x rows with
// 16-byte loads several in flight -- the same additions in the same order as
// accumulating token by token.
//
// partial[c][e][i] = sum_{t in chunk c} x[t,i] dl[t,e];  dbp[c][e] = sum_t dl[t,e]
constexpr int kDwThreads = 128;
constexpr int kDwColsPerThread = 8;

template <typename T>
__device__ __forceinline__ void load8(const T* p, float* v) {
  if (sizeof(T) == 2) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __bfloat1622float2(h[q]);
      v[2 * q] = f.x;
      v[2 * q + 1] = f.y;
    }
  } else {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

template <typename T>
__global__ void __launch_bounds__(kDwThreads)
route_dw_partial_kernel(const T* __restrict__ x, const int32_t* __restrict__ idx,
                        const float* __restrict__ dl, int T_, int d, int E, int k, int chunk,
                        float* __restrict__ partial, float* __restrict__ dbp) {
  extern __shared__ float4 sm4[];
  const int ns = chunk * k;                               // routing slots per chunk
  int* idx_s = reinterpret_cast<int*>(sm4);               // [ns]
  float* dl_s = reinterpret_cast<float*>(idx_s + ns);     // [ns]
  int* lst_t = reinterpret_cast<int*>(dl_s + ns);         // [ns] token of each entry
  float* lst_v = reinterpret_cast<float*>(lst_t + ns);    // [ns] its dl
  int* off = reinterpret_cast<int*>(lst_v + ns);          // [E + 1]
  const int c = blockIdx.x;
  const int i = (blockIdx.y * kDwThreads + threadIdx.x) * kDwColsPerThread;
  const int t0 = c * chunk;
  const int nt = min(T_, t0 + chunk) - t0;
  for (int q = threadIdx.x; q < nt * k; q += kDwThreads) {
    idx_s[q] = idx[(size_t)t0 * k + q];
    dl_s[q] = dl[(size_t)t0 * k + q];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kDwThreads) {  // list lengths (a token's experts are distinct)
    int n = 0;
    for (int q = 0; q < nt * k; ++q) n += idx_s[q] == e;
    off[e + 1] = n;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    off[0] = 0;
    for (int e = 0; e < E; ++e) off[e + 1] += off[e];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kDwThreads) {
    int pos = off[e];
    for (int q = 0; q < nt * k; ++q)
      if (idx_s[q] == e) {
        lst_t[pos] = q / k;
        lst_v[pos] = dl_s[q];
        ++pos;
      }
  }
  __syncthreads();
  if (i < d) {
    const T* xc = x + (size_t)t0 * d + i;
    for (int e = 0; e < E; ++e) {
      float a[kDwColsPerThread];
#pragma unroll
      for (int j = 0; j < kDwColsPerThread; ++j) a[j] = 0.0f;
      int u = off[e];
      const int u1 = off[e + 1];
      for (; u + 4 <= u1; u += 4) {  // four rows in flight, summed in list order
        float v[4][kDwColsPerThread];
#pragma unroll
        for (int r = 0; r < 4; ++r) load8(xc + (size_t)lst_t[u + r] * d, v[r]);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float g = lst_v[u + r];
#pragma unroll
          for (int j = 0; j < kDwColsPerThread; ++j) a[j] = fmaf(v[r][j], g, a[j]);
        }
      }
      for (; u < u1; ++u) {
        float v[kDwColsPerThread];
        load8(xc + (size_t)lst_t[u] * d, v);
        const float g = lst_v[u];
#pragma unroll
        for (int j = 0; j < kDwColsPerThread; ++j) a[j] = fmaf(v[j], g, a[j]);
      }
      float4* dst = reinterpret_cast<float4*>(partial + ((size_t)c * E + e) * d + i);
      dst[0] = make_float4(a[0], a[1], a[2], a[3]);
      dst[1] = make_float4(a[4], a[5], a[6], a[7]);
    }
  }
  if (blockIdx.y == 0)
    for (int e = threadIdx.x; e < E; e += kDwThreads) {  // bias: one expert per thread, token order
      float sb = 0.0f;
      for (int u = off[e]; u < off[e + 1]; ++u) sb += lst_v[u];
      dbp[(size_t)c * E + e] = sb;
    }
}

// dw_r[i][e] = sum_c partial[c][e][i] (ascending c); db[e] = sum_c dbp[c][e]
__global__ void route_dw_reduce_kernel(const float* __restrict__ partial,
                                       const float* __restrict__ dbp, int n_chunks, int d, int E,
                                       float* __restrict__ dw_r, float* __restrict__ db_r) {
  const int q = blockIdx.x * blockDim.x + threadIdx.x;  // q = e * d + i
  if (q < d * E) {
    const int e = q / d, i = q % d;
    // ascending chunk order; the loads are independent, so several are in flight
    const float* pp = partial + (size_t)e * d + i;
    const size_t step = (size_t)E * d;
    float s = 0.0f;
    int c = 0;
    for (; c + 8 <= n_chunks; c += 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldg(pp + (size_t)(c + u) * step);
#pragma unroll
      for (int u = 0; u < 8; ++u) s += v[u];
    }
    for (; c < n_chunks; ++c) s += __ldg(pp + (size_t)c * step);
    dw_r[(size_t)i * E + e] = s;
  }
  if (db_r != nullptr && q < E) {
    float s = 0.0f;
    for (int c = 0; c < n_chunks; ++c) s += dbp[(size_t)c * E + q];
    db_r[q] = s;
  }
}

// dx[t,i] += sum_j dl[t,j] W_r[i, idx[t,j]]
template <typename T>
__global__ void route_dx_kernel(const float* __restrict__ dl, const int32_t* __restrict__ idx,
                                const T* __restrict__ w_r, int T_, int d, int E, int k,
                                T* __restrict__ dx) {
  const size_t q = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= (size_t)T_ * d) return;
  const int t = (int)(q / d), i = (int)(q % d);
  float s = to_f(dx[q]);
  for (int j = 0; j < k; ++j) {
    const int e = idx[(size_t)t * k + j];
    if (e >= 0 && e < E) s = fmaf(dl[(size_t)t * k + j], to_f(w_r[(size_t)i * E + e]), s);
  }
  dx[q] = from_f<T>(s);
}

}  // namespace

cudaError_t launch_route(const void* x, const void* w_r, const float* b_r, int T_, int d, int E,
                         int k, smoe_dtype dt, int32_t* idx, float* gates, unsigned* err,
                         cudaStream_t s) {
  if (dt == SMOE_BF16) return launch_route_dt<bf16>(x, w_r, b_r, T_, d, E, k, idx, gates, err, s);
  return launch_route_dt<float>(x, w_r, b_r, T_, d, E, k, idx, gates, err, s);
}

cudaError_t launch_route_dl(const float* gates, const float* dgates, int T_, int k, float* dl,
                            cudaStream_t s) {
  route_dl_kernel<<<cdiv(T_, 256), 256, 0, s>>>(gates, dgates, T_, k, dl);
  return cudaGetLastError();
}

namespace {
struct DwPlan {
  int chunk, n_chunks;
};
// 8 feature columns per thread, 1024 per block.  Tokens per chunk: halved from 256
// until the grid has two blocks per SM of a 148-SM B200 (a fixed count, so the
// summation order is the same on any GPU) and at most 4096 routing slots.
DwPlan route_dw_plan(int T_, int d, int E, int k) {
  DwPlan p;
  const int col_blocks = cdiv(d, kDwThreads * kDwColsPerThread);
  p.chunk = 256;
  while (p.chunk > 16 && (long long)cdiv(T_, p.chunk) * col_blocks < 2 * 148) p.chunk >>= 1;
  while (p.chunk > 1 && p.chunk * k > 4096) p.chunk >>= 1;
  p.n_chunks = cdiv(T_ > 0 ? T_ : 1, p.chunk);
  (void)E;
  return p;
}
}  // namespace

int route_dw_chunks(int T_, int d, int E, int k) { return route_dw_plan(T_, d, E, k).n_chunks; }

cudaError_t launch_route_dw(const void* x, const int32_t* idx, const float* dl, int T_, int d,
                            int E, int k, smoe_dtype dt, float* partial, int n_chunks,
                            float* dw_r, float* db_r, cudaStream_t s) {
  const DwPlan p = route_dw_plan(T_, d, E, k);
  if (p.n_chunks != n_chunks) return cudaErrorInvalidValue;  // workspace laid out for another plan
  float* dbp = partial + (size_t)n_chunks * E * d;
  const size_t smem = (size_t)p.chunk * k * 16 + (size_t)(E + 1) * 4;
  dim3 grid(n_chunks, cdiv(d, kDwThreads * kDwColsPerThread));
  if (dt == SMOE_BF16) {
    cudaError_t e = cudaFuncSetAttribute(route_dw_partial_kernel<bf16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    route_dw_partial_kernel<bf16><<<grid, kDwThreads, smem, s>>>((const bf16*)x, idx, dl, T_, d, E,
                                                                 k, p.chunk, partial, dbp);
  } else {
    cudaError_t e = cudaFuncSetAttribute(route_dw_partial_kernel<float>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    route_dw_partial_kernel<float><<<grid, kDwThreads, smem, s>>>((const float*)x, idx, dl, T_, d, E,
                                                                  k, p.chunk, partial, dbp);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  route_dw_reduce_kernel<<<cdiv(d * E, 256), 256, 0, s>>>(partial, dbp, n_chunks, d, E, dw_r, db_r);
  return cudaGetLastError();
}

cudaError_t launch_route_dx(const float* dl, const int32_t* idx, const void* w_r, int T_, int d,
                            int E, int k, smoe_dtype dt, void* dx, cudaStream_t s) {
  const size_t n = (size_t)T_ * d;
  const unsigned blocks = (unsigned)((n + 255) / 256);
  if (dt == SMOE_BF16)
    route_dx_kernel<bf16><<<blocks, 256, 0, s>>>(dl, idx, (const bf16*)w_r, T_, d, E, k, (bf16*)dx);
  else
    route_dx_kernel<float><<<blocks, 256, 0, s>>>(dl, idx, (const float*)w_r, T_, d, E, k, (float*)dx);
  return cudaGetLastError();
}

}  // namespace smoe
