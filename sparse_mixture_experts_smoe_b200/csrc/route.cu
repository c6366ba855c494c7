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
// Two kernels compute these sums.  route_tiled_kernel (E * sizeof(T) a multiple
// of 16 bytes) blocks the (token, expert) tile over the warps and registers and
// streams W_r and x through a cp.async pipeline (see its comment).  route_kernel
// serves the other shapes: a warp handles TM tokens; a block of 8 warps stages CH
// rows of W_r in shared memory as fp32 with a row stride = 4 (mod 32) words, so
// the eight lanes of a 128-bit shared load phase read eight different bank
// groups, and the block's CH-feature slice of x with 16-byte coalesced loads
// (lane L then reads its features L, L+32, ... from shared memory; the
// accumulation order above is unchanged).
#include "common.cuh"

namespace smoe {
namespace {

constexpr int kRouteWarps = 8;

__host__ __device__ constexpr int route_row_stride(int emax) {
  // smallest stride >= emax with stride % 32 == 4 (floats)
  return emax + ((4 - emax % 32) + 32) % 32;
}

// Top-k of one token, warp-parallel: lane L holds the logits lv[j] of experts
// e = L + 32 j (bit j of fr: e is a candidate).  Each round reproduces the
// sequential scan "start at the first free expert, replace on a strictly greater
// logit": if the first free expert's logit is NaN it is taken, else the largest
// free non-NaN logit, the lower expert id on ties.  Gates: softmax over the
// selected logits (the first is the maximum).  Lane 0 writes idx_t[0:k], gates_t[0:k].
template <int NC>
__device__ __forceinline__ void select_topk(const float (&lv)[NC], unsigned fr, int k, int lane,
                                            int32_t* __restrict__ idx_t,
                                            float* __restrict__ gates_t) {
  constexpr int kNone = 0x7fffffff;
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
    if (lane == 0) idx_t[jj] = win;
  }
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
      gates_t[j] = expf(sel[j] - sel[0]) / z;
    }
  }
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

  constexpr int NC = EMAX >= 32 ? EMAX / 32 : 1;
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
    select_topk<NC>(lv, fr, k, lane, idx + (size_t)t * k, gates + (size_t)t * k);
  }
}

// ---------------------------------------------------------------------------
// Register-blocked router, for E * sizeof(T) a multiple of 16 bytes.  Same sums
// in the same order as route_kernel: lane L accumulates, for each (token, expert)
// of its warp's tile, the products of the features i = L (mod 32) in ascending i
// with fmaf (as packed pairs of experts, each component an fmaf).  The 8 warps of
// a block split its tile into GE expert groups of TE
// experts times GT token groups of TM tokens (TM * TE accumulators per lane), so a
// lane reads TM x values and TE W_r values per feature for TM * TE products.
// W_r and x rows stream through an NST-stage cp.async pipeline in their storage
// type and are converted at use (exact).  The 32 lane partials meet in a
// reduce-scatter whose pairings (lanes L ^ 16, ^ 8, ^ 4, ^ 2, ^ 1) are those of the
// xor butterfly, so every sum is the same fp32 value; lane L ends with values
// 4L .. 4L + 3 of the flattened tile (NV = TM * TE / 32 per lane in general).
__device__ __forceinline__ uint32_t rt_smem(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void rt_cp16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void rt_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void rt_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// one reduce-scatter step: keep half H of the values, add the partner lane's copy
template <int H, int O, int N>
__device__ __forceinline__ void rs_step(float (&v)[N], int lane) {
  const bool up = (lane & O) != 0;
#pragma unroll
  for (int q = 0; q < H; ++q) {
    const float send = up ? v[q] : v[q + H];
    const float keep = up ? v[q + H] : v[q];
    v[q] = keep + __shfl_xor_sync(0xffffffffu, send, O);
  }
}

// 8 values of T from 16 bytes (bf16) or 4 (fp32) as fp32
__device__ __forceinline__ void cvt16(const uint4 u, float* f, bf16) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 a = __bfloat1622float2(h[q]);
    f[2 * q] = a.x;
    f[2 * q + 1] = a.y;
  }
}
__device__ __forceinline__ void cvt16(const uint4 u, float* f, float) {
  f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
}

template <typename T, int EMAX, int TE, int TM>
struct RouteTile {
  static constexpr int SZ = (int)sizeof(T);
  static constexpr int GE = EMAX / TE, GT = 8 / GE, BT = GT * TM;
  static constexpr int CH = SZ == 2 ? 128 : 64;  // features per stage
  static constexpr int NST = SZ == 2 ? 4 : 3;    // pipeline stages
  static constexpr int WQ = EMAX * SZ / 16;      // 16-byte pieces of a staged W_r row
  // staged W_r row stride: an odd number of 16-byte units, so the 16-byte reads of
  // 8 consecutive lanes (consecutive rows) fall on 8 different bank groups
  static constexpr int WROW = (WQ % 2 == 1) ? WQ * 16 : WQ * 16 + 16;
  static constexpr int XQ = CH * SZ / 16;        // 16-byte pieces of a staged x row
  static constexpr int WBYTES = CH * WROW, XBYTES = BT * CH * SZ;
  static constexpr int STAGE = WBYTES + XBYTES;
  static constexpr int NACC = TM * TE, NV = NACC / 32;
  static constexpr size_t SMEM = (size_t)NST * STAGE + (size_t)BT * EMAX * 4;
  static_assert(GE * GT == 8 && NACC % 32 == 0 && NV % 2 == 0 && TE % NV == 0, "tile");
  static_assert((TE * SZ) % 16 == 0 && STAGE % 16 == 0, "16-byte pieces");
};

template <typename T, int EMAX, int TE, int TM, int MINB, bool FULL>
__global__ void __launch_bounds__(256, MINB)
route_tiled_kernel(const T* __restrict__ x, const T* __restrict__ w_r,
                   const float* __restrict__ b_r, int T_, int d, int E, int k,
                   int32_t* __restrict__ idx, float* __restrict__ gates) {
  using P = RouteTile<T, EMAX, TE, TM>;
  constexpr int SZ = P::SZ, CH = P::CH, NST = P::NST, NV = P::NV;
  extern __shared__ float4 smem_f4[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(smem_f4);
  float* logit = reinterpret_cast<float*>(sm + NST * P::STAGE);  // [BT][EMAX]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ge = warp % P::GE, tg = warp / P::GE;
  const int tb = blockIdx.x * P::BT;
  const int nchunks = cdiv(d, CH);
  // 16-byte pieces of a W_r row in global memory (a constant power of two when FULL)
  const int wq = FULL ? P::WQ : E * SZ / 16;

  // W_r columns [E, EMAX) of every stage are zero (the copies never write them)
  if constexpr (!FULL) {
    const int np = P::WQ - wq;  // > 0: E < EMAX
    for (int q = tid; q < NST * CH * np; q += blockDim.x) {
      const int st = q / (CH * np), rem = q % (CH * np);
      const int r = rem / np, pc = wq + rem % np;
      *reinterpret_cast<uint4*>(sm + st * P::STAGE + r * P::WROW + pc * 16) = make_uint4(0, 0, 0, 0);
    }
  }

  auto issue = [&](int c) {
    uint8_t* st = sm + (c % NST) * P::STAGE;
    const uint32_t wbase = rt_smem(st), xbase = rt_smem(st + P::WBYTES);
    const int i0 = c * CH;
    for (int q = tid; q < CH * wq; q += blockDim.x) {
      const int r = q / wq, pc = q % wq;
      const bool ok = i0 + r < d;
      const T* src = ok ? w_r + (size_t)(i0 + r) * E + pc * (16 / SZ) : w_r;
      rt_cp16(wbase + r * P::WROW + pc * 16, src, ok ? 16u : 0u);
    }
    for (int q = tid; q < P::BT * P::XQ; q += blockDim.x) {
      const int m = q / P::XQ, i = i0 + (q % P::XQ) * (16 / SZ);
      const int t = tb + m;
      const bool ok = t < T_ && i < d;  // d % 8 == 0: a 16-byte piece is all in or all out
      const T* src = ok ? x + (size_t)t * d + i : x;
      rt_cp16(xbase + q * 16, src, ok ? 16u : 0u);
    }
  };

  float2 acc[TM][TE / 2];  // (expert 2 e2, expert 2 e2 + 1) of token m
#pragma unroll
  for (int m = 0; m < TM; ++m)
#pragma unroll
    for (int e2 = 0; e2 < TE / 2; ++e2) acc[m][e2] = make_float2(0.0f, 0.0f);

#pragma unroll
  for (int st = 0; st < NST - 1; ++st) {
    if (st < nchunks) issue(st);
    rt_commit();
  }
  for (int c = 0; c < nchunks; ++c) {
    rt_wait<NST - 2>();  // this thread's copies of chunk c have landed ...
    __syncthreads();     // ... and everyone's; chunk c - 1's buffer is free
    if (c + NST - 1 < nchunks) issue(c + NST - 1);
    rt_commit();
    const uint8_t* st = sm + (c % NST) * P::STAGE;
    const T* xs = reinterpret_cast<const T*>(st + P::WBYTES) + (size_t)(tg * TM) * CH;
    const uint8_t* wsb = st + ge * TE * SZ;
    const int i0 = c * CH;
#pragma unroll 2
    for (int j = 0; j < CH / 32; ++j) {
      const int r = lane + 32 * j;
      if (i0 + r >= d) break;
      float xv[TM];
#pragma unroll
      for (int m = 0; m < TM; ++m) xv[m] = to_f(xs[m * CH + r]);
      float w[TE];
#pragma unroll
      for (int u = 0; u < TE * SZ / 16; ++u)
        cvt16(*reinterpret_cast<const uint4*>(wsb + r * P::WROW + u * 16), w + u * (16 / SZ), T());
      // packed pairs of experts: per component exactly fmaf(x, w, acc)
#pragma unroll
      for (int e2 = 0; e2 < TE / 2; ++e2) {
        const float2 w2 = make_float2(w[2 * e2], w[2 * e2 + 1]);
#pragma unroll
        for (int m = 0; m < TM; ++m) acc[m][e2] = __ffma2_rn(make_float2(xv[m], xv[m]), w2, acc[m][e2]);
      }
    }
  }
  rt_wait<0>();

  // lane partials -> sums (the butterfly's pairings), NV per lane
  float v[P::NACC];
#pragma unroll
  for (int m = 0; m < TM; ++m)
#pragma unroll
    for (int e2 = 0; e2 < TE / 2; ++e2) {
      v[m * TE + 2 * e2] = acc[m][e2].x;
      v[m * TE + 2 * e2 + 1] = acc[m][e2].y;
    }
  rs_step<P::NACC / 2, 16>(v, lane);
  rs_step<P::NACC / 4, 8>(v, lane);
  rs_step<P::NACC / 8, 4>(v, lane);
  rs_step<P::NACC / 16, 2>(v, lane);
  rs_step<P::NACC / 32, 1>(v, lane);
  {
    const int f = NV * lane;  // flattened (m, e) of v[0]; NV consecutive e, TE % NV == 0
    const int m = f / TE, e = f % TE;
    float* dst = logit + (tg * TM + m) * EMAX + ge * TE + e;
#pragma unroll
    for (int q = 0; q < NV; q += 2) *reinterpret_cast<float2*>(dst + q) = make_float2(v[q], v[q + 1]);
  }
  __syncthreads();

  constexpr int NC = EMAX >= 32 ? EMAX / 32 : 1;
  for (int m = warp; m < P::BT; m += 8) {
    const int t = tb + m;
    if (t >= T_) break;
    float lv[NC];
    unsigned fr = 0u;
#pragma unroll
    for (int j = 0; j < NC; ++j) {
      const int e = lane + 32 * j;
      const bool in = e < E;
      const float a = in ? logit[m * EMAX + e] : 0.0f;
      lv[j] = (in && b_r != nullptr) ? a + b_r[e] : a;
      if (in) fr |= 1u << j;
    }
    select_topk<NC>(lv, fr, k, lane, idx + (size_t)t * k, gates + (size_t)t * k);
  }
}

template <typename T, int EMAX, int TE, int TM, int MINB>
cudaError_t launch_route_tiled(const void* x, const void* w_r, const float* b_r, int T_, int d,
                               int E, int k, int32_t* idx, float* gates, cudaStream_t s) {
  using P = RouteTile<T, EMAX, TE, TM>;
  auto kern = E == EMAX ? route_tiled_kernel<T, EMAX, TE, TM, MINB, true>
                        : route_tiled_kernel<T, EMAX, TE, TM, MINB, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<cdiv(T_, P::BT), 256, P::SMEM, s>>>((const T*)x, (const T*)w_r, b_r, T_, d, E, k, idx, gates);
  return cudaGetLastError();
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

// ---------------------------------------------------------------------------
// Router for a few tokens (decode).  With T tokens there are only 32 * E * T
// lane chains, too few to fill a pipeline of feature chunks, so each chain gets
// its own thread: one block per token, warp w takes experts w, w + 16, ...; lane L
// accumulates x[t, i] * W_r[i, e] over i = L (mod 32) in ascending i with fmaf
// (several loads in flight), then the xor butterfly 16, 8, 4, 2, 1 and + b: the
// documented order, so the logits are the same bits as the other kernels'.
constexpr int kChainWarps = 16;
constexpr int kChainMaxT = 64;

template <typename T>
__global__ void __launch_bounds__(kChainWarps * 32)
route_chain_kernel(const T* __restrict__ x, const T* __restrict__ w_r,
                   const float* __restrict__ b_r, int d, int E, int k,
                   int32_t* __restrict__ idx, float* __restrict__ gates) {
  __shared__ float logit[128];
  const int t = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const T* xt = x + (size_t)t * d;
  for (int e = warp; e < E; e += kChainWarps) {
    float acc = 0.0f;
#pragma unroll 8
    for (int i = lane; i < d; i += 32) acc = fmaf(to_f(xt[i]), to_f(w_r[(size_t)i * E + e]), acc);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) acc = acc + __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) logit[e] = b_r != nullptr ? acc + b_r[e] : acc;
  }
  __syncthreads();
  if (warp == 0) {
    float lv[4];
    unsigned fr = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = lane + 32 * j;
      lv[j] = e < E ? logit[e] : 0.0f;
      if (e < E) fr |= 1u << j;
    }
    select_topk<4>(lv, fr, k, lane, idx + (size_t)t * k, gates + (size_t)t * k);
  }
}

template <typename T>
cudaError_t launch_route_dt(const void* x, const void* w_r, const float* b_r, int T_, int d, int E,
                            int k, int32_t* idx, float* gates, unsigned* err, cudaStream_t s) {
  if (T_ <= kChainMaxT) {
    route_chain_kernel<T><<<T_, kChainWarps * 32, 0, s>>>((const T*)x, (const T*)w_r, b_r, d, E, k,
                                                          idx, gates);
    return cudaGetLastError();
  }
  // Tiles of 64 accumulators per lane (two blocks per SM) measured faster than
  // 128 (one block per SM) on the 64-expert router: the shorter per-lane work
  // hides the shared-memory and conversion latencies better.
  if ((E * (int)sizeof(T)) % 16 == 0) {  // W_r rows copy as 16-byte pieces
    if (E <= 8) return launch_route_tiled<T, 8, 8, 8, 2>(x, w_r, b_r, T_, d, E, k, idx, gates, s);
    if (E <= 16) return launch_route_tiled<T, 16, 16, 4, 2>(x, w_r, b_r, T_, d, E, k, idx, gates, s);
    if (E <= 32) return launch_route_tiled<T, 32, 16, 4, 2>(x, w_r, b_r, T_, d, E, k, idx, gates, s);
    if (E <= 64) return launch_route_tiled<T, 64, 16, 4, 2>(x, w_r, b_r, T_, d, E, k, idx, gates, s);
    return launch_route_tiled<T, 128, 16, 4, 2>(x, w_r, b_r, T_, d, E, k, idx, gates, s);
  }
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

// Router weight gradient, dw_r[i, e] = sum_t x[t, i] dl[t, e], over the slots in
// grouped order (sorted by expert, token order within an expert).  The grouped
// rows are cut into segments of R rows; a warp walks one segment for one slab
// of columns, accumulating the current expert's sum in registers, and writes one
// partial row per (segment w, expert e) run it meets.  Along the grouped order the
// expert never decreases, so w + e numbers the runs without collisions
// (S / R + E rows).  A second pass sums, for each expert, the runs of the
// segments its slice covers in ascending w.  The order of every addition depends
// only on (T, k, E) and the routing, not on the GPU.  x is read once per slot,
// mostly from L2 (k reads of each token row).
// R (128, 64 or 32 rows) and the slab width (2 or 1 16-byte loads per lane and row)
// follow from (S, d) alone -- the largest that still gives two blocks per SM of a
// 148-SM B200 -- so the order of the additions is fixed by the shape.
struct DwPlan {
  int rows, loads;
};
DwPlan dw_plan(int S, int d) {
  const int cands[4][2] = {{128, 2}, {64, 2}, {32, 2}, {32, 1}};
  for (const auto& c : cands) {
    const long long blocks = (long long)cdiv(cdiv(S > 0 ? S : 1, c[0]), 8) * cdiv(d, 32 * c[1] * 8);
    if (blocks >= 2 * 148) return {c[0], c[1]};
  }
  return {32, 1};
}

template <typename T, int LOADS>
struct DwSlab {
  static constexpr int VPL = 16 / (int)sizeof(T);       // elements per 16-byte load
  static constexpr int COLS = 32 * LOADS * VPL;          // slab width
};

template <typename T, int LOADS>
__global__ void __launch_bounds__(256)
route_dw_run_kernel(const T* __restrict__ x, const int32_t* __restrict__ idx,
                    const int32_t* __restrict__ sorted_slot, const float* __restrict__ dl, int S,
                    int d, int E, int k, int R, float* __restrict__ part,
                    float* __restrict__ partb) {
  constexpr int VPL = DwSlab<T, LOADS>::VPL, NA = LOADS * VPL;
  const int lane = threadIdx.x & 31;
  const int w = blockIdx.x * 8 + (threadIdx.x >> 5);  // segment
  const int r0 = w * R;
  if (r0 >= S) return;
  const int r1 = min(S, r0 + R);
  const int c0 = blockIdx.y * DwSlab<T, LOADS>::COLS + lane * VPL;  // column of load u: c0 + 32 u VPL
  float2 acc[NA / 2];
#pragma unroll
  for (int a = 0; a < NA / 2; ++a) acc[a] = make_float2(0.f, 0.f);
  float bsum = 0.f;
  int cur = -1;
  auto flush = [&]() {
    if (cur < 0) return;
    float* dst = part + (size_t)(w + cur) * d;
#pragma unroll
    for (int u = 0; u < LOADS; ++u) {
      const int col = c0 + u * 32 * VPL;
      if (col >= d) continue;
#pragma unroll
      for (int v = 0; v < VPL; v += 4)
        *reinterpret_cast<float4*>(dst + col + v) =
            make_float4(acc[(u * VPL + v) / 2].x, acc[(u * VPL + v) / 2].y,
                        acc[(u * VPL + v) / 2 + 1].x, acc[(u * VPL + v) / 2 + 1].y);
    }
    if (blockIdx.y == 0 && lane == 0) partb[w + cur] = bsum;
  };
  for (int b0 = r0; b0 < r1; b0 += 32) {
    const int n = min(32, r1 - b0);
    // this batch's rows, one per lane: slot, expert, token, gate gradient
    int e = -1, t = 0;
    float g = 0.f;
    if (lane < n) {
      const int p = sorted_slot[b0 + lane];
      if (p >= 0 && p < S) {
        const int ee = idx[p];
        if (ee >= 0 && ee < E) { e = ee; t = p / k; g = dl[p]; }
      }
    }
    for (int j = 0; j < n; j += 4) {
      uint4 xv[4][LOADS];
      int ej[4];
      float gj[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {  // four rows' loads in flight
        const int jj = j + q;        // < 32
        const int e_q = __shfl_sync(0xffffffffu, e, jj);
        const int t_q = __shfl_sync(0xffffffffu, t, jj);
        gj[q] = __shfl_sync(0xffffffffu, g, jj);
        ej[q] = jj < n ? e_q : -1;
#pragma unroll
        for (int u = 0; u < LOADS; ++u) {
          const int col = c0 + u * 32 * VPL;
          xv[q][u] = (ej[q] >= 0 && col < d)
                         ? __ldg(reinterpret_cast<const uint4*>(x + (size_t)t_q * d + col))
                         : make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (ej[q] < 0) continue;  // warp-uniform
        if (ej[q] != cur) {
          flush();
#pragma unroll
          for (int a = 0; a < NA / 2; ++a) acc[a] = make_float2(0.f, 0.f);
          bsum = 0.f;
          cur = ej[q];
        }
        const float2 g2 = make_float2(gj[q], gj[q]);
#pragma unroll
        for (int u = 0; u < LOADS; ++u) {
          float xf[VPL];
          cvt16(xv[q][u], xf, T());
#pragma unroll
          for (int v = 0; v < VPL; v += 2)
            acc[(u * VPL + v) / 2] = __ffma2_rn(make_float2(xf[v], xf[v + 1]), g2, acc[(u * VPL + v) / 2]);
        }
        bsum += gj[q];
      }
    }
  }
  flush();
}

// dw_r[i][e] = sum over the segments w covering expert e's rows (ascending) of
// part[w + e][i]; db_r[e] likewise from partb
__global__ void route_dw_sum_kernel(const float* __restrict__ part, const float* __restrict__ partb,
                                    const int32_t* __restrict__ offsets, int S, int d, int E, int R,
                                    float* __restrict__ dw_r, float* __restrict__ db_r) {
  const int q = blockIdx.x * blockDim.x + threadIdx.x;  // q = e * d + i
  if (q >= d * E) return;
  const int e = q / d, i = q % d;
  const int lo = min(max(offsets[e], 0), S), hi = min(max(offsets[e + 1], lo), S);
  float s = 0.f, sb = 0.f;
  if (hi > lo) {
    const int w1 = (hi - 1) / R;
    for (int w = lo / R; w <= w1; ++w) {
      s += __ldg(part + (size_t)(w + e) * d + i);
      if (i == 0) sb += partb[w + e];
    }
  }
  dw_r[(size_t)i * E + e] = s;
  if (i == 0 && db_r != nullptr) db_r[e] = sb;
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

int route_dw_runs(int S, int E, int d) { return cdiv(S > 0 ? S : 1, dw_plan(S, d).rows) + E; }

cudaError_t launch_route_dw(const void* x, const int32_t* idx, const int32_t* sorted_slot,
                            const int32_t* offsets, const float* dl, int T_, int d, int E, int k,
                            smoe_dtype dt, float* part, float* dw_r, float* db_r, cudaStream_t s) {
  const int S = T_ * k;
  const DwPlan pl = dw_plan(S, d);
  const int nseg = cdiv(S, pl.rows);
  float* partb = part + (size_t)route_dw_runs(S, E, d) * d;
  if (dt == SMOE_BF16) {
    if (pl.loads == 2) {
      dim3 grid(cdiv(nseg, 8), cdiv(d, DwSlab<bf16, 2>::COLS));
      route_dw_run_kernel<bf16, 2><<<grid, 256, 0, s>>>((const bf16*)x, idx, sorted_slot, dl, S, d, E, k,
                                                        pl.rows, part, partb);
    } else {
      dim3 grid(cdiv(nseg, 8), cdiv(d, DwSlab<bf16, 1>::COLS));
      route_dw_run_kernel<bf16, 1><<<grid, 256, 0, s>>>((const bf16*)x, idx, sorted_slot, dl, S, d, E, k,
                                                        pl.rows, part, partb);
    }
  } else {
    if (pl.loads == 2) {
      dim3 grid(cdiv(nseg, 8), cdiv(d, DwSlab<float, 2>::COLS));
      route_dw_run_kernel<float, 2><<<grid, 256, 0, s>>>((const float*)x, idx, sorted_slot, dl, S, d,
                                                         E, k, pl.rows, part, partb);
    } else {
      dim3 grid(cdiv(nseg, 8), cdiv(d, DwSlab<float, 1>::COLS));
      route_dw_run_kernel<float, 1><<<grid, 256, 0, s>>>((const float*)x, idx, sorted_slot, dl, S, d,
                                                         E, k, pl.rows, part, partb);
    }
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  route_dw_sum_kernel<<<cdiv(d * E, 256), 256, 0, s>>>(part, partb, offsets, S, d, E, pl.rows, dw_r,
                                                       db_r);
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
