// fp8.cu -- e4m3 quantisation for the FP8 inference forward (sourcepulse.org project
// summary: inference speed as a target).
//
// Weights: one fp32 scale per (expert, output column) over that column's K values,
// codes stored K-major [E, N, K] so that both operands of the tcgen05 FP8 product
// are K-major.  Activations: one scale per row.  The scale maps the row's (column's)
// largest magnitude to 448, the largest e4m3 value: scale = amax / 448 in fp32 (1 for
// an all-zero row), code = e4m3(fl32(v / scale)), rounded to nearest even and
// saturated by the hardware conversion (cvt.rn.satfinite.e4m3x2.f32).
#include "tc_ptx.cuh"

namespace smoe {
namespace {

// Two fp32 values -> two e4m3 codes (lo in the low byte).
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

// One warp per row of a [rows, cols] bf16 matrix (cols % 8 == 0): scale, then codes.
__global__ void quantize_rows_kernel(const bf16* __restrict__ x, int rows, int cols,
                                     uint8_t* __restrict__ codes, float* __restrict__ scales) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= rows) return;
  const bf16* xr = x + (size_t)row * cols;
  float amax = 0.0f;
  for (int c = 8 * lane; c < cols; c += 256) {
    float v[8];
    unpack8(*reinterpret_cast<const uint4*>(xr + c), v);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
  }
  amax = warp_max(amax);
  const float s = amax > 0.0f ? amax / 448.0f : 1.0f;
  uint8_t* cr = codes + (size_t)row * cols;
  for (int c = 8 * lane; c < cols; c += 256) {
    float v[8];
    unpack8(*reinterpret_cast<const uint4*>(xr + c), v);
    uint2 out;
    out.x = (uint32_t)e4m3x2(v[0] / s, v[1] / s) | ((uint32_t)e4m3x2(v[2] / s, v[3] / s) << 16);
    out.y = (uint32_t)e4m3x2(v[4] / s, v[5] / s) | ((uint32_t)e4m3x2(v[6] / s, v[7] / s) << 16);
    *reinterpret_cast<uint2*>(cr + c) = out;
  }
  if (lane == 0) scales[row] = s;
}

// Weights W [E, K, N] bf16 -> codes [E, N, K], scales [E, N].  A block takes 32
// output columns of one expert: its warps first find each column's largest
// magnitude (coalesced along N), then write the codes through a shared-memory
// transpose, 32 columns x 64 K values at a time (coalesced along K).
__global__ void quantize_weights_kernel(const bf16* __restrict__ w, int K, int N,
                                        uint8_t* __restrict__ codes, float* __restrict__ scales) {
  __shared__ float part[8][32];
  __shared__ float sc[32];
  __shared__ uint8_t tile[32][64 + 4];
  const int e = blockIdx.y, n0 = blockIdx.x * 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = n0 + lane;
  const bf16* we = w + (size_t)e * K * N;
  float amax = 0.0f;
  if (n < N)
    for (int k = warp; k < K; k += 8) amax = fmaxf(amax, fabsf(__bfloat162float(we[(size_t)k * N + n])));
  part[warp][lane] = amax;
  __syncthreads();
  if (warp == 0) {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, part[i][lane]);
    const float s = m > 0.0f ? m / 448.0f : 1.0f;
    sc[lane] = s;
    if (n < N) scales[(size_t)e * N + n] = s;
  }
  __syncthreads();
  for (int k0 = 0; k0 < K; k0 += 64) {
    // load 64 K rows x 32 columns (warp w: rows k0 + w + 8 i), quantise, stage transposed
    for (int i = 0; i < 8; ++i) {
      const int kk = warp + 8 * i, k = k0 + kk;
      uint8_t cde = 0;
      if (n < N && k < K) {
        const float v = __bfloat162float(we[(size_t)k * N + n]) / sc[lane];
        cde = (uint8_t)(e4m3x2(v, 0.0f) & 0xFF);
      }
      tile[lane][kk] = cde;
    }
    __syncthreads();
    // write: warp w covers columns w, w + 8, w + 16, w + 24; lane l writes K bytes 2l, 2l+1
    for (int i = 0; i < 4; ++i) {
      const int cl = warp + 8 * i, nn = n0 + cl, k = k0 + 2 * lane;
      if (nn < N && k < K) {
        uint8_t* dst = codes + ((size_t)e * N + nn) * K + k;
        dst[0] = tile[cl][2 * lane];
        if (k + 1 < K) dst[1] = tile[cl][2 * lane + 1];
      }
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_quantize_rows_fp8(const void* x, int rows, int cols, uint8_t* codes, float* scales,
                                     cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  quantize_rows_kernel<<<cdiv(rows, 8), 256, 0, s>>>((const bf16*)x, rows, cols, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_quantize_weights_fp8(const void* w, int E, int K, int N, uint8_t* codes, float* scales,
                                        cudaStream_t s) {
  dim3 grid(cdiv(N, 32), E);
  quantize_weights_kernel<<<grid, 256, 0, s>>>((const bf16*)w, K, N, codes, scales);
  return cudaGetLastError();
}

}  // namespace smoe
