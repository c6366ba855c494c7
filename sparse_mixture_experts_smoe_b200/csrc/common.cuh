// common.cuh -- device helpers shared by the kernels of libsmoe.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace smoe {

typedef __nv_bfloat16 bf16;

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(bf16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ void report_error(unsigned* err, unsigned bit) {
  if (err) atomicOr(err, bit);
}

// Source row of grouped row i for a row-indexed operand.
__device__ __forceinline__ int src_row(int mode, int i, const int32_t* sorted_slot, int fan_out) {
  return mode == ROWS_GROUPED ? i : sorted_slot[i] / fan_out;
}

// Activations in fp32 (tanh-approximated GELU and SiLU) and their derivatives.
__device__ __forceinline__ float gelu_tanh_f(float h) {
  const float u = 0.7978845608028654f * fmaf(0.044715f * h, h * h, h);
  return 0.5f * h * (1.0f + tanhf(u));
}
__device__ __forceinline__ float gelu_tanh_grad_f(float h) {
  const float u = 0.7978845608028654f * fmaf(0.044715f * h, h * h, h);
  const float th = tanhf(u);
  const float du = 0.7978845608028654f * fmaf(3.0f * 0.044715f, h * h, 1.0f);
  return 0.5f * (1.0f + th) + 0.5f * h * (1.0f - th * th) * du;
}
__device__ __forceinline__ float sigmoid_f(float z) { return 1.0f / (1.0f + expf(-z)); }
__device__ __forceinline__ float silu_f(float z) { return z * sigmoid_f(z); }
__device__ __forceinline__ float silu_grad_f(float z) {
  const float s = sigmoid_f(z);
  return s * (1.0f + z * (1.0f - s));
}

// Ceil-div.
__host__ __device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }

}  // namespace smoe
