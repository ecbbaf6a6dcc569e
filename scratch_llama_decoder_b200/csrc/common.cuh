// Device-side helpers shared by the kernels of the training step.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

#define LLM_DEV __device__ __forceinline__


// ---------------------------------------------------------------- types
LLM_DEV float to_f(float x) { return x; }
LLM_DEV float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> LLM_DEV T from_f(float x);
template <> LLM_DEV float from_f<float>(float x) { return x; }
template <> LLM_DEV __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// ---------------------------------------------------------------- reductions
LLM_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
LLM_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// silu and its derivative (Hephaistos, Architecture at a glance: SwiGLU).
LLM_DEV float sigmoidf_(float a) { return 1.0f / (1.0f + expf(-a)); }

// Column map of the interleaved W1|W3 block layout used by the low-precision
// weight copy and the saved [a|b] activations: hidden unit j's W1 column sits
// at (j/64)*128 + j%64 and its W3 column 64 further.
constexpr int SWIGLU_BLOCK = 64;
__host__ __device__ __forceinline__ int64_t w1_col(int64_t j) { return (j / SWIGLU_BLOCK) * (2 * SWIGLU_BLOCK) + (j % SWIGLU_BLOCK); }
