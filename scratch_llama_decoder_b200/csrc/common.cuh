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
// sigmoid by the fast exponential and reciprocal intrinsics (relative error
// ~1e-6, far below the bf16 rounding of the results)
LLM_DEV float sigmoid_fast(float a) { return __fdividef(1.0f, 1.0f + __expf(-a)); }
// One SwiGLU unit, u = a sigmoid(a) b, and its backward (g = du): the one
// arithmetic of the separate SwiGLU passes and of the GEMM epilogues that
// take them over, so both give the same bits.
LLM_DEV float swiglu_unit(float a, float b) { return a * sigmoid_fast(a) * b; }
LLM_DEV void swiglu_bwd_unit(float a, float b, float g, float &da, float &db) {
  const float sg = sigmoid_fast(a);
  da = g * b * sg * (1.f + a * (1.f - sg));
  db = g * a * sg;
}
LLM_DEV float round_bf16(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }
// The forward unit from float32 a and b rounded as the stored [a|b] is.
LLM_DEV float swiglu_unit_bf16(float a, float b) { return swiglu_unit(round_bf16(a), round_bf16(b)); }
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

// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy
// as 1, 2, 3", SC 2011): ten rounds of two 32x32 -> 64-bit products with the
// round keys bumped by the Weyl constants.
LLM_DEV void philox4x32_10(uint32_t c[4], uint32_t k0, uint32_t k1) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u, W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; r++) {
    uint32_t hi0 = __umulhi(M0, c[0]), lo0 = M0 * c[0];
    uint32_t hi1 = __umulhi(M1, c[2]), lo1 = M1 * c[2];
    uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0; c[1] = lo1; c[2] = n2; c[3] = lo0;
    k0 += W0; k1 += W1;
  }
}
// Keep bits of the elements 4g .. 4g + 3 of the dropout site a (bit j for
// element 4g + j): one generator call on counter (g, site, step), element
// 4g + j kept when output word j is >= a.thr (step: *a.step, read once by the
// caller).
LLM_DEV uint32_t drop_bits4(const llm::DropArgs &a, uint64_t g, uint32_t step) {
  uint32_t c[4] = {(uint32_t)g, (uint32_t)(g >> 32), a.site, step};
  philox4x32_10(c, a.k0, a.k1);
  return (uint32_t)(c[0] >= a.thr) | (uint32_t)(c[1] >= a.thr) << 1 |
         (uint32_t)(c[2] >= a.thr) << 2 | (uint32_t)(c[3] >= a.thr) << 3;
}
// 0 or a.scale for element e of the context's part of the dropout site a
// (whole-batch element a.e0 + e).
LLM_DEV float drop_factor(const llm::DropArgs &a, uint64_t e, uint32_t step) {
  const uint64_t E = a.e0 + e;
  return (drop_bits4(a, E >> 2, step) >> (E & 3)) & 1u ? a.scale : 0.f;
}
