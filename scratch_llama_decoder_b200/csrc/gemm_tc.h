// Tensor-core (tcgen05 / TMEM / TMA) paths of the training step: the GEMMs with
// their fused epilogues and the flash-style attention.  A TcPlan exists only
// for bfloat16 contexts; every entry returns false (or falls back to the SIMT
// kernels) for shapes it does not tile.
#pragma once
#include "internal.h"

namespace llm {

struct TcPlan;

enum TcEpi {
  TC_EPI_NONE = 0,   // plain output as selected by GemmOut
  TC_EPI_ROPE = 1,   // QKV forward: rotate q and k columns (RoPE) in the epilogue
  TC_EPI_SWIGLU = 2  // W13 forward: besides the interleaved [a|b], u = silu(a) b into U
};

TcPlan *tc_plan_create(DType dt, const float *cos_t, const float *sin_t, int T, int hd,
                       int64_t rot_cols, int64_t hp);
void tc_plan_destroy(TcPlan *p);
// Device flag word that records a bounded wait giving up (FLAG_TIMEOUT).
void tc_plan_set_flag(TcPlan *p, int *flag);
// U, ldu: the SwiGLU output of TC_EPI_SWIGLU (bf16 [M][ldu]; unused otherwise).
bool tc_gemm(TcPlan *p, const GemmOperands &g, GemmOut out, void *C, int64_t ldc, const float *R,
             int64_t ldr, int splits, int epi, cudaStream_t s, void *U = nullptr,
             int64_t ldu = 0);
// Whether tc_gemm runs an [M, N] product on CTA pairs (256 x 256 tiles, 74
// pairs on 148 SMs) rather than single CTAs (128 x 256 tiles).
bool tc_gemm_pairs(const TcPlan *p, int64_t M, int64_t N);

// Attention dispatch: tensor-core kernels when the plan covers the head size,
// else the SIMT kernels.
void attention_fwd(TcPlan *p, const void *qkv, void *o, float *lse, DType dt, int B, int T, int H,
                   int Hkv, int hd, cudaStream_t s);
// attention_bwd also applies the RoPE backward (rotation by -angle) to the dq
// and dk columns of dqkv: fused into the tensor-core kernels, a separate pass
// after the SIMT kernels.
void attention_bwd(TcPlan *p, const void *qkv, const void *o, const void *dout, const float *lse,
                   float *Dbuf, void *dqkv, DType dt, int B, int T, int H, int Hkv, int hd,
                   const float *cos_t, const float *sin_t, cudaStream_t s);

}  // namespace llm
