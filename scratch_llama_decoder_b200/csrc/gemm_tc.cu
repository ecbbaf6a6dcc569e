// tcgen05 GEMM (placeholder: no shapes covered yet; the SIMT kernels run).
#include "gemm_tc.h"

namespace llm {

struct TcPlan {
  int unused;
};

TcPlan *tc_plan_create(DType, const float *, const float *, int, int, int64_t, int64_t) {
  return nullptr;
}
void tc_plan_destroy(TcPlan *p) { delete p; }
bool tc_gemm(TcPlan *, const GemmOperands &, GemmOut, void *, int64_t, const float *, int64_t, int,
             int, const void *, cudaStream_t) {
  return false;
}
void attention_fwd(TcPlan *, const void *qkv, void *o, float *lse, DType dt, int B, int T, int H,
                   int Hkv, int hd, cudaStream_t s) {
  attn_fwd_simt(qkv, o, lse, dt, B, T, H, Hkv, hd, s);
}
void attention_bwd(TcPlan *, const void *qkv, const void *o, const void *dout, const float *lse,
                   float *Dbuf, void *dqkv, DType dt, int B, int T, int H, int Hkv, int hd,
                   cudaStream_t s) {
  attn_bwd_simt(qkv, o, dout, lse, Dbuf, dqkv, dt, B, T, H, Hkv, hd, s);
}

}  // namespace llm
