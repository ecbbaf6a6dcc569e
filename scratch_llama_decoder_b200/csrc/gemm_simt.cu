// CUDA-core GEMM for the float32 configurations and for shapes the tensor-core
// path does not tile (tiny heads, ragged sizes).  64x64 output tile per block,
// K in steps of 16, 4x4 outputs per thread, float32 accumulation.
#include "common.cuh"
#include "internal.h"

namespace llm {

constexpr int SB_M = 64, SB_N = 64, SB_K = 16;

template <typename T, bool KMAJOR>
LLM_DEV void load_tile(const T *__restrict__ X, int64_t ld, int rows, int K, int r0, int k0,
                       float (*S)[SB_M + 4]) {
  // S[k][r] = X(r0 + r, k0 + k); element (r,k) = KMAJOR ? X[r*ld + k] : X[k*ld + r]
  int t = threadIdx.x;
#pragma unroll
  for (int it = 0; it < 4; it++) {
    int r, k;
    if (KMAJOR) { k = t % SB_K; r = t / SB_K + 16 * it; }
    else { r = t % SB_M; k = t / SB_M + 4 * it; }
    int gr = r0 + r, gk = k0 + k;
    float v = 0.f;
    if (gr < rows && gk < K) v = to_f(KMAJOR ? X[(int64_t)gr * ld + gk] : X[(int64_t)gk * ld + gr]);
    S[k][r] = v;
  }
}

template <typename T, bool AK, bool BK>
__global__ void __launch_bounds__(256) k_gemm_simt(int M, int N, int K, const T *__restrict__ A,
                                                   int64_t lda, const T *__restrict__ B,
                                                   int64_t ldb, int out, void *C, int64_t ldc,
                                                   const float *__restrict__ R, int64_t ldr,
                                                   int kchunk) {
  __shared__ float As[SB_K][SB_M + 4], Bs[SB_K][SB_N + 4];
  int m0 = blockIdx.y * SB_M, n0 = blockIdx.x * SB_N;
  int kb = blockIdx.z * kchunk, ke = min(K, kb + kchunk);
  int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = kb; k0 < ke; k0 += SB_K) {
    load_tile<T, AK>(A, lda, M, ke, m0, k0, As);
    load_tile<T, BK>(B, ldb, N, ke, n0, k0, Bs);
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SB_K; kk++) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; i++) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; j++) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; i++) {
    int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; j++) {
      int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc[i][j];
      if (out == OUT_F32) ((float *)C)[(int64_t)m * ldc + n] = v;
      else if (out == OUT_ACT) ((T *)C)[(int64_t)m * ldc + n] = from_f<T>(v);
      else if (out == OUT_ADD_F32) ((float *)C)[(int64_t)m * ldc + n] = R[(int64_t)m * ldr + n] + v;
      else ((float *)C)[(int64_t)blockIdx.z * M * ldc + (int64_t)m * ldc + n] = v;
    }
  }
}

template <typename T>
static void launch(const GemmOperands &g, GemmOut out, void *C, int64_t ldc, const float *R,
                   int64_t ldr, int splits, cudaStream_t s) {
  int kchunk = (g.K + splits - 1) / splits;
  kchunk = ((kchunk + SB_K - 1) / SB_K) * SB_K;
  dim3 grid((g.N + SB_N - 1) / SB_N, (g.M + SB_M - 1) / SB_M, splits);
  const T *A = (const T *)g.A, *B = (const T *)g.B;
#define L(AK, BK)                                                                    \
  k_gemm_simt<T, AK, BK><<<grid, 256, 0, s>>>(g.M, g.N, g.K, A, g.lda, B, g.ldb, out, C, ldc, R, \
                                              ldr, kchunk)
  if (g.a_kmajor && g.b_kmajor) L(true, true);
  else if (g.a_kmajor) L(true, false);
  else if (g.b_kmajor) L(false, true);
  else L(false, false);
#undef L
  count_launch();
}

void gemm_simt(const GemmOperands &g, GemmOut out, void *C, int64_t ldc, const float *R,
               int64_t ldr, int splits, cudaStream_t s) {
  if (splits < 1) splits = 1;
  if (out != OUT_PARTIAL) splits = 1;
  if (g.in == DT_BF16) launch<__nv_bfloat16>(g, out, C, ldc, R, ldr, splits, s);
  else launch<float>(g, out, C, ldc, R, ldr, splits, s);
}

}  // namespace llm
