/*
 * llm_kernels.h -- single hot-path kernels of the training step exposed for
 * parity tests and micro-benchmarks.  Same conventions as llm.h: d_* are
 * caller-owned DEVICE pointers, work is enqueued on `stream` (a cudaStream_t),
 * return codes are the LLM_* values of llm.h, nothing is allocated.
 */
#ifndef LLM_KERNELS_H_
#define LLM_KERNELS_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The projection matmuls of the step (Hephaistos, Architecture at a glance:
 * every projection is x W; the backward needs dy W^T and x^T dy):
 *   C[M,N] (float32, row-major, leading dimension ldc) = sum_k A(m,k) B(n,k)
 * with bfloat16 operands
 *   A(m,k) = a_kmajor ? A[m*lda + k] : A[k*lda + m]
 *   B(n,k) = b_kmajor ? B[n*ldb + k] : B[k*ldb + n]
 * and float32 accumulation.  tensor_cores = 1 runs the tcgen05/TMA kernel
 * (LLM_ERR_ARG if it does not cover the arguments: 16-byte aligned pointers,
 * lda and ldb multiples of 8, ldc a multiple of 4); 0 runs the CUDA-core
 * kernel.  d_flag: one device int the tcgen05 kernel ORs a time-out bit into
 * (LLM_ERR_TIMEOUT semantics of llm.h); it is never cleared here. */
int llm_kernel_gemm_bf16(int M, int N, int K, const void *d_A, int64_t lda, int a_kmajor,
                         const void *d_B, int64_t ldb, int b_kmajor, float *d_C, int64_t ldc,
                         int tensor_cores, int *d_flag, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LLM_KERNELS_H_ */
