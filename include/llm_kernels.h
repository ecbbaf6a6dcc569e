/*
 * llm_kernels.h -- single hot-path kernels of the training step exposed for
 * parity tests and micro-benchmarks.  Same conventions as llm.h: d_* are
 * caller-owned DEVICE pointers, work is enqueued on `stream` (a cudaStream_t),
 * return codes are the LLM_* values of llm.h, nothing is allocated.  The
 * one-device-per-process rule of llm.h holds here too (LLM_ERR_ARG when
 * another device than the process's is current).
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

/* The same product with float32 operands (the float32 configurations):
 * tensor_cores = 1 runs the split-precision tensor-core kernel (3xTF32: each
 * operand split into a tf32 part and a float32 remainder, three tcgen05
 * kind::tf32 products accumulated in float32; relative error about 2^-21
 * per product), which first writes both parts of A and B, K-major, into
 * d_scratch: at least llm_kernel_gemm_f32_scratch_floats(M, N, K) floats,
 * 16-byte aligned, contents need no initialisation, LLM_ERR_ARG if smaller;
 * 0 runs the CUDA-core kernel (d_scratch unused).  d_flag as above. */
int llm_kernel_gemm_f32_scratch_floats(int M, int N, int K, int64_t *floats);
int llm_kernel_gemm_f32(int M, int N, int K, const float *d_A, int64_t lda, int a_kmajor,
                        const float *d_B, int64_t ldb, int b_kmajor, float *d_C, int64_t ldc,
                        int tensor_cores, float *d_scratch, int64_t scratch_floats, int *d_flag,
                        void *stream);

/* Causal self-attention of the step, bfloat16 operands and float32 softmax
 * (Hephaistos, Architecture at a glance: causal multi-head attention with a
 * numerically stable softmax; strata: n_head and n_kv_head independent,
 * flash-style forward and backward).  d_qkv: bf16 [batch*ctx, qkvw] with
 * qkvw = (n_head + 2*n_kv_head)*head_dim, per row all q heads, then k heads,
 * then v heads (RoPE already applied); query head h uses kv head
 * h / (n_head/n_kv_head); scale 1/sqrt(head_dim), the diagonal is kept.
 * Forward: d_o bf16 [batch*ctx, n_head*head_dim] (heads concatenated),
 * d_lse float32 [batch, n_head, ctx] = natural-log sum of exp of each score
 * row.  Backward: from d_o, d_lse and d_dout (bf16, like d_o) writes d_dqkv
 * (bf16, like d_qkv; every element written) and d_D float32 [batch, n_head,
 * ctx] = rowsum(dout * o) as scratch.  tensor_cores selects the kernels:
 * 2 = the tcgen05/TMEM kernels (head_dim 32 or 64; pointers 16-byte aligned),
 * 1 = the warp-level mma kernels (head_dim 32 or 64), 0 = the CUDA-core
 * kernels; LLM_ERR_ARG if the selection does not cover head_dim.  The calls
 * are asynchronous on `stream`.  The tcgen05 kernels bound every internal
 * wait (2 s); a wait that runs out ends the kernel early (outputs incomplete)
 * and is recorded only in a library-owned device word, which these entries do
 * not report (the training-step entries do report it, as LLM_ERR_TIMEOUT). */
int llm_kernel_attention_fwd_bf16(const void *d_qkv, void *d_o, float *d_lse, int batch, int ctx,
                                  int n_head, int n_kv_head, int head_dim, int tensor_cores,
                                  void *stream);
int llm_kernel_attention_bwd_bf16(const void *d_qkv, const void *d_o, const void *d_dout,
                                  const float *d_lse, float *d_D, void *d_dqkv, int batch,
                                  int ctx, int n_head, int n_kv_head, int head_dim,
                                  int tensor_cores, void *stream);

/* The same attention in float32 (the float32 configurations): d_qkv, d_o,
 * d_dout, d_dqkv float32 with the layouts above, d_lse and d_D as above.
 * tiled = 1 selects the tiled CUDA-core kernels (head_dim 32 or 64; rows
 * 16-byte aligned: pointers 16-byte aligned), 0 the one-warp-per-row
 * kernels (any head_dim); LLM_ERR_ARG otherwise.  Asynchronous on `stream`. */
int llm_kernel_attention_fwd_f32(const float *d_qkv, float *d_o, float *d_lse, int batch, int ctx,
                                 int n_head, int n_kv_head, int head_dim, int tiled, void *stream);
int llm_kernel_attention_bwd_f32(const float *d_qkv, const float *d_o, const float *d_dout,
                                 const float *d_lse, float *d_D, float *d_dqkv, int batch,
                                 int ctx, int n_head, int n_kv_head, int head_dim, int tiled,
                                 void *stream);

/* Embedding backward (Hephaistos, Architecture at a glance: token embedding;
 * its gradient is a scatter-add): dwte[v,:] = sum over positions i with
 * tokens[i] = v of dx[i,:], summed in increasing i (deterministic), zero for
 * ids that do not occur.  d_tokens: int32 [n_tokens] (ids outside
 * [0, vocab) are treated as 0); d_dx: float32 [n_tokens, d_model];
 * d_dwte: float32 [vocab, d_model], fully overwritten.  d_scratch: device
 * memory of at least llm_kernel_embed_bwd_scratch_bytes() bytes, 16-byte
 * aligned, used while the call's kernels run (its contents need no
 * initialisation).  LLM_ERR_ARG for null pointers, sizes < 1 or a small
 * scratch. */
int llm_kernel_embed_bwd_scratch_bytes(int64_t n_tokens, int vocab, int64_t *bytes);
int llm_kernel_embed_bwd(const int32_t *d_tokens, const float *d_dx, float *d_dwte,
                         int64_t n_tokens, int d_model, int vocab, void *d_scratch,
                         int64_t scratch_bytes, void *stream);

/* The embedding backward of llm_kernel_embed_bwd(), for callers that cannot
 * allocate device memory at call time: code running while a CUDA graph is
 * being captured, hooks inside an allocator, plug-ins whose host framework
 * owns all device memory, or loops that forbid allocation after start-up.
 * The source pages have no counterpart of this call; it exists for such
 * callers.  Same arguments, layout and result as llm_kernel_embed_bwd(),
 * without the scratch arguments: the scratch is one library-owned device
 * array of 1.5 MiB (394,307 int32) on every GPU that loads the library, kept
 * until the process exits.  Limits: n_tokens <= 65536 and vocab <= 65536,
 * else LLM_ERR_ARG with nothing launched.  The call allocates nothing (no
 * cudaMalloc, cudaFree or allocating library routine).  Its first call on a
 * device looks up the array's device address (cudaGetSymbolAddress, on the
 * current device) and caches it; make that first call before any stream
 * capture.  All calls on a device share the array: calls whose kernels
 * overlap on the GPU (different streams without ordering) race and give
 * wrong results; calls on one stream are ordered and safe.  Each call
 * re-initialises what it needs, so no state carries over between calls. */
int llm_kernel_embed_bwd_noalloc(const int32_t *d_tokens, const float *d_dx, float *d_dwte,
                                 int64_t n_tokens, int d_model, int vocab, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LLM_KERNELS_H_ */
