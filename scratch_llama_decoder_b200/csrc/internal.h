// Host-side launchers of the training-step kernels (internal to the library).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace llm {

// Error bits of the per-step flag word in device memory.
enum : int { FLAG_TOKEN = 1, FLAG_NONFINITE = 2, FLAG_TIMEOUT = 4 };

// Activation/operand element type of a launch: float32 or bfloat16.
enum DType { DT_F32 = 0, DT_BF16 = 1 };

// Inverted-dropout masks of one site (Hephaistos: dropout on the embeddings,
// the attention weights and the attention and MLP outputs; masks drawn by the
// training forward and reused by its backward).  Element e of the site is kept
// when word 0 of Philox4x32-10(counter = (e low, e high, site, *step), key =
// (k0, k1)) is >= thr = floor(p * 2^32); kept elements are scaled by `scale`
// = 1 / (1 - p).  on = 0: no dropout.
struct DropArgs {
  int on = 0;
  uint32_t thr = 0, k0 = 0, k1 = 0, site = 0;
  float scale = 1.f;
  const int *step = nullptr;  // device word: the training forward's number
  // index of the context's first element of the site in the whole batch (its
  // first sequence's offset, llm_set_dropout_offset, times the elements a
  // sequence has at the site); kernels index masks at e0 + their own index
  uint64_t e0 = 0;
};

// ------------------------------------------------------------ GEMM (shared)
// C[M,N] = A[M,K] * B^T where B is given as an [N,K] operand:
//   A element (m,k) = a_kmajor ? A[m*lda + k] : A[k*lda + m]
//   B element (n,k) = b_kmajor ? B[n*ldb + k] : B[k*ldb + n]
struct GemmOperands {
  int M, N, K;
  const void *A; int64_t lda; bool a_kmajor;
  const void *B; int64_t ldb; bool b_kmajor;
  DType in;  // operand type of A and B
};
enum GemmOut {
  OUT_F32 = 0,      // C (float) = acc
  OUT_ACT = 1,      // C (operand type) = acc, rounded
  OUT_ADD_F32 = 2,  // C (float) = R + acc
  OUT_PARTIAL = 3   // C (float) [split][M][ldc] = partial sum over the split's K range
};
// float32 GEMM on the tensor cores in split precision (3xTF32, gemm_tf32.cu):
// false (nothing launched) unless A, B are float32 and the scratch holds
// gemm_tf32_scratch_floats(M, N, K) floats (16-byte aligned).  Counts launches.
int64_t gemm_tf32_scratch_floats(int64_t M, int64_t N, int64_t K);
bool gemm_tf32(const GemmOperands &g, GemmOut out, void *C, int64_t ldc, const float *R,
               int64_t ldr, int splits, float *scratch, int64_t scratch_floats, int *flag,
               cudaStream_t s);
// SIMT (CUDA-core) GEMM: any shape, float32 accumulation.  Counts launches.
void gemm_simt(const GemmOperands &g, GemmOut out, void *C, int64_t ldc, const float *R,
               int64_t ldr, int splits, cudaStream_t s);

// ------------------------------------------------------------- elementwise
// cos/sin [T, hd/2] of the angles (t / scale) * base^(-2j/hd).
void rope_table(float *cos_t, float *sin_t, int T, int hd, float base, cudaStream_t s,
                double scale = 1.0);
// Low-precision (or float32) padded copy of one weight matrix.
//   mode 0: dst[r, c] = src[r, c] (zero outside rows x cols), dst [rows_p, cols_p]
//   mode 1: W13 interleave: src [rows, 2h], dst [rows, 2hp] block-interleaved
void cast_weight(const float *src, void *dst, DType dt, int64_t rows, int64_t cols,
                 int64_t rows_p, int64_t cols_p, int mode, int64_t h, int64_t hp, int batch,
                 int64_t src_batch_stride, int64_t dst_batch_stride, cudaStream_t s);
void embed_fwd(const float *wte, const int32_t *tok, float *x, int64_t N, int d, int V,
               int *flag, cudaStream_t s);
void rmsnorm_fwd(const float *x, const float *g, void *y, DType dt, float *rstd, int64_t N, int d,
                 float eps, cudaStream_t s);
// dx = dres + rmsnorm_bwd(dy); optional low-precision copy dx_act; dg partial
// sums per block into part[nblk, d].  Returns the number of partial blocks.
int rmsnorm_bwd(const float *x, const float *rstd, const float *g, const float *dy,
                const float *dres, float *dx, void *dx_act, DType dt, float *part, int64_t N,
                int d, cudaStream_t s);
int rmsnorm_bwd_blocks(int64_t N);
void reduce_partials(const float *part, int nblk, int d, float *out, cudaStream_t s);
void rope_apply(void *qkv, DType dt, const float *cos_t, const float *sin_t, int64_t N, int T,
                int ncols_rot, int64_t ld, int hd, int sign, cudaStream_t s);
void swiglu_fwd(const void *ab, void *u, DType dt, int64_t N, int64_t hp, cudaStream_t s);
void swiglu_bwd(const void *ab, const void *du, void *dab, DType dt, int64_t N, int64_t hp,
                cudaStream_t s);
void cross_entropy(void *logits, DType dt, const int32_t *tgt, float *rowloss, int64_t N, int V,
                   int64_t ldz, float inv_n, int *flag, cudaStream_t s);
void loss_reduce(const float *rowloss, int64_t N, float *loss, int *flag, cudaStream_t s);
void logits_out(const void *logits, DType dt, float *out, int64_t N, int V, int64_t ldz,
                cudaStream_t s);
// hyper: device [lr, wd, bc1, bc2], written by set_hyper.
void set_hyper(float *hyper, float lr, float wd, float bc1, float bc2, cudaStream_t s);
void adamw(float *p, const float *g, float *m, float *v, int64_t n, const float *hyper, float b1,
           float b2, float eps, const int *flag, cudaStream_t s);
// grad[r, c] (unpadded rows x cols) = sum over splits of part[s][r'][c'].
//   mode 0: identity; mode 1: W13 de-interleave (cols = 2h, part cols 2hp)
void wgrad_finish(const float *part, int splits, int64_t part_rows, int64_t ldp, float *grad,
                  int64_t rows, int64_t cols, int mode, int64_t h, cudaStream_t s);
// Deterministic embedding backward: dwte[v] = sum over i with tok_i = v of dx[i],
// summed in increasing i; rows without tokens are zero.
void embed_bwd(const int32_t *tok, const float *dx, float *dwte, int64_t N, int d, int V,
               int32_t *scratch, cudaStream_t s);
int64_t embed_bwd_scratch_ints(int64_t N, int V);
void init_params(float *p, int64_t n, uint64_t seed, uint64_t counter_base, float std,
                 int constant_one, cudaStream_t s);
// Global-norm clipping of g [n] (16-byte aligned) in place: part holds
// clip_part_blocks() doubles; *norm gets the norm before clipping, *scale the
// factor applied (max_norm / norm when norm > max_norm, else 1).
int clip_part_blocks();
// The same with the L-infinity norm (the largest |g|).
void clip_grads_inf(float *g, int64_t n, float max_norm, double *part, double *norm,
                    float *scale, cudaStream_t s);
// g [n] (16-byte aligned) *= sc in place.
void scale_grads(float *g, int64_t n, float sc, cudaStream_t s);
void clip_grads(float *g, int64_t n, float max_norm, double *part, double *norm, float *scale,
                cudaStream_t s);
// The norm of a gradient spread over ranks: g [n] *= sc in place, then the
// range's part -- sum of squares (L2) or largest |g| (linf), float64 -- is
// written to *out, or with accumulate added to it (L2) or maxed into it.
// part: clip_part_blocks() doubles of scratch.
void grad_norm_part(float *g, int64_t n, float sc, int linf, int accumulate, double *part,
                    double *out, cudaStream_t s);
// From the ranks' combined part *total: *norm (sqrt of it for L2), *scale
// (max_norm / norm when norm > max_norm, else 1), then g [n] *= scale.
void clip_from_total(float *g, int64_t n, const double *total, int linf, float max_norm,
                     double *norm, float *scale, cudaStream_t s);
// Dropout of [n] row-major elements of a site (element index = position):
//   drop_rows: x *= f in place;  drop_add: out = x + f y;
//   drop_to_act: out (operand type) = f dx.
void drop_rows(float *x, int64_t n, const DropArgs &a, cudaStream_t s);
void drop_add(const float *x, const float *y, float *out, int64_t n, const DropArgs &a,
              cudaStream_t s);
void drop_to_act(const float *dx, void *out, DType dt, int64_t n, const DropArgs &a,
                 cudaStream_t s);
void set_flag_zero(int *flag, cudaStream_t s);
void or_flag(const int *src, int *dst, cudaStream_t s);

// --------------------------------------------------------------- attention
// qkv [N, qkvw] (q heads | k heads | v heads, RoPE applied), o [N, H*hd],
// lse [B, H, T]; SIMT reference kernels for any head size.
// With drop.on, the probabilities are dropped (element ((b*H + h)*T + i)*T + j
// of the site): o uses P f, the backward uses the same f.
void attn_fwd_simt(const void *qkv, void *o, float *lse, DType dt, int B, int T, int H, int Hkv,
                   int hd, cudaStream_t s, DropArgs drop = DropArgs{});
// float32 tiled kernels (head size 32 or 64; false otherwise) and the
// one-warp-per-row kernels alone.
bool attn_fwd_f32_tiled(const float *qkv, float *o, float *lse, int B, int T, int H, int Hkv,
                        int hd, cudaStream_t s, DropArgs drop = DropArgs{});
bool attn_bwd_f32_tiled(const float *qkv, const float *o, const float *dout, const float *lse,
                        float *Dbuf, float *dqkv, int B, int T, int H, int Hkv, int hd,
                        cudaStream_t s, DropArgs drop = DropArgs{});
void attn_fwd_rows(const void *qkv, void *o, float *lse, DType dt, int B, int T, int H, int Hkv,
                   int hd, cudaStream_t s, DropArgs drop);
void attn_bwd_rows(const void *qkv, const void *o, const void *dout, const float *lse, float *Dbuf,
                   void *dqkv, DType dt, int B, int T, int H, int Hkv, int hd, cudaStream_t s,
                   DropArgs drop);
void attn_bwd_simt(const void *qkv, const void *o, const void *dout, const float *lse, float *Dbuf,
                   void *dqkv, DType dt, int B, int T, int H, int Hkv, int hd, cudaStream_t s,
                   DropArgs drop = DropArgs{});

// Tensor-core (mma.sync, bf16) kernels for head sizes 32 and 64.
bool attn_mma_covers(DType dt, int hd);
// drop: inverted dropout on the attention probabilities (the masks of the
// CUDA-core kernels, element ((b H + h) T + i) T + j); off by default.
void attn_fwd_mma(const void *qkv, void *o, float *lse, int B, int T, int H, int Hkv, int hd,
                  cudaStream_t s, DropArgs drop = DropArgs{});
// With cos_t/sin_t (RoPE tables [T, hd/2]) non-null, dq and dk are rotated
// back by -angle before they are stored.
void attn_bwd_mma(const void *qkv, const void *o, const void *dout, const float *lse, float *Dbuf,
                  void *dqkv, int B, int T, int H, int Hkv, int hd, const float *cos_t,
                  const float *sin_t, cudaStream_t s, DropArgs drop = DropArgs{});

// tcgen05 flash-attention forward (bf16, head size 64); false when it does not
// cover the arguments.  flag: device word for FLAG_TIMEOUT.
bool attn_tc_covers(DType dt, int hd, int T);
bool attn_fwd_tc(const void *qkv, void *o, float *lse, int B, int T, int H, int Hkv, int hd,
                 int *flag, cudaStream_t s);
// tcgen05 backward (dQ kernel, which also writes Dbuf, then dK/dV kernel);
// same arguments as attn_bwd_mma plus the time-out flag.  False (nothing
// launched) when it does not cover the arguments.
bool attn_bwd_tc(const void *qkv, const void *o, const void *dout, const float *lse, float *Dbuf,
                 void *dqkv, int B, int T, int H, int Hkv, int hd, const float *cos_t,
                 const float *sin_t, int *flag, cudaStream_t s);

// ------------------------------------------------------------------ decode
// Matrix-vector products of a decode step: y[b, n] = sum_k A[b, k] W[k, n]
// for B rows, W [K, ldw] in operand type.  A is either fp32 rows x [B, ldx]
// normalised on the fly (gain non-null: A = round(g * x * rstd), RMSNorm over
// the K = d entries of the row) or operand-type rows xa [B, ldxa].  The grid
// splits K into ks slices of kslice rows (gemv_plan); partial sums go to
// part [ks, B, N] and the last slice of each 128-column block to finish adds
// them in slice order (count [column blocks], zero between launches).
enum DecEpi {
  DEC_QKV = 0,     // RoPE on columns < rot_cols at position *pos, store out[b*ldo + *pos*pos_stride + n] (n < nvalid)
  DEC_RESID = 1,   // float out[b*ldo + n] += y (n < nvalid)
  DEC_SWIGLU = 2,  // interleaved a|b columns -> out[b*ldo + j] = silu(a_j) b_j (j < nvalid)
  DEC_LOGITS = 3   // float out[b*ldo + n] = y (n < nvalid)
};
struct GemvArgs {
  int B, K, N;
  const void *W;
  int64_t ldw;
  int vec;  // W rows may be read with 16-byte loads
  const float *x;
  int64_t ldx;
  const float *gain;
  float eps;
  const void *xa;
  int64_t ldxa;
  int ks, kslice;
  float *part;
  unsigned *count;
  int epi;
  void *out;
  int64_t ldo, pos_stride;
  int nvalid;
  const float *cos_t, *sin_t;
  const int *pos;
  int hd, rot_cols;
};
void gemv_plan(int64_t K, int64_t N, int *ks, int *kslice);
// The plan of a [K, N] product stays within the K slices the finishing
// block adds (K up to 16 slices of 1024 rows).
bool gemv_fits(int64_t K, int64_t N);
int gemv_col_blocks(int64_t N);
void gemv(const GemvArgs &a, DType dt, cudaStream_t s);
// Attention of the query at position *pos of every sequence against the
// cached keys/values 0..*pos of qkv [B*T, qkvw] (one layer), o [B, H*hd];
// part: B * H * attn_decode_chunks(T) * (hd + 2) floats; count: B * Hkv
// counters, zero between launches.  Needs 128 % hd == 0.
int attn_decode_chunks(int T);
void attn_decode(const void *qkv, int64_t qkvw, int B, int T, const int *pos, int H, int Hkv,
                 int hd, float *part, unsigned *count, void *o, DType dt, cudaStream_t s);
// One token id per row of logits [rows, ld] (V valid columns).
void sample_tokens(const float *logits, int64_t ld, int rows, int V, float temperature, int top_k,
                   const float *uni, int32_t *out, cudaStream_t s);
// The same with the repetition penalty (ids of hist [rows, hist_ld], first
// hist_len used; penalty != 1 needs V <= sample_ex_max_vocab_penalty()) and
// top-p inside the top-k set (top_p < 1 needs 1 <= top_k <= sample_ex_max_top_k()).
int sample_ex_max_top_k();
int64_t sample_ex_max_vocab_penalty();
void sample_tokens_ex(const float *logits, int64_t ld, int rows, int V, float temperature,
                      int top_k, float top_p, float penalty, const int32_t *hist,
                      int64_t hist_ld, int hist_len, const float *uni, int32_t *out,
                      cudaStream_t s);
void set_device_int(int *p, int v, cudaStream_t s);

// Opts `func` into `bytes` of dynamic shared memory on the current device.
// The attribute belongs to the device's context, so it is set once per
// (device, kernel), under a lock; false when the runtime refuses it.
bool smem_optin(const void *func, int bytes);
// Streaming multiprocessors of the current device (cached per device).
int device_sms();

// Launch counter (kernels enqueued by the current call).
extern thread_local int g_launches;
inline void count_launch(int n = 1) { g_launches += n; }

}  // namespace llm
