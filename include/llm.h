/*
 * llm.h -- C ABI of a B200 (sm_100a) library that runs one training step of a
 * bias-free, pre-norm Llama-style decoder: token embedding -> per layer
 * [RMSNorm -> causal MHA/GQA attention with RoPE on q,k -> residual -> RMSNorm
 * -> SwiGLU FFN -> residual] -> final RMSNorm -> untied lm_head -> softmax
 * cross-entropy, its hand-derived backward pass, and an AdamW update.
 *
 * Sources (page title, section):
 *   Hephaistos, "Architecture at a glance": the block, RMSNorm with cached
 *     rstd, RoPE on q/k, causal attention with a stable softmax, SwiGLU
 *     (silu(x W1) * x W3) W2 with hidden floor(8/3 d), untied lm_head, AdamW
 *     with decoupled weight decay and bias correction; dropout is fixed at 0.
 *   Hephaistos, "Design notes": parameters in one flat buffer described by
 *     (offset, len) per tensor; an activation arena cached for backward.
 *   strata, capability table: n_head and n_kv_head are independent (MHA, GQA,
 *     MQA); flash-style attention forward and backward with online softmax.
 *   randyGPT, "Training (Metal GPU path)": cross-entropy over all positions.
 *
 * Conventions for every call:
 *   - Pointers named d_* are DEVICE pointers owned by the caller (for example
 *     torch tensors passed by data_ptr()).  The library never frees them.
 *   - Parameters, gradients and Adam moments are flat, unpadded float32
 *     buffers of llm_param_layout()'s n_params elements, in its order:
 *     wte[V,d]; per layer g1[d], Wqkv[d, d+2*kvd], Wo[d,d], g2[d],
 *     W13[d, 2*d_ff] (W1 = columns [0,d_ff), W3 = columns [d_ff, 2*d_ff)),
 *     W2[d_ff, d]; then gf[d], Wlm[d, V].  Matrices are row-major [in, out],
 *     so every projection is x W.  kvd = n_kv_head * (d_model / n_head).
 *     In Wqkv the columns are all q heads, then all k heads, then all v heads;
 *     query head h uses kv head h / (n_head / n_kv_head).
 *   - Tokens and targets are int32 [batch, ctx], row-major.
 *   - All work is enqueued asynchronously on the stream given to llm_create;
 *     no call synchronises the host except llm_status().
 *   - One device per process: a context belongs to the CUDA device current
 *     when llm_create is called (its stream, workspace and every buffer
 *     passed to it are on that device), and every call on it must be made
 *     with that device current.  The first context (or llm_kernels.h entry)
 *     of a process fixes the process's device; creating a context, or calling
 *     a kernel entry, with another device current returns LLM_ERR_ARG, and so
 *     does a call on a context with another device current.  Run one process
 *     per GPU (torch.distributed) to use several.
 *   - Return codes are the LLM_* values below; no exception or abort ever
 *     crosses this boundary.  LLM_ERR_CONFIG and LLM_ERR_ARG are detected on
 *     the host before anything is launched.  LLM_ERR_TOKEN and
 *     LLM_ERR_NONFINITE are detected on the device and reported by
 *     llm_status(); a step that detects either leaves params, m and v
 *     unchanged.
 */
#ifndef LLM_H_
#define LLM_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  LLM_OK = 0,
  LLM_ERR_CONFIG = -1,    /* invalid configuration */
  LLM_ERR_ARG = -2,       /* null/misaligned pointer, workspace too small, bad size,
                             another device current (one device per process) */
  LLM_ERR_TOKEN = -3,     /* a token or target id outside [0, vocab) */
  LLM_ERR_NONFINITE = -4, /* the loss was not finite */
  LLM_ERR_CUDA = -5,      /* a CUDA runtime error */
  LLM_ERR_TIMEOUT = -6    /* a bounded device-side wait gave up */
};

enum { LLM_FP32 = 0, LLM_BF16 = 1 };

/* Model and optimiser configuration.  d_model must be divisible by n_head,
 * n_head by n_kv_head, and the head size d_model/n_head must be even (RoPE
 * rotates pairs (j, j + hd/2)).  compute = LLM_FP32 runs every matmul in
 * float32; LLM_BF16 runs matmuls and attention with bfloat16 operands and
 * float32 accumulation, keeping float32 master weights, Adam state and the
 * residual stream.  rope_base: RoPE base (10000); rms_eps: RMSNorm epsilon
 * added to the mean square (MicroGPT in Rust, "RMSNorm": 1e-5); beta1, beta2,
 * adam_eps: AdamW constants (eps is added outside the square root).
 * recompute = 1 keeps only each layer's input between the forward and the
 * backward and recomputes the layer's other activations from it in the
 * backward (the same kernels, so the gradients do not change); it cuts the
 * workspace by the saved activations of all but one layer at the cost of a
 * second forward of every layer, and llm_decode (whose cache is every layer's
 * saved q|k|v) returns LLM_ERR_CONFIG.  0 keeps them (the default). */
typedef struct {
  int32_t vocab, d_model, n_layer, n_head, n_kv_head, d_ff, ctx, batch;
  float rope_base, rms_eps, beta1, beta2, adam_eps;
  int32_t compute;
  int32_t recompute;
} llm_config;

/* One tensor of the flat parameter buffer: element (r, c) of a [rows, cols]
 * tensor sits at offset + r*cols + c.  name is NUL-terminated ("wte",
 * "l0.g1", "l0.Wqkv", ..., "gf", "Wlm"). */
typedef struct {
  char name[32];
  int64_t offset, rows, cols;
} llm_tensor_info;

typedef struct llm_ctx llm_ctx;

/* Hephaistos, "Design notes" (flat buffers, named offsets).  On input
 * *n_tensors is the capacity of out (ignored when out is NULL); on output it
 * is the number of tensors, and *n_params the total element count.  When out
 * is non-null and large enough it receives one entry per tensor in buffer
 * order (LLM_ERR_ARG if too small).  Host-only; LLM_ERR_CONFIG for an invalid
 * config. */
int llm_param_layout(const llm_config *cfg, llm_tensor_info *out, int *n_tensors,
                     int64_t *n_params);

/* Bytes of device workspace llm_create() needs for this config: saved
 * activations, logits, padded low-precision weight copies, the RoPE table and
 * scratch.  Host-only. */
int llm_workspace_bytes(const llm_config *cfg, int64_t *bytes);

/* Builds a context that carves its buffers out of d_workspace (caller-owned,
 * 256-byte aligned, at least llm_workspace_bytes() long, alive until
 * llm_destroy) and enqueues work on cuda_stream (a cudaStream_t; NULL = the
 * legacy default stream).  Enqueues a one-time RoPE table build.  The context
 * must be used from one host thread at a time. */
int llm_create(const llm_config *cfg, void *d_workspace, int64_t ws_bytes, void *cuda_stream,
               llm_ctx **out);

/* Releases host-side state (never the caller's buffers). NULL is ignored. */
void llm_destroy(llm_ctx *ctx);

/* Fills d_params with a fresh initialisation: every matrix ~ N(0, init_std)
 * drawn by a counter-based generator keyed by seed; when scale_out_proj != 0,
 * Wo and W2 use init_std / sqrt(2 n_layer) (randyGPT, Features: GPT-2 style
 * scaled output projections); RMSNorm gains are 1. */
int llm_init(llm_ctx *ctx, uint64_t seed, float init_std, int scale_out_proj, float *d_params);

/* Forward pass only: d_logits (float32 [batch, ctx, vocab]) = lm_head output
 * for d_tokens.  Leaves d_params untouched.  Out-of-range tokens are clamped
 * for the read and reported by llm_status() as LLM_ERR_TOKEN. */
int llm_forward(llm_ctx *ctx, const float *d_params, const int32_t *d_tokens, float *d_logits);

/* One training step on the pre-update parameters: loss = mean over all
 * batch*ctx positions of the cross-entropy of the logits against d_targets,
 * written to d_loss (one float32 on the device); d_grads is OVERWRITTEN with
 * d loss / d params; then AdamW updates d_params, d_m and d_v in place
 * (t = 1-based step count; lr and wd as in p -= lr*wd*p + lr*mhat/(sqrt(vhat)+eps)).
 * If the step sees an invalid token/target or a non-finite loss, params, m
 * and v are left untouched and llm_status() reports the error. */
int llm_step(llm_ctx *ctx, float *d_params, float *d_grads, float *d_m, float *d_v, int64_t t,
             const int32_t *d_tokens, const int32_t *d_targets, float lr, float wd,
             float *d_loss);

/* llm_step in two halves, for data parallelism with one process per GPU and
 * the batch split across ranks (each rank a context over its share):
 *   llm_grad:  the step's forward, loss and backward without the update:
 *              d_grads = d loss / d params and d_loss = the mean loss over
 *              this context's batch*ctx positions.
 *   llm_adamw: the step's update: d_grads *= grad_scale in place (1/ranks after
 *              a summing all-reduce turns the sum of the ranks' mean gradients
 *              into the mean over the whole batch), then clipping when
 *              llm_set_grad_clip is on (by the norm llm_set_grad_clip_mode
 *              selects), then AdamW as in llm_step.  It is
 *              skipped (params, m, v untouched) when the error word holds an
 *              error: the word the last llm_grad set, ORed with llm_flag_in.
 *   llm_flag_out copies that int32 error word (0 = none) to d_flag (device);
 *   llm_flag_in ORs d_flag into it, so ranks that all-reduce their words (MAX)
 *   skip or take the update together.
 * llm_grad then llm_adamw(grad_scale = 1) gives llm_step's results bit for
 * bit.  These run as individual launches (no graph).  LLM_ERR_ARG for null or
 * misaligned (16-byte) buffers, t < 1 or a non-finite grad_scale. */
int llm_grad(llm_ctx *ctx, const float *d_params, float *d_grads, const int32_t *d_tokens,
             const int32_t *d_targets, float *d_loss);
int llm_adamw(llm_ctx *ctx, float *d_params, float *d_grads, float *d_m, float *d_v, int64_t t,
              float lr, float wd, float grad_scale);
/* The update of llm_adamw over `count` consecutive elements for a sharded
 * optimiser (each rank updates its 1/ranks of the parameters after a
 * reduce-scatter of the gradient, then the ranks all-gather the parameters):
 * d_params, d_grads, d_m and d_v each point at the range's first element
 * (16-byte aligned); d_grads *= grad_scale, then AdamW with the context's
 * betas and eps, skipped on the error word like llm_adamw.  No clipping (the
 * global norm needs the whole gradient: llm_adamw_range_clip below).  LLM_ERR_ARG for misaligned
 * pointers, count < 0, t < 1 or a non-finite grad_scale. */
int llm_adamw_range(llm_ctx *ctx, float *d_params, float *d_grads, float *d_m, float *d_v,
                    int64_t count, int64_t t, float lr, float wd, float grad_scale);

/* Clipping for the sharded optimiser, where no rank holds the whole gradient
 * (MicroGPT in Rust, "Gradient Clipping"; Transformer-In-Rust, "Gradient
 * Clipping -- By global norm": the threshold applies to the norm of every
 * gradient element together).  Per step, on each rank:
 *   llm_grad_norm_part: d_grads[0, count) *= grad_scale in place (1/ranks, as
 *     llm_adamw_range's grad_scale), then the range's part of the norm is
 *     written to d_part (one float64 on the device, 8-byte aligned; with
 *     accumulate = 1 combined with the value already there): the sum of
 *     squares, in float64 and a fixed order, for the L2 norm, or the largest
 *     |g| for the L-infinity norm (llm_set_grad_clip_mode).  A rank whose
 *     share is several ranges calls it once per range, accumulating.
 *   the caller combines the ranks' parts: all-reduce SUM (L2) or MAX
 *     (L-infinity) of the float64;
 *   llm_adamw_range_clip: from the combined part d_total the norm (its square
 *     root for L2) and the scale of llm_set_grad_clip's rule (threshold /
 *     norm when the norm exceeds the threshold, else 1; a NaN norm gives 1),
 *     d_grads[0, count) *= scale, then AdamW over the range as
 *     llm_adamw_range does with grad_scale 1 (skipped on the error word).
 *     The norm is what llm_read_grad_norm returns afterwards.  With clipping
 *     off (threshold 0) d_total is not read (may be NULL) and nothing is
 *     clipped.  A rank with several ranges calls it once per range with the
 *     same d_total.
 * Every rank then applies the same scale, the one the whole-gradient
 * clipping of llm_adamw would apply to the same summed gradient (equal up to
 * the order of the float64 sum).  LLM_ERR_ARG for null or misaligned
 * buffers, count < 0, t < 1, accumulate not 0 or 1 or a non-finite
 * grad_scale. */
int llm_grad_norm_part(llm_ctx *ctx, float *d_grads, int64_t count, float grad_scale,
                       int accumulate, double *d_part);
int llm_adamw_range_clip(llm_ctx *ctx, float *d_params, float *d_grads, float *d_m, float *d_v,
                         int64_t count, int64_t t, float lr, float wd, const double *d_total);
int llm_flag_out(llm_ctx *ctx, int32_t *d_flag);
int llm_flag_in(llm_ctx *ctx, const int32_t *d_flag);

/* Gradient buckets, so that a data-parallel exchange of the gradient overlaps
 * the backward that produces it (one process per GPU; the exchange, e.g. an
 * NCCL all-reduce per bucket, runs on the caller's own stream).  The flat
 * gradient splits into n_layer + 2 contiguous buckets, numbered in the order
 * the backward finishes them: 0 = gf and Wlm (the end of the buffer), k = 1 ..
 * n_layer = layer n_layer - k, n_layer + 1 = wte (the start of the buffer).
 *   llm_grad_bucket_range (host only): offset and element count of bucket k
 *     in the flat buffer; LLM_ERR_CONFIG for an invalid config, LLM_ERR_ARG
 *     for k outside [0, n_layer + 1] or a null pointer.
 *   llm_set_grad_buckets: with enable = 1 every later llm_grad records one
 *     event per bucket on the context's stream once that bucket's gradients
 *     are final (nothing else changes: the gradients are bit-identical);
 *     0 turns it off (the default).  llm_step never records them.
 *   llm_grad_bucket_wait: makes `stream` (a cudaStream_t on the context's
 *     device) wait until bucket k of the most recent llm_grad is final.
 *     LLM_ERR_ARG for k out of range or when that llm_grad ran without
 *     buckets. */
int llm_grad_bucket_range(const llm_config *cfg, int k, int64_t *offset, int64_t *count);
int llm_set_grad_buckets(llm_ctx *ctx, int enable);
int llm_grad_bucket_wait(llm_ctx *ctx, int k, void *stream);

/* Single-token decode against a key/value cache (Hephaistos, feature list:
 * "True KV Cache", the prompt is processed once and every later position
 * costs one pass over a single row per sequence; strata, model table: the
 * cache holds keys already rotated by RoPE, and decoding position by position
 * gives the full forward's logits).
 *
 * The cache is the context's own saved q|k|v activations: llm_forward over
 * d_tokens [batch, ctx] fills positions 0..ctx-1 of every sequence (llm_step's
 * forward does too, but with dropout on it holds a training forward's
 * values); that forward over a prompt in positions 0..p-1 is the prefill
 * (positions >= p may hold any ids: causality keeps them out of positions
 * < p).  llm_decode then runs position pos for every sequence: d_tokens
 * [batch] holds each sequence's id at pos, the call writes that position's
 * rotated keys and values into the cache (so decoding pos, pos+1, ... in
 * order extends the sequences), and d_logits (float32 [batch, vocab]) gets
 * the logits of position pos, which attend to cached positions 0..pos.
 * d_params must be the parameters of that forward: the embedding and the
 * RMSNorm gains are read from it, the matrices from the low-precision copies
 * the forward made.  Requires 0 <= pos < ctx (LLM_ERR_ARG otherwise), and
 * head_dim dividing 128, d_ff at most 16384 and a context made without
 * recompute (LLM_ERR_CONFIG otherwise); nothing is launched on an error.  Out-of-range
 * ids are clamped for the read and reported by llm_status() as
 * LLM_ERR_TOKEN.  The position goes to device memory first, so the second call
 * in a row with the same (d_params, d_tokens, d_logits) captures the decode
 * body into a CUDA graph that later calls replay for any pos (graphs follow
 * llm_set_graphs).  Results are bit-reproducible. */
int llm_decode(llm_ctx *ctx, const float *d_params, const int32_t *d_tokens, int pos,
               float *d_logits);

/* Token sampling (Hephaistos, Sampling: temperature + top-k) for each of
 * n_rows rows of d_logits (float32, row stride ld >= vocab of the context):
 *   temperature <= 0 or top_k == 1: greedy, the largest logit (lowest id
 *     among equal maxima);
 *   otherwise the top-k set is the first top_k ids ordered by (logit
 *     descending, id ascending) -- the whole vocabulary when top_k <= 0 or
 *     top_k >= vocab -- with weights exp((z - max z) / temperature), and the
 *     token is the smallest id of the set, in increasing id order, whose
 *     cumulative weight exceeds u * (total weight), u = d_uniform[row]
 *     clamped to [0, 1).
 * The uniforms are inputs (device float32 [n_rows]); d_out gets int32
 * [n_rows] ids.  One block per row; deterministic. */
int llm_sample(llm_ctx *ctx, const float *d_logits, int64_t ld, int n_rows, float temperature,
               int top_k, const float *d_uniform, int32_t *d_out);

/* llm_sample with the rest of the sampling pipeline (Transformer-In-Rust,
 * Features: repetition penalty -> temperature -> top-k -> top-p -> random
 * sample; strata and randyGPT: top-p nucleus sampling).  First, when
 * repetition_penalty != 1, every id present among the first history_len
 * entries of the row's history (device int32, row b at d_history + b *
 * history_ld; entries outside [0, vocab) ignored) has its logit divided by
 * repetition_penalty when positive and multiplied by it otherwise (float32).
 * Then temperature and top-k as in llm_sample; then, when top_p < 1, only the
 * shortest prefix of the top-k set walked in (logit descending, id
 * ascending) order whose weight reaches top_p of the set's total is kept
 * (at least one id), and the draw is made from it as in llm_sample.
 * top_p = 1 and repetition_penalty = 1 give llm_sample's ids.  LLM_ERR_ARG
 * unless 0 < top_p <= 1 (top_p < 1 needs 1 <= top_k <= 1024),
 * repetition_penalty > 0 and finite, history_len >= 0, and with a penalty a
 * history, history_ld >= history_len and vocab <= 524288. */
int llm_sample_ex(llm_ctx *ctx, const float *d_logits, int64_t ld, int n_rows, float temperature,
                  int top_k, float top_p, float repetition_penalty, const int32_t *d_history,
                  int64_t history_ld, int history_len, const float *d_uniform, int32_t *d_out);

/* Learning-rate schedule (host only: needs no context and no GPU; the value
 * is passed to llm_step as lr).  Transformer-In-Rust, Features: cosine decay
 * with linear warmup, and cosine / linear / constant schedulers; randyGPT,
 * Training: constant at max_lr, then cosine decay to min_lr over the final
 * 40%; strata: cosine + warmup.  For 1-based step t:
 *   t <= warmup_steps (when > 0):  lr = max_lr * t / warmup_steps
 *   t <= decay_start:               lr = max_lr
 *   else, p = min(1, (t - decay_start) / (total_steps - decay_start)), or 1
 *   when total_steps <= decay_start:
 *     LLM_LR_COSINE:   min_lr + (max_lr - min_lr) * (1 + cos(pi p)) / 2
 *     LLM_LR_LINEAR:   max_lr + (min_lr - max_lr) * p
 *     LLM_LR_CONSTANT: max_lr
 * computed in double precision and rounded to float into *lr.  LLM_ERR_ARG
 * for a null pointer, t < 1, warmup_steps < 0, decay_start < warmup_steps, an
 * unknown shape or a non-finite rate. */
enum { LLM_LR_CONSTANT = 0, LLM_LR_COSINE = 1, LLM_LR_LINEAR = 2 };
typedef struct {
  float max_lr, min_lr;
  int64_t warmup_steps, decay_start, total_steps;
  int32_t shape;
} llm_lr_schedule;
int llm_lr_at(const llm_lr_schedule *sched, int64_t t, float *lr);

/* Learning-rate reduction on a plateau (host only; randyGPT, Training:
 * ReduceLROnPlateau halves max_lr on stagnation, up to 3 times, patience 30).
 * llm_plateau_init sets factor, patience, max_reductions and a relative
 * threshold and starts the scale at 1.  llm_plateau_update takes one
 * evaluation's metric (lower is better): a metric below best * (1 -
 * threshold) becomes the best and restarts the count; otherwise the count
 * grows, and once it exceeds patience the scale is multiplied by factor (at
 * most max_reductions times) and the count restarts.  *scale receives the
 * current scale, to multiply the schedule's rate by.  LLM_ERR_ARG for a null
 * pointer, factor outside (0, 1], a negative patience or max_reductions, a
 * threshold outside [0, 1) or a NaN metric. */
typedef struct {
  double best, threshold, scale;
  int64_t bad, patience;
  int32_t reductions, max_reductions;
  float factor;
} llm_plateau;
int llm_plateau_init(llm_plateau *pl, float factor, int64_t patience, int32_t max_reductions,
                     double threshold);
int llm_plateau_update(llm_plateau *pl, double metric, float *scale);

/* Global-norm gradient clipping inside llm_step (MicroGPT in Rust, Gradient
 * Clipping: when the gradient norm exceeds max_norm every gradient is scaled
 * by max_norm / norm; Transformer-In-Rust: clipping by global norm).  With
 * max_norm > 0, every later llm_step (and llm_adamw) computes the norm of the
 * whole gradient buffer -- Euclidean by default, from double-precision sums in
 * a fixed order, or the L-infinity norm (llm_set_grad_clip_mode) --, scales d_grads in
 * place by max_norm / norm when norm > max_norm, and AdamW then uses the
 * clipped gradient (d_grads holds it after the step).  max_norm <= 0 turns
 * clipping off (the default).  A change frees the captured step graph
 * (synchronising the stream first).  LLM_ERR_ARG for NaN. */
int llm_set_grad_clip(llm_ctx *ctx, float max_norm);

/* RoPE position interpolation (strata, RoPE row: context scaling folds
 * extended positions into the trained range): every later call rotates q and
 * k at position t by the angles (t / factor) * base^(-2j/hd) -- the forward,
 * the backward and decode alike (the context's one angle table is rebuilt,
 * on its stream).  factor = 1 is plain RoPE (the default); a model trained at
 * context L runs at context factor * L with its positions in [0, L).
 * LLM_ERR_ARG unless factor > 0 and finite. */
int llm_set_rope_scale(llm_ctx *ctx, float factor);

/* Inverted dropout in the training forward and backward of llm_step and
 * llm_grad (Hephaistos, Architecture at a glance: dropout on the embeddings,
 * the attention weights and the attention and MLP outputs; masks drawn by the
 * training forward and reused by its backward).  With 0 < p < 1 each element
 * of the embedding output [B*T, d], the attention probabilities [B, H, T, T],
 * and the attention and MLP branch outputs [B*T, d] (before their residual
 * adds) is kept with probability 1 - p and scaled by 1 / (1 - p).  The masks
 * come from Philox4x32-10 (Salmon et al., SC 2011), one call per group of
 * four consecutive elements: key = the seed's two 32-bit halves, counter =
 * (group index low word, high word, site + 4 * layer, n), group index =
 * element index / 4, with sites 0 embedding, 1 attention probabilities,
 * 2 attention output, 3 MLP output, element indices row-major over those
 * shapes of the whole batch (the context's sequences start at the offset of
 * llm_set_dropout_offset, 0 by default), n = the number of training calls (llm_step or llm_grad) since the
 * last llm_set_dropout; element e is kept when output word e mod 4 of its
 * group's call is >= floor(p * 2^32).  llm_forward and llm_decode never drop.
 * While dropout is on, bf16 attention with head size 32 or 64 runs in the
 * mma.sync kernels and fp32 attention with those head sizes in the tiled
 * CUDA-core kernels, both drawing the masks inside; other head sizes use the
 * one-warp-per-row kernels (the tcgen05 kernels draw no masks).  p = 0 turns
 * it off (the default).  A changed setting frees the
 * captured step graph; every call restarts n at 0.  LLM_ERR_ARG unless
 * 0 <= p < 1. */
int llm_set_dropout(llm_ctx *ctx, float p, uint64_t seed);

/* The mask counter n of llm_set_dropout: the number the next training call
 * draws its masks with.  Host only (no device work, no synchronisation).  A
 * run checkpointed by saving params, m, v, t and n, and resumed in a new
 * context with the same llm_set_dropout(p, seed) then llm_set_dropout_calls(n),
 * continues with the masks the uninterrupted run would have drawn.
 * LLM_ERR_ARG for a null pointer or n outside [0, 2^31). */
int llm_get_dropout_calls(llm_ctx *ctx, int64_t *n);
int llm_set_dropout_calls(llm_ctx *ctx, int64_t n);

/* The index b0 of the context's first sequence in the whole batch of a
 * data-parallel step (default 0).  The masks of llm_set_dropout are indexed
 * over the whole batch: the context's sequence b draws those of sequence
 * b0 + b, so ranks whose contexts hold consecutive shares of the batch
 * (b0 = rank * batch) draw together the masks of one context over the whole
 * batch, and no two ranks draw the same ones.  A changed offset frees the
 * captured step graph.  LLM_ERR_ARG for a null pointer, b0 outside
 * [0, 2^31), or a context whose device is not current. */
int llm_set_dropout_offset(llm_ctx *ctx, int64_t b0);

/* The norm clipping uses: LLM_CLIP_L2, the Euclidean norm of the whole
 * gradient (the default), or LLM_CLIP_LINF, its largest absolute element
 * (randyGPT, Training: gradient clipping by the L-infinity norm at 1.0); the
 * rule is the same, scale = max_norm / norm when norm > max_norm.  A change
 * frees the captured step graph.  LLM_ERR_ARG for another mode. */
enum { LLM_CLIP_L2 = 0, LLM_CLIP_LINF = 1 };
int llm_set_grad_clip_mode(llm_ctx *ctx, int mode);

/* Synchronises the context's stream and returns in *norm the gradient norm
 * (before clipping, in the selected norm) of the most recent llm_step or
 * llm_adamw run with clipping on; LLM_ERR_ARG if no such call has run on this
 * context. */
int llm_read_grad_norm(llm_ctx *ctx, double *norm);

/* Synchronises the context's stream and returns the errors that calls on
 * this context raised on the device since the previous llm_status() (then
 * clears them): LLM_ERR_TIMEOUT before LLM_ERR_TOKEN before LLM_ERR_NONFINITE
 * when several were raised; LLM_ERR_CUDA if the stream reports a CUDA error;
 * else LLM_OK.  An error word brought in by llm_flag_in is not reported here
 * (it only skips the update). */
int llm_status(llm_ctx *ctx);

/* A static, human-readable string for a return code. */
const char *llm_error_string(int code);

/* Number of kernels the most recent llm_step / llm_forward call enqueued
 * (for a replayed step graph: its kernel nodes plus the scalar write). */
int llm_last_launch_count(const llm_ctx *ctx);

/* Step graphs (default on).  llm_step writes the step's scalars (lr, wd and
 * the AdamW bias corrections of t) to device memory with one small kernel,
 * then runs the step body.  The second llm_step call in a row with the same
 * buffers (params, grads, m, v, tokens, targets, loss) captures the body
 * into a CUDA graph on the context's stream and launches it; later calls with
 * those buffers replay the graph (the buffers' contents may change freely
 * between calls).  No graph is used on the legacy default stream (stream 0),
 * while kernel timing is on (llm_set_kernel_timing), or after a capture
 * failed (the context then runs every step as individual launches).  enable = 0 turns replay off (and frees
 * the graph after synchronising the stream); enable = 1 turns it back on. */
int llm_set_graphs(llm_ctx *ctx, int enable);

/* Measurement hooks (strata, bench harness: time what is claimed).  With
 * timing enabled, the launches of later llm_step calls are bracketed by CUDA
 * events on the context's stream, per kernel class, and each bracket is
 * credited with its algorithmic work: FLOPs for the contractions (GEMM, on
 * tensor cores or, for float32 operands, CUDA cores: 2*M*N*K with unpadded
 * sizes; attention: the causal T(T+1)/2 (query, key)
 * pairs per (sequence, head) times 4 hd FLOPs forward, 8 hd backward), bytes
 * for the memory-bound passes (what the pass must read and write once:
 * RMSNorm forward 4 + ab bytes per element plus the rstd, backward the float32
 * input, upstream gradient, residual gradient (when added) and output plus
 * the activation-type copy; SwiGLU a, b, u (forward) and a, b, du, da, db
 * (backward) at ab bytes; cross-entropy the logits read and written once;
 * embedding gather 8 bytes per element read and written; embedding scatter
 * the upstream rows and the whole table; AdamW 28 bytes per parameter; the
 * weight copies 4 + ab bytes per weight; the split-K finish its partials and
 * outputs).  ab = bytes of an activation element (2 bf16, 4 fp32).
 * llm_read_kernel_class_timing() synchronises the stream and returns, for
 * class cls (LLM_KT_*), the summed device time in milliseconds, the credited
 * work and the number of brackets since the last reset;
 * llm_read_kernel_timing() does the same for LLM_KT_GEMM, then resets every
 * class.  Events are created on demand (two per bracket) and kept until
 * llm_destroy(); reading after every few steps bounds their number.  Steps
 * run as individual launches on the one stream while timing is on (no step
 * graph, no side stream).  LLM_ERR_ARG for a class out of range. */
enum {
  LLM_KT_GEMM = 0,           /* tcgen05 projection GEMMs (FLOPs) */
  LLM_KT_ATTN_FWD = 1,       /* attention forward (FLOPs) */
  LLM_KT_ATTN_BWD = 2,       /* attention backward (FLOPs) */
  LLM_KT_RMSNORM_FWD = 3,    /* bytes from here on */
  LLM_KT_RMSNORM_BWD = 4,    /* with the gain-gradient reduction */
  LLM_KT_SWIGLU_FWD = 5,
  LLM_KT_SWIGLU_BWD = 6,
  LLM_KT_CROSS_ENTROPY = 7,  /* with the loss reduction */
  LLM_KT_EMBED_FWD = 8,
  LLM_KT_EMBED_BWD = 9,
  LLM_KT_ADAMW = 10,
  LLM_KT_WEIGHT_CAST = 11,
  LLM_KT_WGRAD_FINISH = 12,
  LLM_KT_GEMM_CUDA_CORE = 13, /* float32 projection GEMMs on CUDA cores (FLOPs) */
  LLM_KT_GEMM_TF32 = 14,      /* float32 projection GEMMs on the tensor cores, split
                                 precision (3xTF32), with their operand split (FLOPs) */
  LLM_KT_CLASSES = 15
};
int llm_set_kernel_timing(llm_ctx *ctx, int enable);
int llm_read_kernel_timing(llm_ctx *ctx, double *ms, double *flops, int64_t *launches);
int llm_read_kernel_class_timing(llm_ctx *ctx, int cls, double *ms, double *work,
                                 int64_t *launches);

#ifdef __cplusplus
}
#endif

#endif /* LLM_H_ */
