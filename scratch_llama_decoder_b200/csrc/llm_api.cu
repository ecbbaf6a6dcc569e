// C ABI (include/llm.h) and host orchestration of one training step: the
// parameter layout, the carving of the caller's workspace, and the launch
// sequence forward -> cross-entropy -> backward -> AdamW on one stream.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>
#include <vector>

#include "../../include/llm.h"
#include "gemm_tc.h"
#include "internal.h"

using namespace llm;

namespace {

int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

// Sizes derived from a config.  hp / Vp: hidden and vocabulary padded to the
// tile multiples of the low-precision weight copies (pad weights are zero, so
// pad activations are zero and pad gradients are discarded).
struct Dims {
  int V, d, L, H, Hkv, hd, kvd, h, T, B;
  int64_t N, qkvw, hp, Vp, P, layer_sz;
  DType dt;
  int ab;  // bytes of one activation element
  bool rc;  // recompute: one slot of per-layer activations
  int LS;   // slots of per-layer activations (L, or 1 with recompute)
};

bool valid_config(const llm_config *c) {
  if (!c) return false;
  if (c->vocab < 1 || c->d_model < 4 || c->n_layer < 0 || c->n_head < 1 || c->n_kv_head < 1 ||
      c->d_ff < 1 || c->ctx < 1 || c->batch < 1)
    return false;
  if (c->d_model % c->n_head) return false;
  if (c->n_head % c->n_kv_head) return false;
  int hd = c->d_model / c->n_head;
  if (hd % 2 || hd > 128) return false;
  if (c->d_model % 4 || c->d_model > 4096) return false;
  if (c->compute != LLM_FP32 && c->compute != LLM_BF16) return false;
  if (c->recompute != 0 && c->recompute != 1) return false;
  if (!(c->rms_eps >= 0.f) || !(c->rope_base > 0.f)) return false;
  if ((int64_t)c->batch * c->ctx > (int64_t)1 << 30) return false;
  return true;
}

Dims make_dims(const llm_config *c) {
  Dims D;
  D.V = c->vocab; D.d = c->d_model; D.L = c->n_layer; D.H = c->n_head; D.Hkv = c->n_kv_head;
  D.hd = D.d / D.H; D.kvd = D.Hkv * D.hd; D.h = c->d_ff; D.T = c->ctx; D.B = c->batch;
  D.N = (int64_t)D.B * D.T;
  D.qkvw = D.d + 2LL * D.kvd;
  D.hp = round_up(D.h, 64);
  D.Vp = round_up(D.V, 128);
  D.layer_sz = (int64_t)D.d + (int64_t)D.d * D.qkvw + (int64_t)D.d * D.d + D.d +
               (int64_t)D.d * 2 * D.h + (int64_t)D.h * D.d;
  D.P = (int64_t)D.V * D.d + D.L * D.layer_sz + D.d + (int64_t)D.d * D.V;
  D.dt = c->compute == LLM_BF16 ? DT_BF16 : DT_F32;
  D.ab = D.dt == DT_BF16 ? 2 : 4;
  D.rc = c->recompute != 0;
  D.LS = D.rc ? std::min(1, D.L) : D.L;
  return D;
}

// Offsets of the flat parameter buffer (Hephaistos, Design notes).
struct POff {
  const Dims &D;
  int64_t layer(int l) const { return (int64_t)D.V * D.d + l * D.layer_sz; }
  int64_t g1(int l) const { return layer(l); }
  int64_t wqkv(int l) const { return g1(l) + D.d; }
  int64_t wo(int l) const { return wqkv(l) + (int64_t)D.d * D.qkvw; }
  int64_t g2(int l) const { return wo(l) + (int64_t)D.d * D.d; }
  int64_t w13(int l) const { return g2(l) + D.d; }
  int64_t w2(int l) const { return w13(l) + (int64_t)D.d * 2 * D.h; }
  int64_t gf() const { return layer(D.L); }
  int64_t wlm() const { return gf() + D.d; }
};

// Split count of a weight-gradient GEMM (K = tokens).  The GEMM runs
// (128 x 256 tile, split) items on 148 SMs in whole waves, so the split count
// minimises an estimate of waves x k-blocks per item (520 cycles per block of
// 64 at the tensor rate, 1.9 GHz) plus the partial sums' extra HBM traffic
// (written by the GEMM, read by the finish pass, 6.5 TB/s); every split keeps
// at least 8 k-blocks, at most 32 splits.
// With CTA pairs (pairs = true) an item is a 256 x 256 tile on two SMs, so
// 74 items run at once and each takes the same time per k-block.
int wgrad_splits(const Dims &D, int64_t M, int64_t Ncols, bool pairs = false) {
  const int64_t tiles = pairs ? ((M + 255) / 256) * ((Ncols + 255) / 256)
                              : ((M + 127) / 128) * ((Ncols + 255) / 256);
  const int64_t units = pairs ? 74 : 148;
  const int64_t kb = (D.N + 63) / 64;
  int best = 1;
  double best_us = 1e300;
  for (int s = 1; s <= 32; s++) {
    const int64_t kbs = (kb + s - 1) / s;
    if (s > 1 && kbs < 8) break;
    const double waves = (double)((tiles * s + units - 1) / units);
    const double us = waves * (double)kbs * 520.0 / 1900.0 +
                      2.0 * s * (double)M * (double)Ncols * 4.0 / 6.5e6;
    if (us < best_us * (1.0 - 1e-9)) {
      best_us = us;
      best = s;
    }
  }
  return best;
}

// Workspace carve: the same sequence of (size) requests both sizes and
// places the buffers, so llm_workspace_bytes and llm_create agree.
struct Carver {
  char *base;
  int64_t off = 0;
  void *take(int64_t bytes) {
    off = round_up(off, 256);
    void *p = base ? base + off : nullptr;
    off += bytes;
    return p;
  }
};

}  // namespace

struct llm_ctx {
  llm_config cfg;
  Dims D;
  int dev = -1;  // the device current at llm_create
  cudaStream_t s;
  // weight-gradient GEMMs run on a side stream s2 (forked from / joined to s
  // with events); cur is the stream the GEMM launchers use
  cudaStream_t s2 = nullptr, cur = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  int last_launches = 0;
  bool use_tc = false;
  // device buffers (all inside the caller's workspace)
  int *flag_step, *flag_sticky;
  float *cos_t, *sin_t;
  void *w_qkv, *w_o, *w_13, *w_2, *w_lm;  // low-precision copies, layer-strided
  float *xs;                               // [L+1][N,d] residual stream
  float *x1;                               // [L][N,d]
  void *xn1, *qkv, *o, *xn2, *ab, *u;      // [L][...] saved activations
  float *rstd1, *rstd2, *lse;              // [L][N], [L][N], [L][B,H,T]
  void *xf, *logits;
  float *rstdf, *rowloss;
  float *dx, *dtmp, *Dbuf, *part, *dgpart;
  // float32 configurations: split-precision operand copies of the tensor-core
  // GEMM, one region per stream (the side stream's weight gradients run
  // concurrently with the main stream's GEMMs)
  float *tf32_scratch[2] = {nullptr, nullptr};
  int64_t tf32_floats = 0;
  void *dxA, *du, *dab, *dO, *dqkv;
  int32_t *sort_scratch;
  TcPlan *tc = nullptr;
  float *hyper;  // device [lr, wd, bc1, bc2] of the current step
  // optional event timing of the step's launches by kernel class
  // (llm_set_kernel_timing): event pairs in order, the class of each pair,
  // and per class the algorithmic work credited (FLOPs or bytes)
  bool timing = false;
  std::vector<cudaEvent_t> ev_pool;
  std::vector<int> ev_class;  // class of pair k (events 2k, 2k + 1)
  size_t ev_used = 0;
  double pending_work[LLM_KT_CLASSES] = {};
  int64_t pending_count[LLM_KT_CLASSES] = {};
  // step graph: captured on the second llm_step with the same buffers,
  // replayed afterwards; steps with kernel timing on run as launches
  bool graphs = true;  // replay allowed (off after any capture failure)
  cudaGraphExec_t gexec = nullptr;
  struct Key {
    const void *p[7];
    bool operator==(const Key &o) const {
      for (int i = 0; i < 7; i++)
        if (p[i] != o.p[i]) return false;
      return true;
    }
  } gkey{}, prev_key{};
  bool have_prev = false;
  int graph_launches = 0;  // kernels per replay
  // decode (llm_decode): per-call rows, split-K partials, attention chunk
  // records, column-block counters, the position word, and its own graph
  float *dec_x = nullptr, *dec_part = nullptr, *dec_attn = nullptr;
  void *dec_o = nullptr, *dec_u = nullptr;
  unsigned *dec_count = nullptr, *dec_acount = nullptr;
  int *dec_pos = nullptr;
  cudaGraphExec_t dexec = nullptr;
  Key dkey{}, dprev_key{};
  bool dhave_prev = false;
  int dgraph_launches = 0;
  // dropout (llm_set_dropout): rate, seed, training calls so far, and the
  // device word holding the current call's number
  float drop_p = 0.f;
  uint64_t drop_seed = 0;
  int64_t train_calls = 0;
  int *drop_step = nullptr;
  int64_t drop_b0 = 0;  // llm_set_dropout_offset: first sequence's index in the whole batch
  // gradient buckets (llm_set_grad_buckets): one event per bucket, recorded by
  // llm_grad's backward on the main stream once the bucket's gradients are final
  std::vector<cudaEvent_t> ev_bucket;
  bool buckets_on = false, buckets_recorded = false;
  // gradient clipping (llm_set_grad_clip): threshold, block sums, norm, scale
  float clip = 0.f;
  int clip_mode = 0;  // LLM_CLIP_L2 or LLM_CLIP_LINF
  bool have_norm = false;
  double *clip_part = nullptr, *clip_norm = nullptr;
  float *clip_scale = nullptr;
  int64_t carve(char *base);
};

int64_t llm_ctx::carve(char *base) {
  const Dims &D_ = D;
  Carver c{base};
  int64_t N = D_.N, d = D_.d, L = D_.L, ab = D_.ab;
  flag_step = (int *)c.take(64);
  flag_sticky = (int *)c.take(64);
  hyper = (float *)c.take(64);
  cos_t = (float *)c.take(4 * (int64_t)D_.T * (D_.hd / 2));
  sin_t = (float *)c.take(4 * (int64_t)D_.T * (D_.hd / 2));
  w_qkv = c.take(ab * L * d * D_.qkvw);
  w_o = c.take(ab * L * d * d);
  w_13 = c.take(ab * L * d * 2 * D_.hp);
  w_2 = c.take(ab * L * D_.hp * d);
  w_lm = c.take(ab * d * D_.Vp);
  xs = (float *)c.take(4 * (L + 1) * N * d);
  const int64_t LS = D_.LS;  // per-layer activation slots
  x1 = (float *)c.take(4 * LS * N * d);
  xn1 = c.take(ab * LS * N * d);
  qkv = c.take(ab * LS * N * D_.qkvw);
  o = c.take(ab * LS * N * d);
  xn2 = c.take(ab * LS * N * d);
  this->ab = c.take(ab * LS * N * 2 * D_.hp);
  u = c.take(ab * LS * N * D_.hp);
  rstd1 = (float *)c.take(4 * LS * N);
  rstd2 = (float *)c.take(4 * LS * N);
  lse = (float *)c.take(4 * LS * N * D_.H);
  xf = c.take(ab * N * d);
  logits = c.take(ab * N * D_.Vp);
  rstdf = (float *)c.take(4 * N);
  rowloss = (float *)c.take(4 * N);
  dx = (float *)c.take(4 * N * d);
  dtmp = (float *)c.take(4 * N * d);
  Dbuf = (float *)c.take(4 * N * D_.H);
  dxA = c.take(ab * N * d);
  du = c.take(ab * N * D_.hp);
  dab = c.take(ab * N * 2 * D_.hp);
  dO = c.take(ab * N * d);
  dqkv = c.take(ab * N * D_.qkvw);
  int64_t part_elems = 0;
  auto need = [&](int64_t M, int64_t Nc) {
    // room for the split count of either kernel (single CTAs or CTA pairs)
    const int64_t sp = std::max(wgrad_splits(D_, M, Nc, false), wgrad_splits(D_, M, Nc, true));
    part_elems = std::max<int64_t>(part_elems, sp * M * Nc);
  };
  need(d, D_.Vp); need(D_.hp, d); need(d, 2 * D_.hp); need(d, d); need(d, D_.qkvw);
  part = (float *)c.take(4 * part_elems);
  if (D_.dt == DT_F32) {
    // every GEMM of the step: forward (M = tokens), data gradients, weight
    // gradients (K = tokens)
    int64_t tf = 0;
    auto tneed = [&](int64_t M, int64_t Nn, int64_t K) {
      tf = std::max<int64_t>(tf, gemm_tf32_scratch_floats(M, Nn, K));
    };
    tneed(N, D_.qkvw, d); tneed(N, d, d); tneed(N, 2 * D_.hp, d); tneed(N, d, D_.hp);
    tneed(N, D_.Vp, d); tneed(N, d, D_.Vp); tneed(N, D_.hp, d); tneed(N, d, 2 * D_.hp);
    tneed(N, d, D_.qkvw);
    tneed(d, D_.Vp, N); tneed(D_.hp, d, N); tneed(d, 2 * D_.hp, N); tneed(d, d, N);
    tneed(d, D_.qkvw, N);
    tf32_floats = tf;
    tf32_scratch[0] = (float *)c.take(4 * tf);
    tf32_scratch[1] = (float *)c.take(4 * tf);
  }
  dgpart = (float *)c.take(4 * (int64_t)rmsnorm_bwd_blocks(N) * d);
  sort_scratch = (int32_t *)c.take(4 * embed_bwd_scratch_ints(N, D_.V));
  // decode: the four matrix-vector shapes of a layer and the lm_head
  const int64_t B = D_.B;
  int64_t dpart = 0, dblocks = 0;
  auto dneed = [&](int64_t K, int64_t Nc) {
    int ks, sl;
    gemv_plan(K, Nc, &ks, &sl);
    if (ks > 1) dpart = std::max<int64_t>(dpart, (int64_t)ks * B * Nc);
    dblocks = std::max<int64_t>(dblocks, gemv_col_blocks(Nc));
  };
  dneed(d, D_.qkvw); dneed(d, d); dneed(d, 2 * D_.hp); dneed(D_.hp, d); dneed(d, D_.Vp);
  dec_x = (float *)c.take(4 * B * d);
  dec_o = c.take(ab * B * d);
  dec_u = c.take(ab * B * D_.hp);
  dec_part = (float *)c.take(4 * std::max<int64_t>(1, dpart));
  dec_attn = (float *)c.take(4 * B * D_.H * attn_decode_chunks(D_.T) * (int64_t)(D_.hd + 2));
  dec_count = (unsigned *)c.take(4 * dblocks);
  dec_acount = (unsigned *)c.take(4 * B * D_.Hkv);
  dec_pos = (int *)c.take(64);
  drop_step = (int *)c.take(64);
  clip_part = (double *)c.take(8 * (int64_t)clip_part_blocks());
  clip_norm = (double *)c.take(64);
  clip_scale = (float *)c.take(64);
  return round_up(c.off, 256);
}

// ------------------------------------------------------------- C ABI: host
extern "C" {

int llm_param_layout(const llm_config *cfg, llm_tensor_info *out, int *n_tensors,
                     int64_t *n_params) {
  if (!n_tensors || !n_params) return LLM_ERR_ARG;
  if (!valid_config(cfg)) return LLM_ERR_CONFIG;
  Dims D = make_dims(cfg);
  POff O{D};
  int cap = *n_tensors;
  int n = 3 + 6 * D.L;
  *n_tensors = n;
  *n_params = D.P;
  if (!out) return LLM_OK;
  if (cap < n) return LLM_ERR_ARG;
  int k = 0;
  auto put = [&](const char *nm, int64_t off, int64_t r, int64_t c) {
    memset(out[k].name, 0, sizeof(out[k].name));
    strncpy(out[k].name, nm, sizeof(out[k].name) - 1);
    out[k].offset = off; out[k].rows = r; out[k].cols = c;
    k++;
  };
  char nm[32];
  put("wte", 0, D.V, D.d);
  for (int l = 0; l < D.L; l++) {
    snprintf(nm, sizeof nm, "l%d.g1", l);   put(nm, O.g1(l), 1, D.d);
    snprintf(nm, sizeof nm, "l%d.Wqkv", l); put(nm, O.wqkv(l), D.d, D.qkvw);
    snprintf(nm, sizeof nm, "l%d.Wo", l);   put(nm, O.wo(l), D.d, D.d);
    snprintf(nm, sizeof nm, "l%d.g2", l);   put(nm, O.g2(l), 1, D.d);
    snprintf(nm, sizeof nm, "l%d.W13", l);  put(nm, O.w13(l), D.d, 2LL * D.h);
    snprintf(nm, sizeof nm, "l%d.W2", l);   put(nm, O.w2(l), D.h, D.d);
  }
  put("gf", O.gf(), 1, D.d);
  put("Wlm", O.wlm(), D.d, D.V);
  return LLM_OK;
}

int llm_workspace_bytes(const llm_config *cfg, int64_t *bytes) {
  if (!bytes) return LLM_ERR_ARG;
  if (!valid_config(cfg)) return LLM_ERR_CONFIG;
  llm_ctx tmp;
  tmp.cfg = *cfg;
  tmp.D = make_dims(cfg);
  *bytes = tmp.carve(nullptr);
  return LLM_OK;
}

// Every context and kernel entry of a process runs on one device (the
// kernels opt in to their shared-memory sizes once per process): the first
// call that needs a device fixes it, later calls with another device current
// are refused.
static std::atomic<int> g_device{-1};
static bool claim_device(int *dev) {
  int d = -1;
  if (cudaGetDevice(&d) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  int first = -1;
  if (!g_device.compare_exchange_strong(first, d) && first != d) return false;
  if (dev) *dev = d;
  return true;
}
// The context's device is the current one.
static bool on_device(const llm_ctx *c) {
  int d = -1;
  return cudaGetDevice(&d) == cudaSuccess && d == c->dev;
}

int llm_create(const llm_config *cfg, void *d_workspace, int64_t ws_bytes, void *cuda_stream,
               llm_ctx **out) {
  if (!out) return LLM_ERR_ARG;
  *out = nullptr;
  if (!valid_config(cfg)) return LLM_ERR_CONFIG;
  if (!d_workspace || ((uintptr_t)d_workspace & 255)) return LLM_ERR_ARG;
  llm_ctx *c = new (std::nothrow) llm_ctx();
  if (!c) return LLM_ERR_ARG;
  c->cfg = *cfg;
  c->D = make_dims(cfg);
  if (ws_bytes < c->carve(nullptr) || !claim_device(&c->dev)) { delete c; return LLM_ERR_ARG; }
  c->s = (cudaStream_t)cuda_stream;
  c->cur = c->s;
  if (cudaStreamCreateWithFlags(&c->s2, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&c->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&c->ev_join, cudaEventDisableTiming) != cudaSuccess) {
    // no side stream: every launch stays on the caller's stream
    (void)cudaGetLastError();
    c->s2 = nullptr;
  }
  c->carve((char *)d_workspace);
  g_launches = 0;
  cudaMemsetAsync(c->flag_step, 0, 64, c->s);
  cudaMemsetAsync(c->flag_sticky, 0, 64, c->s);
  cudaMemsetAsync(c->dec_count, 0, 4 * (size_t)gemv_col_blocks(std::max<int64_t>(
                                           std::max<int64_t>(c->D.qkvw, 2 * c->D.hp),
                                           std::max<int64_t>(c->D.d, c->D.Vp))),
                  c->s);
  cudaMemsetAsync(c->dec_acount, 0, 4 * (size_t)c->D.B * c->D.Hkv, c->s);
  cudaMemsetAsync(c->dec_pos, 0, 64, c->s);
  cudaMemsetAsync(c->drop_step, 0, 64, c->s);
  rope_table(c->cos_t, c->sin_t, c->D.T, c->D.hd, cfg->rope_base, c->s);
  c->tc = tc_plan_create(c->D.dt, c->cos_t, c->sin_t, c->D.T, c->D.hd, c->D.d + c->D.kvd, c->D.hp);
  tc_plan_set_flag(c->tc, c->flag_step);
  if (cudaGetLastError() != cudaSuccess) { delete c; return LLM_ERR_CUDA; }
  *out = c;
  return LLM_OK;
}

void llm_destroy(llm_ctx *c) {
  if (!c) return;
  if (c->s2) {
    cudaStreamSynchronize(c->s2);
    cudaStreamDestroy(c->s2);
  }
  if (c->ev_fork) cudaEventDestroy(c->ev_fork);
  if (c->ev_join) cudaEventDestroy(c->ev_join);
  if (c->gexec) cudaGraphExecDestroy(c->gexec);
  if (c->dexec) cudaGraphExecDestroy(c->dexec);
  for (cudaEvent_t e : c->ev_pool) cudaEventDestroy(e);
  for (cudaEvent_t e : c->ev_bucket) cudaEventDestroy(e);
  tc_plan_destroy(c->tc);
  delete c;
}

const char *llm_error_string(int code) {
  switch (code) {
    case LLM_OK: return "ok";
    case LLM_ERR_CONFIG: return "invalid configuration";
    case LLM_ERR_ARG: return "invalid argument (null or misaligned pointer, small workspace)";
    case LLM_ERR_TOKEN: return "token or target id outside [0, vocab)";
    case LLM_ERR_NONFINITE: return "non-finite loss";
    case LLM_ERR_CUDA: return "CUDA error";
    case LLM_ERR_TIMEOUT: return "a bounded device-side wait gave up";
    default: return "unknown error";
  }
}

int llm_last_launch_count(const llm_ctx *c) { return c ? c->last_launches : 0; }

int llm_set_kernel_timing(llm_ctx *c, int enable) {
  if (!c) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  c->timing = enable != 0;
  return LLM_OK;
}

int llm_set_graphs(llm_ctx *c, int enable) {
  if (!c) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  c->graphs = enable != 0;
  if (!c->graphs && (c->gexec || c->dexec)) {
    if (cudaStreamSynchronize(c->s) != cudaSuccess) return LLM_ERR_CUDA;
    if (c->gexec) cudaGraphExecDestroy(c->gexec);
    if (c->dexec) cudaGraphExecDestroy(c->dexec);
    c->gexec = nullptr;
    c->dexec = nullptr;
  }
  c->have_prev = false;
  c->dhave_prev = false;
  return LLM_OK;
}

int llm_set_grad_clip(llm_ctx *c, float max_norm) {
  if (!c || max_norm != max_norm) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  const float v = max_norm > 0.f ? max_norm : 0.f;
  if (v != c->clip) {
    // the threshold is baked into a captured step: drop the graph
    if (c->gexec) {
      if (cudaStreamSynchronize(c->s) != cudaSuccess) return LLM_ERR_CUDA;
      cudaGraphExecDestroy(c->gexec);
      c->gexec = nullptr;
    }
    c->have_prev = false;
    c->clip = v;
  }
  return LLM_OK;
}

int llm_set_rope_scale(llm_ctx *c, float factor) {
  if (!c || !(factor > 0.f) || !std::isfinite(factor)) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  g_launches = 0;
  rope_table(c->cos_t, c->sin_t, c->D.T, c->D.hd, c->cfg.rope_base, c->s, (double)factor);
  c->last_launches = g_launches;
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}

int llm_set_dropout(llm_ctx *c, float p, uint64_t seed) {
  if (!c || !(p >= 0.f) || !(p < 1.f)) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  if (p != c->drop_p || seed != c->drop_seed) {
    // the rate is baked into a captured step: drop the graph
    if (c->gexec) {
      if (cudaStreamSynchronize(c->s) != cudaSuccess) return LLM_ERR_CUDA;
      cudaGraphExecDestroy(c->gexec);
      c->gexec = nullptr;
    }
    c->have_prev = false;
    c->drop_p = p;
    c->drop_seed = seed;
  }
  c->train_calls = 0;
  return LLM_OK;
}

int llm_get_dropout_calls(llm_ctx *c, int64_t *n) {
  if (!c || !n) return LLM_ERR_ARG;
  *n = c->train_calls;
  return LLM_OK;
}

int llm_set_dropout_calls(llm_ctx *c, int64_t n) {
  if (!c || n < 0 || n > INT32_MAX) return LLM_ERR_ARG;
  c->train_calls = n;
  return LLM_OK;
}

int llm_set_dropout_offset(llm_ctx *c, int64_t b0) {
  if (!c || b0 < 0 || b0 > INT32_MAX) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  if (b0 != c->drop_b0) {
    // the offsets are baked into a captured step: drop the graph
    if (c->gexec) {
      if (cudaStreamSynchronize(c->s) != cudaSuccess) return LLM_ERR_CUDA;
      cudaGraphExecDestroy(c->gexec);
      c->gexec = nullptr;
    }
    c->have_prev = false;
    c->drop_b0 = b0;
  }
  return LLM_OK;
}

int llm_set_grad_clip_mode(llm_ctx *c, int mode) {
  if (!c || (mode != LLM_CLIP_L2 && mode != LLM_CLIP_LINF)) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  if (mode != c->clip_mode) {
    // the norm is part of a captured step: drop the graph
    if (c->gexec) {
      if (cudaStreamSynchronize(c->s) != cudaSuccess) return LLM_ERR_CUDA;
      cudaGraphExecDestroy(c->gexec);
      c->gexec = nullptr;
    }
    c->have_prev = false;
    c->clip_mode = mode;
  }
  return LLM_OK;
}

int llm_read_grad_norm(llm_ctx *c, double *norm) {
  if (!c || !norm || !c->have_norm) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  if (cudaStreamSynchronize(c->s) != cudaSuccess) return LLM_ERR_CUDA;
  if (cudaMemcpy(norm, c->clip_norm, sizeof(double), cudaMemcpyDeviceToHost) != cudaSuccess)
    return LLM_ERR_CUDA;
  return LLM_OK;
}

int llm_lr_at(const llm_lr_schedule *sc, int64_t t, float *lr) {
  if (!sc || !lr || t < 1 || sc->warmup_steps < 0 || sc->decay_start < sc->warmup_steps)
    return LLM_ERR_ARG;
  if (sc->shape != LLM_LR_CONSTANT && sc->shape != LLM_LR_COSINE && sc->shape != LLM_LR_LINEAR)
    return LLM_ERR_ARG;
  if (!std::isfinite(sc->max_lr) || !std::isfinite(sc->min_lr)) return LLM_ERR_ARG;
  const double mx = sc->max_lr, mn = sc->min_lr;
  double v;
  if (sc->warmup_steps > 0 && t <= sc->warmup_steps) {
    v = mx * (double)t / (double)sc->warmup_steps;
  } else if (t <= sc->decay_start || sc->shape == LLM_LR_CONSTANT) {
    v = mx;
  } else {
    double p = 1.0;
    if (sc->total_steps > sc->decay_start)
      p = std::min(1.0, (double)(t - sc->decay_start) /
                            (double)(sc->total_steps - sc->decay_start));
    v = sc->shape == LLM_LR_COSINE ? mn + (mx - mn) * (1.0 + cos(M_PI * p)) / 2.0
                                   : mx + (mn - mx) * p;
  }
  *lr = (float)v;
  return LLM_OK;
}

int llm_plateau_init(llm_plateau *pl, float factor, int64_t patience, int32_t max_reductions,
                     double threshold) {
  if (!pl || !(factor > 0.f) || !(factor <= 1.f) || patience < 0 || max_reductions < 0 ||
      !(threshold >= 0.0) || !(threshold < 1.0))
    return LLM_ERR_ARG;
  pl->best = INFINITY;
  pl->threshold = threshold;
  pl->scale = 1.0;
  pl->bad = 0;
  pl->patience = patience;
  pl->reductions = 0;
  pl->max_reductions = max_reductions;
  pl->factor = factor;
  return LLM_OK;
}

int llm_plateau_update(llm_plateau *pl, double metric, float *scale) {
  if (!pl || !scale || metric != metric) return LLM_ERR_ARG;
  if (metric < pl->best * (1.0 - pl->threshold)) {
    pl->best = metric;
    pl->bad = 0;
  } else if (++pl->bad > pl->patience && pl->reductions < pl->max_reductions) {
    pl->reductions++;
    pl->scale *= (double)pl->factor;
    pl->bad = 0;
  }
  *scale = (float)pl->scale;
  return LLM_OK;
}

int llm_read_kernel_class_timing(llm_ctx *c, int cls, double *ms, double *work,
                                 int64_t *launches) {
  if (!c || !ms || !work || !launches || cls < 0 || cls >= LLM_KT_CLASSES) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  if (cudaStreamSynchronize(c->s) != cudaSuccess) return LLM_ERR_CUDA;
  double total = 0.0;
  for (size_t i = 0; i + 1 < c->ev_used; i += 2) {
    if (c->ev_class[i / 2] != cls) continue;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, c->ev_pool[i], c->ev_pool[i + 1]) != cudaSuccess)
      return LLM_ERR_CUDA;
    total += t;
  }
  *ms = total;
  *work = c->pending_work[cls];
  *launches = c->pending_count[cls];
  return LLM_OK;
}

int llm_read_kernel_timing(llm_ctx *c, double *ms, double *flops, int64_t *launches) {
  if (!c || !ms || !flops || !launches) return LLM_ERR_ARG;
  const int rc = llm_read_kernel_class_timing(c, LLM_KT_GEMM, ms, flops, launches);
  if (rc != LLM_OK) return rc;
  c->ev_used = 0;
  for (int k = 0; k < LLM_KT_CLASSES; k++) {
    c->pending_work[k] = 0.0;
    c->pending_count[k] = 0;
  }
  return LLM_OK;
}

int llm_status(llm_ctx *c) {
  if (!c) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  if (cudaStreamSynchronize(c->s) != cudaSuccess) return LLM_ERR_CUDA;
  int f = 0;
  if (cudaMemcpy(&f, c->flag_sticky, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return LLM_ERR_CUDA;
  // cleared on the context's stream, so it lands before any later call's work
  if (cudaMemsetAsync(c->flag_sticky, 0, sizeof(int), c->s) != cudaSuccess) return LLM_ERR_CUDA;
  if (f & FLAG_TIMEOUT) return LLM_ERR_TIMEOUT;
  if (f & FLAG_TOKEN) return LLM_ERR_TOKEN;
  if (f & FLAG_NONFINITE) return LLM_ERR_NONFINITE;
  return LLM_OK;
}

}  // extern "C"

// ------------------------------------------------------- step orchestration
namespace {

bool aligned16(const void *p) { return p && ((uintptr_t)p & 15) == 0; }

// With kernel timing on, brackets the launches of its scope with CUDA events
// on the context's current stream and credits them to a kernel class with
// their algorithmic work (FLOPs or bytes); drop() takes back a scope that
// launched nothing.
struct KTimer {
  llm_ctx *c;
  int cls;
  double work;
  cudaEvent_t e1 = nullptr;
  KTimer(llm_ctx *c_, int cls_, double work_) : c(c_), cls(cls_), work(work_) {
    if (!c->timing) return;
    while (c->ev_pool.size() < c->ev_used + 2) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) return;
      c->ev_pool.push_back(e);
    }
    cudaEventRecord(c->ev_pool[c->ev_used], c->cur);
    e1 = c->ev_pool[c->ev_used + 1];
  }
  void drop() { e1 = nullptr; }
  ~KTimer() {
    if (!e1) return;
    cudaEventRecord(e1, c->cur);
    if (c->ev_class.size() < c->ev_used / 2 + 1) c->ev_class.resize(c->ev_used / 2 + 1);
    c->ev_class[c->ev_used / 2] = cls;
    c->ev_used += 2;
    c->pending_work[cls] += work;
    c->pending_count[cls] += 1;
  }
};

// Algorithmic work of the step's kernels (bytes a kernel must move, or FLOPs),
// the units the timing classes are credited with.
double rms_fwd_bytes(const Dims &D) { return (double)D.N * D.d * (4 + D.ab) + 4.0 * D.N; }
double rms_bwd_bytes(const Dims &D, bool dres, bool act) {
  return (double)D.N * D.d * (4.0 * (dres ? 4 : 3) + (act ? D.ab : 0)) + 4.0 * D.N;
}
double attn_flops(const Dims &D, double mult) {  // causal: T (T + 1) / 2 pairs
  return mult * D.B * D.H * ((double)D.T * (D.T + 1) / 2.0) * D.hd;
}

// Tensor-core GEMM launch; when timing is on, timed as class GEMM with its
// algorithmic FLOPs (unpadded sizes).
bool run_tc(llm_ctx *c, const GemmOperands &g, GemmOut out, void *C, int64_t ldc, const float *R,
            int64_t ldr, int splits, int epi, double alg_flops, void *U = nullptr,
            int64_t ldu = 0) {
  if (!c->tc) return false;
  KTimer kt(c, LLM_KT_GEMM, alg_flops);
  const bool ok = tc_gemm(c->tc, g, out, C, ldc, R, ldr, splits, epi, c->cur, U, ldu);
  if (!ok) kt.drop();
  return ok;
}

// C[M,N] = A . B^T with the operand conventions of GemmOperands; routes to
// the tensor-core kernel when it covers the shape, else to the SIMT kernel.
void gemm(llm_ctx *c, const GemmOperands &g, GemmOut out, void *C, int64_t ldc, const float *R,
          int64_t ldr, int splits, double alg_flops) {
  if (run_tc(c, g, out, C, ldc, R, ldr, splits, TC_EPI_NONE, alg_flops)) return;
  if (g.in == DT_F32 && c->tf32_floats > 0) {
    KTimer kt(c, LLM_KT_GEMM_TF32, alg_flops);
    float *scr = c->tf32_scratch[c->cur == c->s2 && c->s2 ? 1 : 0];
    if (gemm_tf32(g, out, C, ldc, R, ldr, splits, scr, c->tf32_floats, c->flag_step, c->cur))
      return;
    kt.drop();
  }
  KTimer kt(c, LLM_KT_GEMM_CUDA_CORE, alg_flops);
  gemm_simt(g, out, C, ldc, R, ldr, splits, c->cur);
}

// Gradient clipping of the whole gradient buffer with the context's norm.
void clip_step(llm_ctx *c, float *g) {
  if (c->clip_mode == LLM_CLIP_LINF)
    clip_grads_inf(g, c->D.P, c->clip, c->clip_part, c->clip_norm, c->clip_scale, c->s);
  else
    clip_grads(g, c->D.P, c->clip, c->clip_part, c->clip_norm, c->clip_scale, c->s);
}

// Dropout masks of (site, layer) for the current training call (sites: 0
// embedding output, 1 attention probabilities, 2 attention branch output, 3
// MLP branch output).
DropArgs drop_args(const llm_ctx *c, int site, int layer) {
  DropArgs a;
  a.on = 1;
  a.thr = (uint32_t)floor((double)c->drop_p * 4294967296.0);
  a.scale = (float)(1.0 / (1.0 - (double)c->drop_p));
  a.k0 = (uint32_t)c->drop_seed;
  a.k1 = (uint32_t)(c->drop_seed >> 32);
  a.site = (uint32_t)(site + 4 * layer);
  a.step = c->drop_step;
  // site 1 is [B, H, T, T], the others [B*T, d]
  const Dims &D = c->D;
  a.e0 = (uint64_t)c->drop_b0 *
         (site == 1 ? (uint64_t)D.H * D.T * D.T : (uint64_t)D.T * D.d);
  return a;
}
bool dropping(const llm_ctx *c) { return c->drop_p > 0.f; }

// One layer of the forward from its input xs[l]: the activations the
// backward reads go to slot sl (l, or 0 with recompute), and with `out` the
// layer output xs[l + 1] too.
void layer_fwd(llm_ctx *c, const float *p, int l, int sl, bool drop, bool out) {
  const Dims &D = c->D;
  POff O{D};
  cudaStream_t s = c->s;
  const int64_t N = D.N, d = D.d;
  const int ab = D.ab;
  auto A = [&](void *base, int64_t k, int64_t per) { return (char *)base + k * per * ab; };
  float *x = c->xs + l * N * d, *x1 = c->x1 + sl * N * d, *x2 = c->xs + (l + 1) * N * d;
  void *xn1 = A(c->xn1, sl, N * d), *qkv = A(c->qkv, sl, N * D.qkvw), *o = A(c->o, sl, N * d);
  void *xn2 = A(c->xn2, sl, N * d), *abuf = A(c->ab, sl, N * 2 * D.hp), *u = A(c->u, sl, N * D.hp);
  float *rstd1 = c->rstd1 + sl * N, *rstd2 = c->rstd2 + sl * N, *lse = c->lse + sl * N * D.H;
  void *wqkv = A(c->w_qkv, l, d * D.qkvw), *wo = A(c->w_o, l, d * d);
  void *w13 = A(c->w_13, l, d * 2 * D.hp), *w2 = A(c->w_2, l, D.hp * d);
  // x1 = x + Attn(RMSNorm_g1(x))
  {
    KTimer kt(c, LLM_KT_RMSNORM_FWD, rms_fwd_bytes(D));
    rmsnorm_fwd(x, p + O.g1(l), xn1, D.dt, rstd1, N, D.d, c->cfg.rms_eps, s);
  }
  {
    GemmOperands g{(int)N, (int)D.qkvw, D.d, xn1, d, true, wqkv, D.qkvw, false, D.dt};
    bool fused = run_tc(c, g, OUT_ACT, qkv, D.qkvw, nullptr, 0, 1, TC_EPI_ROPE,
                        2.0 * N * d * D.qkvw);
    if (!fused) {
      gemm(c, g, OUT_ACT, qkv, D.qkvw, nullptr, 0, 1, 2.0 * N * d * D.qkvw);
      rope_apply(qkv, D.dt, c->cos_t, c->sin_t, N, D.T, D.d + D.kvd, D.qkvw, D.hd, 1, s);
    }
  }
  if (drop) {  // x1 = x + f * (o Wo), o from dropped probabilities
    if (attn_mma_covers(D.dt, D.hd)) {
      KTimer kt(c, LLM_KT_ATTN_FWD, attn_flops(D, 4.0));
      attn_fwd_mma(qkv, o, lse, D.B, D.T, D.H, D.Hkv, D.hd, s, drop_args(c, 1, l));
    } else {
      KTimer kt(c, LLM_KT_ATTN_FWD, attn_flops(D, 4.0));
      attn_fwd_simt(qkv, o, lse, D.dt, D.B, D.T, D.H, D.Hkv, D.hd, s, drop_args(c, 1, l));
    }
    gemm(c, GemmOperands{(int)N, D.d, D.d, o, d, true, wo, d, false, D.dt}, OUT_F32, c->dtmp, d,
         nullptr, 0, 1, 2.0 * N * d * d);
    drop_add(x, c->dtmp, x1, N * d, drop_args(c, 2, l), s);
  } else {
    {
      KTimer kt(c, LLM_KT_ATTN_FWD, attn_flops(D, 4.0));
      attention_fwd(c->tc, qkv, o, lse, D.dt, D.B, D.T, D.H, D.Hkv, D.hd, s);
    }
    gemm(c, GemmOperands{(int)N, D.d, D.d, o, d, true, wo, d, false, D.dt}, OUT_ADD_F32, x1, d,
         x, d, 1, 2.0 * N * d * d);
  }
  // x2 = x1 + SwiGLU(RMSNorm_g2(x1))
  {
    KTimer kt(c, LLM_KT_RMSNORM_FWD, rms_fwd_bytes(D));
    rmsnorm_fwd(x1, p + O.g2(l), xn2, D.dt, rstd2, N, D.d, c->cfg.rms_eps, s);
  }
  // W13 GEMM into the interleaved [a|b] with u = silu(a) * b written by the
  // same epilogue (tensor-core path); else the GEMM, then a separate pass
  {
    const GemmOperands g13{(int)N, (int)(2 * D.hp), D.d, xn2, d, true, w13, 2 * D.hp, false, D.dt};
    if (!run_tc(c, g13, OUT_ACT, abuf, 2 * D.hp, nullptr, 0, 1, TC_EPI_SWIGLU,
                2.0 * N * d * 2 * D.h, u, D.hp)) {
      gemm(c, g13, OUT_ACT, abuf, 2 * D.hp, nullptr, 0, 1, 2.0 * N * d * 2 * D.h);
      KTimer kt(c, LLM_KT_SWIGLU_FWD, 3.0 * N * D.h * ab);  // read a, b; write u
      swiglu_fwd(abuf, u, D.dt, N, D.hp, s);
    }
  }
  if (!out) return;  // the recomputation stops here: x2 exists
  if (drop) {  // x2 = x1 + f * (u W2)
    gemm(c, GemmOperands{(int)N, D.d, (int)D.hp, u, D.hp, true, w2, d, false, D.dt}, OUT_F32,
         c->dtmp, d, nullptr, 0, 1, 2.0 * N * D.h * d);
    drop_add(x1, c->dtmp, x2, N * d, drop_args(c, 3, l), s);
  } else {
    gemm(c, GemmOperands{(int)N, D.d, (int)D.hp, u, D.hp, true, w2, d, false, D.dt},
         OUT_ADD_F32, x2, d, x1, d, 1, 2.0 * N * D.h * d);
  }
}

// Forward pass; leaves logits (padded, activation type) in c->logits.  train:
// a training forward (dropout applies when set; evaluation never drops).
// With dropout on, attention runs in the CUDA-core kernels, which draw the
// probability masks.
void forward(llm_ctx *c, const float *p, const int32_t *tok, bool train) {
  const bool drop = train && dropping(c);
  const Dims &D = c->D;
  POff O{D};
  cudaStream_t s = c->s;
  const int64_t N = D.N, d = D.d;
  // low-precision (or float32) padded copies of the weight matrices
  {
    const double M = (double)D.L * (d * D.qkvw + d * d + d * 2.0 * D.h + D.h * d) + d * D.V;
    KTimer kt(c, LLM_KT_WEIGHT_CAST, M * (4 + D.ab));
    if (D.L > 0) {
      cast_weight(p + O.wqkv(0), c->w_qkv, D.dt, d, D.qkvw, d, D.qkvw, 0, 0, 0, D.L, D.layer_sz,
                  d * D.qkvw, s);
      cast_weight(p + O.wo(0), c->w_o, D.dt, d, d, d, d, 0, 0, 0, D.L, D.layer_sz, d * d, s);
      cast_weight(p + O.w13(0), c->w_13, D.dt, d, 2LL * D.h, d, 2 * D.hp, 1, D.h, D.hp, D.L,
                  D.layer_sz, d * 2 * D.hp, s);
      cast_weight(p + O.w2(0), c->w_2, D.dt, D.h, d, D.hp, d, 0, 0, 0, D.L, D.layer_sz, D.hp * d, s);
    }
    cast_weight(p + O.wlm(), c->w_lm, D.dt, d, D.V, d, D.Vp, 0, 0, 0, 1, 0, 0, s);
  }
  {
    KTimer kt(c, LLM_KT_EMBED_FWD, 8.0 * N * d + 4.0 * N);
    embed_fwd(p, tok, c->xs, N, D.d, D.V, c->flag_step, s);
  }
  if (drop) drop_rows(c->xs, N * d, drop_args(c, 0, 0), s);
  for (int l = 0; l < D.L; l++) layer_fwd(c, p, l, D.rc ? 0 : l, drop, true);
  float *xL = c->xs + D.L * N * d;
  {
    KTimer kt(c, LLM_KT_RMSNORM_FWD, rms_fwd_bytes(D));
    rmsnorm_fwd(xL, p + O.gf(), c->xf, D.dt, c->rstdf, N, D.d, c->cfg.rms_eps, s);
  }
  gemm(c, GemmOperands{(int)N, (int)D.Vp, D.d, c->xf, d, true, c->w_lm, D.Vp, false, D.dt},
       OUT_ACT, c->logits, D.Vp, nullptr, 0, 1, 2.0 * N * d * D.V);
}

// Weight gradient dW[M, Ncols] = X^T dY (K = tokens), written to the unpadded
// gradient tensor through the partial buffer (fixed-order split reduction).
void wgrad(llm_ctx *c, const void *X, int64_t ldx, const void *dY, int64_t ldy, int64_t M,
           int64_t Ncols, float *grad, int64_t rows, int64_t cols, int mode) {
  const Dims &D = c->D;
  int splits = wgrad_splits(D, M, Ncols, tc_gemm_pairs(c->tc, M, Ncols));
  GemmOperands g{(int)M, (int)Ncols, (int)D.N, X, ldx, false, dY, ldy, false, D.dt};
  // one split, the caller's layout and no padding (the lm_head gradient with
  // V a multiple of 128): the product goes straight into the gradient
  if (splits == 1 && mode == 0 && rows == M && cols == Ncols && cols % 4 == 0 &&
      ((uintptr_t)grad & 15) == 0) {
    gemm(c, g, OUT_F32, grad, cols, nullptr, 0, 1, 2.0 * rows * cols * D.N);
    return;
  }
  gemm(c, g, OUT_PARTIAL, c->part, Ncols, nullptr, 0, splits, 2.0 * rows * cols * D.N);
  KTimer kt(c, LLM_KT_WGRAD_FINISH, 4.0 * splits * M * Ncols + 4.0 * rows * cols);
  wgrad_finish(c->part, splits, M, Ncols, grad, rows, cols, mode, D.h, c->cur);
}

// The weight gradients only read saved activations and a dY buffer, and only
// AdamW reads them, so they run on the side stream: forked after the main
// stream has produced their dY, joined back before the main stream
// overwrites that dY (the RMSNorm backwards) and at the end of the backward.
// They all share the split-K partial buffer, so the side stream runs them in
// order.  With kernel timing on everything stays on the main stream.
bool side_on(const llm_ctx *c) { return c->s2 && !c->timing; }
void fork_side(llm_ctx *c) {
  if (!side_on(c)) return;
  cudaEventRecord(c->ev_fork, c->s);
  cudaStreamWaitEvent(c->s2, c->ev_fork, 0);
}
void join_side(llm_ctx *c) {
  if (!side_on(c)) return;
  cudaEventRecord(c->ev_join, c->s2);
  cudaStreamWaitEvent(c->s, c->ev_join, 0);
}
void wgrad_side(llm_ctx *c, const void *X, int64_t ldx, const void *dY, int64_t ldy, int64_t M,
                int64_t Ncols, float *grad, int64_t rows, int64_t cols, int mode) {
  c->cur = side_on(c) ? c->s2 : c->s;
  wgrad(c, X, ldx, dY, ldy, M, Ncols, grad, rows, cols, mode);
  c->cur = c->s;
}

// With `buckets`, an event per gradient bucket is recorded on the main stream
// as soon as the bucket is final (bucket 0: gf and Wlm, after the first join
// of the side stream; bucket L - l: layer l, after its g1 reduction, the
// layer's weight gradients having been joined before; bucket L + 1: wte,
// after the embedding scatter and the last join).
void backward(llm_ctx *c, const float *p, float *gr, const int32_t *tok, bool buckets = false) {
  const Dims &D = c->D;
  POff O{D};
  cudaStream_t s = c->s;
  const int64_t N = D.N, d = D.d;
  const int ab = D.ab;
  const bool lp = D.dt == DT_BF16;
  auto A = [&](void *base, int64_t l, int64_t per) { return (char *)base + l * per * ab; };
  const bool drop = dropping(c);
  // dx as a GEMM operand; with dropout the masked copy of the branch
  // output's gradient (dxA, operand type at both precisions)
  void *dxop = (lp || drop) ? c->dxA : (void *)c->dx;
  void *dxact = lp ? c->dxA : nullptr;
  int nb;
  // lm_head: dxf = dz Wlm^T; dWlm = xf^T dz
  fork_side(c);  // dz (logits) and xf are ready
  wgrad_side(c, c->xf, d, c->logits, D.Vp, d, D.Vp, gr + O.wlm(), d, D.V, 0);
  gemm(c, GemmOperands{(int)N, D.d, (int)D.Vp, c->logits, D.Vp, true, c->w_lm, D.Vp, true, D.dt},
       OUT_F32, c->dtmp, d, nullptr, 0, 1, 2.0 * N * D.V * d);
  float *xL = c->xs + D.L * N * d;
  {
    KTimer kt(c, LLM_KT_RMSNORM_BWD, rms_bwd_bytes(D, false, dxact != nullptr));
    nb = rmsnorm_bwd(xL, c->rstdf, p + O.gf(), c->dtmp, nullptr, c->dx, dxact, D.dt, c->dgpart, N,
                     D.d, s);
    reduce_partials(c->dgpart, nb, D.d, gr + O.gf(), s);
  }
  for (int l = D.L - 1; l >= 0; l--) {
    // with recompute, the layer's activations come back from its input first
    // (the side stream finished with the slot at the end of layer l + 1)
    const int sl = D.rc ? 0 : l;
    if (D.rc) layer_fwd(c, p, l, 0, drop, false);
    float *x = c->xs + l * N * d, *x1 = c->x1 + sl * N * d;
    void *xn1 = A(c->xn1, sl, N * d), *qkv = A(c->qkv, sl, N * D.qkvw), *o = A(c->o, sl, N * d);
    void *xn2 = A(c->xn2, sl, N * d), *abuf = A(c->ab, sl, N * 2 * D.hp), *u = A(c->u, sl, N * D.hp);
    float *rstd1 = c->rstd1 + sl * N, *rstd2 = c->rstd2 + sl * N, *lse = c->lse + sl * N * D.H;
    void *wqkv = A(c->w_qkv, l, d * D.qkvw), *wo = A(c->w_o, l, d * d);
    void *w13 = A(c->w_13, l, d * 2 * D.hp), *w2 = A(c->w_2, l, D.hp * d);
    // FFN branch.  du = dx2 W2^T, then SwiGLU backward into dab.
    if (drop) drop_to_act(c->dx, c->dxA, D.dt, N * d, drop_args(c, 3, l), s);
    fork_side(c);  // dx2 is ready
    wgrad_side(c, u, D.hp, dxop, d, D.hp, d, gr + O.w2(l), D.h, d, 0);
    gemm(c, GemmOperands{(int)N, (int)D.hp, D.d, dxop, d, true, w2, d, true, D.dt}, OUT_ACT, c->du,
         D.hp, nullptr, 0, 1, 2.0 * N * d * D.h);
    {
      KTimer kt(c, LLM_KT_SWIGLU_BWD, 5.0 * N * D.h * ab);  // read a, b, du; write da, db
      swiglu_bwd(abuf, c->du, c->dab, D.dt, N, D.hp, s);
    }
    fork_side(c);  // dab is ready
    wgrad_side(c, xn2, d, c->dab, 2 * D.hp, d, 2 * D.hp, gr + O.w13(l), d, 2LL * D.h, 1);
    gemm(c, GemmOperands{(int)N, D.d, (int)(2 * D.hp), c->dab, 2 * D.hp, true, w13, 2 * D.hp,
                         true, D.dt},
         OUT_F32, c->dtmp, d, nullptr, 0, 1, 2.0 * N * 2 * D.h * d);
    join_side(c);  // the RMSNorm backward overwrites dx2 (dxA)
    if (buckets && l == D.L - 1) cudaEventRecord(c->ev_bucket[0], s);  // gf, Wlm
    {
      KTimer kt(c, LLM_KT_RMSNORM_BWD, rms_bwd_bytes(D, true, dxact != nullptr));
      nb = rmsnorm_bwd(x1, rstd2, p + O.g2(l), c->dtmp, c->dx, c->dx, dxact, D.dt, c->dgpart, N,
                       D.d, s);
      reduce_partials(c->dgpart, nb, D.d, gr + O.g2(l), s);
    }
    // attention branch
    if (drop) drop_to_act(c->dx, c->dxA, D.dt, N * d, drop_args(c, 2, l), s);
    gemm(c, GemmOperands{(int)N, D.d, D.d, dxop, d, true, wo, d, true, D.dt}, OUT_ACT, c->dO, d,
         nullptr, 0, 1, 2.0 * N * d * d);
    if (drop && attn_mma_covers(D.dt, D.hd)) {  // the same probability masks, RoPE fused
      KTimer kt(c, LLM_KT_ATTN_BWD, attn_flops(D, 8.0));
      attn_bwd_mma(qkv, o, c->dO, lse, c->Dbuf, c->dqkv, D.B, D.T, D.H, D.Hkv, D.hd, c->cos_t,
                   c->sin_t, s, drop_args(c, 1, l));
    } else if (drop) {  // the same probability masks, then RoPE backward on dq, dk
      {
        KTimer kt(c, LLM_KT_ATTN_BWD, attn_flops(D, 8.0));
        attn_bwd_simt(qkv, o, c->dO, lse, c->Dbuf, c->dqkv, D.dt, D.B, D.T, D.H, D.Hkv, D.hd, s,
                      drop_args(c, 1, l));
      }
      rope_apply(c->dqkv, D.dt, c->cos_t, c->sin_t, N, D.T, D.d + D.kvd, D.qkvw, D.hd, -1, s);
    } else {
      KTimer kt(c, LLM_KT_ATTN_BWD, attn_flops(D, 8.0));
      attention_bwd(c->tc, qkv, o, c->dO, lse, c->Dbuf, c->dqkv, D.dt, D.B, D.T, D.H, D.Hkv, D.hd,
                    c->cos_t, c->sin_t, s);
    }
    fork_side(c);  // dx1 and dqkv are ready (after the attention, so no TMEM contention)
    wgrad_side(c, o, d, dxop, d, d, d, gr + O.wo(l), d, d, 0);
    wgrad_side(c, xn1, d, c->dqkv, D.qkvw, d, D.qkvw, gr + O.wqkv(l), d, D.qkvw, 0);
    gemm(c, GemmOperands{(int)N, D.d, (int)D.qkvw, c->dqkv, D.qkvw, true, wqkv, D.qkvw, true,
                         D.dt},
         OUT_F32, c->dtmp, d, nullptr, 0, 1, 2.0 * N * D.qkvw * d);
    join_side(c);  // the RMSNorm backward overwrites dx1 (dxA); the next layer dqkv
    {
      KTimer kt(c, LLM_KT_RMSNORM_BWD, rms_bwd_bytes(D, true, dxact != nullptr));
      nb = rmsnorm_bwd(x, rstd1, p + O.g1(l), c->dtmp, c->dx, c->dx, dxact, D.dt, c->dgpart, N,
                       D.d, s);
      reduce_partials(c->dgpart, nb, D.d, gr + O.g1(l), s);
    }
    if (buckets) cudaEventRecord(c->ev_bucket[D.L - l], s);  // layer l
  }
  if (drop) drop_rows(c->dx, N * d, drop_args(c, 0, 0), s);
  {
    KTimer kt(c, LLM_KT_EMBED_BWD, 4.0 * N * d + 4.0 * D.V * d + 4.0 * N);
    embed_bwd(tok, c->dx, gr, N, D.d, D.V, c->sort_scratch, s);
  }
  join_side(c);  // every weight gradient is in place before AdamW
  if (buckets) {
    if (D.L == 0) cudaEventRecord(c->ev_bucket[0], s);
    cudaEventRecord(c->ev_bucket[D.L + 1], s);  // wte
  }
}

// One decode position for every sequence (position in c->dec_pos): the
// layers of the forward on one row per sequence, reading keys and values of
// positions 0..pos from the saved q|k|v activations and writing position
// pos's row of them.  Logits go to logits [B, V] (float32).
void decode_body(llm_ctx *c, const float *p, const int32_t *tok, float *logits) {
  const Dims &D = c->D;
  POff O{D};
  cudaStream_t s = c->s;
  const int64_t N = D.N, d = D.d;
  const int ab = D.ab, esz_vec = 16 / ab;
  auto A = [&](void *base, int64_t l, int64_t per) { return (char *)base + l * per * ab; };
  auto mv = [&](int64_t K, int64_t Ncols, const void *W, int64_t ldw, int epi, void *out,
                int64_t ldo, int nvalid) {
    GemvArgs a{};
    a.B = D.B;
    a.K = (int)K;
    a.N = (int)Ncols;
    a.W = W;
    a.ldw = ldw;
    a.vec = (ldw % esz_vec == 0 && ((uintptr_t)W & 15) == 0) ? 1 : 0;
    a.eps = c->cfg.rms_eps;
    gemv_plan(K, Ncols, &a.ks, &a.kslice);
    a.part = c->dec_part;
    a.count = c->dec_count;
    a.epi = epi;
    a.out = out;
    a.ldo = ldo;
    a.nvalid = nvalid;
    a.cos_t = c->cos_t;
    a.sin_t = c->sin_t;
    a.pos = c->dec_pos;
    a.hd = D.hd;
    a.rot_cols = D.d + D.kvd;
    return a;
  };
  embed_fwd(p, tok, c->dec_x, D.B, D.d, D.V, c->flag_step, s);
  for (int l = 0; l < D.L; l++) {
    void *qkv = A(c->qkv, l, N * D.qkvw);
    // q|k|v of position pos (RMSNorm g1 on the fly, RoPE on q and k) into
    // row (b, pos) of the layer's saved activations
    GemvArgs a = mv(d, D.qkvw, A(c->w_qkv, l, d * D.qkvw), D.qkvw, DEC_QKV, qkv,
                    (int64_t)D.T * D.qkvw, (int)D.qkvw);
    a.x = c->dec_x; a.ldx = d; a.gain = p + O.g1(l); a.pos_stride = D.qkvw;
    gemv(a, D.dt, s);
    attn_decode(qkv, D.qkvw, D.B, D.T, c->dec_pos, D.H, D.Hkv, D.hd, c->dec_attn, c->dec_acount,
                c->dec_o, D.dt, s);
    // x += o Wo
    a = mv(d, d, A(c->w_o, l, d * d), d, DEC_RESID, c->dec_x, d, D.d);
    a.xa = c->dec_o; a.ldxa = d;
    gemv(a, D.dt, s);
    // u = SwiGLU(RMSNorm_g2(x) W13); x += u W2
    a = mv(d, 2 * D.hp, A(c->w_13, l, d * 2 * D.hp), 2 * D.hp, DEC_SWIGLU, c->dec_u, D.hp,
           (int)D.hp);
    a.x = c->dec_x; a.ldx = d; a.gain = p + O.g2(l);
    gemv(a, D.dt, s);
    a = mv(D.hp, d, A(c->w_2, l, D.hp * d), d, DEC_RESID, c->dec_x, d, D.d);
    a.xa = c->dec_u; a.ldxa = D.hp;
    gemv(a, D.dt, s);
  }
  GemvArgs a = mv(d, D.Vp, c->w_lm, D.Vp, DEC_LOGITS, logits, D.V, D.V);
  a.x = c->dec_x; a.ldx = d; a.gain = p + O.gf();
  gemv(a, D.dt, s);
}

}  // namespace

extern "C" {

int llm_forward(llm_ctx *c, const float *d_params, const int32_t *d_tokens, float *d_logits) {
  if (!c || !d_params || !d_tokens || !d_logits) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  g_launches = 0;
  set_flag_zero(c->flag_step, c->s);
  forward(c, d_params, d_tokens, false);
  logits_out(c->logits, c->D.dt, d_logits, c->D.N, c->D.V, c->D.Vp, c->s);
  or_flag(c->flag_step, c->flag_sticky, c->s);
  c->last_launches = g_launches;
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}

int llm_step(llm_ctx *c, float *d_params, float *d_grads, float *d_m, float *d_v, int64_t t,
             const int32_t *d_tokens, const int32_t *d_targets, float lr, float wd,
             float *d_loss) {
  if (!c || !d_tokens || !d_targets || !d_loss || t < 1) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  if (!aligned16(d_params) || !aligned16(d_grads) || !aligned16(d_m) || !aligned16(d_v))
    return LLM_ERR_ARG;
  const Dims &D = c->D;
  g_launches = 0;
  // the step's scalars go to device memory first (outside any graph)
  const double bc1 = 1.0 - pow((double)c->cfg.beta1, (double)t);
  const double bc2 = 1.0 - pow((double)c->cfg.beta2, (double)t);
  set_hyper(c->hyper, lr, wd, (float)bc1, (float)bc2, c->s);
  // the mask step word also goes to device memory outside any graph
  if (dropping(c)) set_device_int(c->drop_step, (int)(c->train_calls++), c->s);
  auto body = [&]() {
    set_flag_zero(c->flag_step, c->s);
    forward(c, d_params, d_tokens, true);
    {
      // logits read and written once (the gradient over them in place), row losses
      KTimer kt(c, LLM_KT_CROSS_ENTROPY, 2.0 * D.N * D.V * D.ab + 8.0 * D.N);
      cross_entropy(c->logits, D.dt, d_targets, c->rowloss, D.N, D.V, D.Vp, 1.0f / (float)D.N,
                    c->flag_step, c->s);
      loss_reduce(c->rowloss, D.N, d_loss, c->flag_step, c->s);
    }
    backward(c, d_params, d_grads, d_tokens);
    if (c->clip > 0.f) clip_step(c, d_grads);
    {
      KTimer kt(c, LLM_KT_ADAMW, 28.0 * D.P);  // read p, g, m, v; write p, m, v
      adamw(d_params, d_grads, d_m, d_v, D.P, c->hyper, c->cfg.beta1, c->cfg.beta2,
            c->cfg.adam_eps, c->flag_step, c->s);
    }
    or_flag(c->flag_step, c->flag_sticky, c->s);
  };
  if (c->clip > 0.f) c->have_norm = true;
  const llm_ctx::Key key{{d_params, d_grads, d_m, d_v, d_tokens, d_targets, d_loss}};
  // graphs need a capturable stream (not the legacy default stream); steps
  // with kernel timing on run as individual launches
  if (c->graphs && !c->timing && c->s != nullptr) {
    if (c->gexec && key == c->gkey) {
      if (cudaGraphLaunch(c->gexec, c->s) != cudaSuccess) return LLM_ERR_CUDA;
      c->last_launches = 1 + c->graph_launches;
      return LLM_OK;
    }
    if (c->have_prev && key == c->prev_key) {
      // second call with these buffers: capture the step, then replay it
      const int before = g_launches;
      cudaGraph_t graph = nullptr;
      bool ok = cudaStreamBeginCapture(c->s, cudaStreamCaptureModeThreadLocal) == cudaSuccess;
      if (ok) {
        body();
        ok = cudaStreamEndCapture(c->s, &graph) == cudaSuccess && graph;
      }
      cudaGraphExec_t exec = nullptr;
      if (ok) ok = cudaGraphInstantiate(&exec, graph, 0) == cudaSuccess;
      if (graph) cudaGraphDestroy(graph);
      if (ok) {
        if (c->gexec) cudaGraphExecDestroy(c->gexec);
        c->gexec = exec;
        c->gkey = key;
        c->graph_launches = g_launches - before;
        if (cudaGraphLaunch(c->gexec, c->s) != cudaSuccess) return LLM_ERR_CUDA;
        c->last_launches = 1 + c->graph_launches;
        return LLM_OK;
      }
      // the capture did not work out: no more graphs for this context
      (void)cudaGetLastError();
      c->graphs = false;
      g_launches = before;
    }
  }
  c->prev_key = key;
  c->have_prev = true;
  body();
  c->last_launches = g_launches;
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}

int llm_grad(llm_ctx *c, const float *d_params, float *d_grads, const int32_t *d_tokens,
             const int32_t *d_targets, float *d_loss) {
  if (!c || !d_tokens || !d_targets || !d_loss) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  if (!aligned16(d_params) || !aligned16(d_grads)) return LLM_ERR_ARG;
  const Dims &D = c->D;
  g_launches = 0;
  if (dropping(c)) set_device_int(c->drop_step, (int)(c->train_calls++), c->s);
  set_flag_zero(c->flag_step, c->s);
  forward(c, d_params, d_tokens, true);
  cross_entropy(c->logits, D.dt, d_targets, c->rowloss, D.N, D.V, D.Vp, 1.0f / (float)D.N,
                c->flag_step, c->s);
  loss_reduce(c->rowloss, D.N, d_loss, c->flag_step, c->s);
  backward(c, d_params, d_grads, d_tokens, c->buckets_on);
  c->buckets_recorded = c->buckets_on;
  or_flag(c->flag_step, c->flag_sticky, c->s);
  c->last_launches = g_launches;
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}

int llm_set_grad_buckets(llm_ctx *c, int enable) {
  if (!c) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  if (enable && c->ev_bucket.empty()) {
    for (int k = 0; k < c->D.L + 2; k++) {
      cudaEvent_t e = nullptr;
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
        for (cudaEvent_t x : c->ev_bucket) cudaEventDestroy(x);
        c->ev_bucket.clear();
        return LLM_ERR_CUDA;
      }
      c->ev_bucket.push_back(e);
    }
  }
  c->buckets_on = enable != 0;
  c->buckets_recorded = false;
  return LLM_OK;
}

int llm_grad_bucket_range(const llm_config *cfg, int k, int64_t *offset, int64_t *count) {
  if (!offset || !count) return LLM_ERR_ARG;
  if (!valid_config(cfg)) return LLM_ERR_CONFIG;
  const Dims D = make_dims(cfg);
  if (k < 0 || k > D.L + 1) return LLM_ERR_ARG;
  POff O{D};
  if (k == 0) {  // gf, Wlm
    *offset = O.gf();
    *count = D.P - O.gf();
  } else if (k <= D.L) {  // layer L - k
    *offset = O.layer(D.L - k);
    *count = D.layer_sz;
  } else {  // wte
    *offset = 0;
    *count = (int64_t)D.V * D.d;
  }
  return LLM_OK;
}

int llm_grad_bucket_wait(llm_ctx *c, int k, void *stream) {
  if (!c) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  if (!c->buckets_recorded || k < 0 || k > c->D.L + 1) return LLM_ERR_ARG;
  return cudaStreamWaitEvent((cudaStream_t)stream, c->ev_bucket[k], 0) == cudaSuccess
             ? LLM_OK
             : LLM_ERR_CUDA;
}

int llm_adamw(llm_ctx *c, float *d_params, float *d_grads, float *d_m, float *d_v, int64_t t,
              float lr, float wd, float grad_scale) {
  if (!c || t < 1 || !std::isfinite(grad_scale)) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  if (!aligned16(d_params) || !aligned16(d_grads) || !aligned16(d_m) || !aligned16(d_v))
    return LLM_ERR_ARG;
  const Dims &D = c->D;
  g_launches = 0;
  const double bc1 = 1.0 - pow((double)c->cfg.beta1, (double)t);
  const double bc2 = 1.0 - pow((double)c->cfg.beta2, (double)t);
  set_hyper(c->hyper, lr, wd, (float)bc1, (float)bc2, c->s);
  if (grad_scale != 1.0f) scale_grads(d_grads, D.P, grad_scale, c->s);
  if (c->clip > 0.f) {
    clip_step(c, d_grads);
    c->have_norm = true;
  }
  adamw(d_params, d_grads, d_m, d_v, D.P, c->hyper, c->cfg.beta1, c->cfg.beta2, c->cfg.adam_eps,
        c->flag_step, c->s);
  c->last_launches = g_launches;
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}

int llm_adamw_range(llm_ctx *c, float *d_params, float *d_grads, float *d_m, float *d_v,
                    int64_t count, int64_t t, float lr, float wd, float grad_scale) {
  if (!c || t < 1 || count < 0 || !std::isfinite(grad_scale)) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  if (!aligned16(d_params) || !aligned16(d_grads) || !aligned16(d_m) || !aligned16(d_v))
    return LLM_ERR_ARG;
  g_launches = 0;
  const double bc1 = 1.0 - pow((double)c->cfg.beta1, (double)t);
  const double bc2 = 1.0 - pow((double)c->cfg.beta2, (double)t);
  set_hyper(c->hyper, lr, wd, (float)bc1, (float)bc2, c->s);
  if (count > 0) {
    if (grad_scale != 1.0f) scale_grads(d_grads, count, grad_scale, c->s);
    adamw(d_params, d_grads, d_m, d_v, count, c->hyper, c->cfg.beta1, c->cfg.beta2,
          c->cfg.adam_eps, c->flag_step, c->s);
  }
  c->last_launches = g_launches;
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}

int llm_grad_norm_part(llm_ctx *c, float *d_grads, int64_t count, float grad_scale,
                       int accumulate, double *d_part) {
  if (!c || count < 0 || !std::isfinite(grad_scale) || (accumulate != 0 && accumulate != 1))
    return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  if (!aligned16(d_grads) || !d_part || ((uintptr_t)d_part & 7)) return LLM_ERR_ARG;
  g_launches = 0;
  grad_norm_part(d_grads, count, grad_scale, c->clip_mode == LLM_CLIP_LINF ? 1 : 0, accumulate,
                 c->clip_part, d_part, c->s);
  c->last_launches = g_launches;
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}

int llm_adamw_range_clip(llm_ctx *c, float *d_params, float *d_grads, float *d_m, float *d_v,
                         int64_t count, int64_t t, float lr, float wd, const double *d_total) {
  if (!c || t < 1 || count < 0) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  if (!aligned16(d_params) || !aligned16(d_grads) || !aligned16(d_m) || !aligned16(d_v))
    return LLM_ERR_ARG;
  if (c->clip > 0.f && (!d_total || ((uintptr_t)d_total & 7))) return LLM_ERR_ARG;
  g_launches = 0;
  const double bc1 = 1.0 - pow((double)c->cfg.beta1, (double)t);
  const double bc2 = 1.0 - pow((double)c->cfg.beta2, (double)t);
  set_hyper(c->hyper, lr, wd, (float)bc1, (float)bc2, c->s);
  if (c->clip > 0.f) {
    clip_from_total(d_grads, count, d_total, c->clip_mode == LLM_CLIP_LINF ? 1 : 0, c->clip,
                    c->clip_norm, c->clip_scale, c->s);
    c->have_norm = true;
  }
  if (count > 0)
    adamw(d_params, d_grads, d_m, d_v, count, c->hyper, c->cfg.beta1, c->cfg.beta2,
          c->cfg.adam_eps, c->flag_step, c->s);
  c->last_launches = g_launches;
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}

int llm_flag_out(llm_ctx *c, int32_t *d_flag) {
  if (!c || !d_flag) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  if (cudaMemcpyAsync(d_flag, c->flag_step, sizeof(int32_t), cudaMemcpyDeviceToDevice, c->s) !=
      cudaSuccess)
    return LLM_ERR_CUDA;
  return LLM_OK;
}

int llm_flag_in(llm_ctx *c, const int32_t *d_flag) {
  if (!c || !d_flag) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  g_launches = 0;
  or_flag(d_flag, c->flag_step, c->s);
  c->last_launches = g_launches;
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}

int llm_decode(llm_ctx *c, const float *d_params, const int32_t *d_tokens, int pos,
               float *d_logits) {
  if (!c || !d_params || !d_tokens || !d_logits) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  const Dims &D = c->D;
  if (pos < 0 || pos >= D.T) return LLM_ERR_ARG;
  if (128 % D.hd || D.rc) return LLM_ERR_CONFIG;
  // every projection's K (d_model, or the padded d_ff of W2) in 16 slices
  if (!gemv_fits(D.d, D.qkvw) || !gemv_fits(D.d, 2 * D.hp) || !gemv_fits(D.hp, D.d) ||
      !gemv_fits(D.d, D.Vp))
    return LLM_ERR_CONFIG;
  if (((uintptr_t)d_params & 3) || ((uintptr_t)d_tokens & 3) || ((uintptr_t)d_logits & 3))
    return LLM_ERR_ARG;
  g_launches = 0;
  set_device_int(c->dec_pos, pos, c->s);  // outside any graph
  const int before = g_launches;
  auto body = [&]() {
    set_flag_zero(c->flag_step, c->s);
    decode_body(c, d_params, d_tokens, d_logits);
    or_flag(c->flag_step, c->flag_sticky, c->s);
  };
  const llm_ctx::Key key{{d_params, d_tokens, d_logits, nullptr, nullptr, nullptr, nullptr}};
  if (c->graphs && c->s != nullptr) {
    if (c->dexec && key == c->dkey) {
      if (cudaGraphLaunch(c->dexec, c->s) != cudaSuccess) return LLM_ERR_CUDA;
      c->last_launches = before + c->dgraph_launches;
      return LLM_OK;
    }
    if (c->dhave_prev && key == c->dprev_key) {
      cudaGraph_t graph = nullptr;
      bool ok = cudaStreamBeginCapture(c->s, cudaStreamCaptureModeThreadLocal) == cudaSuccess;
      if (ok) {
        body();
        ok = cudaStreamEndCapture(c->s, &graph) == cudaSuccess && graph;
      }
      cudaGraphExec_t exec = nullptr;
      if (ok) ok = cudaGraphInstantiate(&exec, graph, 0) == cudaSuccess;
      if (graph) cudaGraphDestroy(graph);
      if (ok) {
        if (c->dexec) cudaGraphExecDestroy(c->dexec);
        c->dexec = exec;
        c->dkey = key;
        c->dgraph_launches = g_launches - before;
        if (cudaGraphLaunch(c->dexec, c->s) != cudaSuccess) return LLM_ERR_CUDA;
        c->last_launches = before + c->dgraph_launches;
        return LLM_OK;
      }
      (void)cudaGetLastError();
      c->graphs = false;
      g_launches = before;
    }
  }
  c->dprev_key = key;
  c->dhave_prev = true;
  body();
  c->last_launches = g_launches;
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}

int llm_sample(llm_ctx *c, const float *d_logits, int64_t ld, int n_rows, float temperature,
               int top_k, const float *d_uniform, int32_t *d_out) {
  if (!c || !d_logits || !d_uniform || !d_out || n_rows < 1 || ld < c->D.V) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  if (!(temperature == temperature)) return LLM_ERR_ARG;  // NaN
  g_launches = 0;
  sample_tokens(d_logits, ld, n_rows, c->D.V, temperature, top_k, d_uniform, d_out, c->s);
  c->last_launches = g_launches;
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}

int llm_sample_ex(llm_ctx *c, const float *d_logits, int64_t ld, int n_rows, float temperature,
                  int top_k, float top_p, float repetition_penalty, const int32_t *d_history,
                  int64_t history_ld, int history_len, const float *d_uniform, int32_t *d_out) {
  if (!c || !d_logits || !d_uniform || !d_out || n_rows < 1 || ld < c->D.V) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  if (!(temperature == temperature) || !(top_p > 0.f) || !(top_p <= 1.f)) return LLM_ERR_ARG;
  if (top_p < 1.f && (top_k < 1 || top_k > sample_ex_max_top_k())) return LLM_ERR_ARG;
  if (!(repetition_penalty > 0.f) || !std::isfinite(repetition_penalty) || history_len < 0)
    return LLM_ERR_ARG;
  const bool pen = repetition_penalty != 1.f && history_len > 0;
  if (pen && (!d_history || history_ld < history_len ||
              (int64_t)c->D.V > sample_ex_max_vocab_penalty()))
    return LLM_ERR_ARG;
  g_launches = 0;
  sample_tokens_ex(d_logits, ld, n_rows, c->D.V, temperature, top_k, top_p, repetition_penalty,
                   d_history, history_ld, pen ? history_len : 0, d_uniform, d_out, c->s);
  c->last_launches = g_launches;
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}

int llm_init(llm_ctx *c, uint64_t seed, float init_std, int scale_out_proj, float *d_params) {
  if (!c || !d_params || !(init_std >= 0.f)) return LLM_ERR_ARG;
  if (!on_device(c)) return LLM_ERR_ARG;
  const Dims &D = c->D;
  POff O{D};
  g_launches = 0;
  float so = scale_out_proj ? init_std / sqrtf(2.0f * (float)std::max(1, D.L)) : init_std;
  auto mat = [&](int64_t off, int64_t n, float sd) { init_params(d_params + off, n, seed, off, sd, 0, c->s); };
  auto one = [&](int64_t off, int64_t n) { init_params(d_params + off, n, seed, off, 0.f, 1, c->s); };
  mat(0, (int64_t)D.V * D.d, init_std);
  for (int l = 0; l < D.L; l++) {
    one(O.g1(l), D.d);
    mat(O.wqkv(l), (int64_t)D.d * D.qkvw, init_std);
    mat(O.wo(l), (int64_t)D.d * D.d, so);
    one(O.g2(l), D.d);
    mat(O.w13(l), (int64_t)D.d * 2 * D.h, init_std);
    mat(O.w2(l), (int64_t)D.h * D.d, so);
  }
  one(O.gf(), D.d);
  mat(O.wlm(), (int64_t)D.d * D.V, init_std);
  c->last_launches = g_launches;
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}

}  // extern "C"

// ----------------------------------------------------- single-kernel entries
#include "../../include/llm_kernels.h"

extern "C" int llm_kernel_gemm_bf16(int M, int N, int K, const void *d_A, int64_t lda,
                                    int a_kmajor, const void *d_B, int64_t ldb, int b_kmajor,
                                    float *d_C, int64_t ldc, int tensor_cores, int *d_flag,
                                    void *stream) {
  if (M < 1 || N < 1 || K < 1 || !d_A || !d_B || !d_C || !d_flag) return LLM_ERR_ARG;
  if (lda < (a_kmajor ? K : M) || ldb < (b_kmajor ? K : N) || ldc < N) return LLM_ERR_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  GemmOperands g{M, N, K, d_A, lda, a_kmajor != 0, d_B, ldb, b_kmajor != 0, DT_BF16};
  if (!claim_device(nullptr)) return LLM_ERR_ARG;  // one device per process
  g_launches = 0;
  if (tensor_cores) {
    static TcPlan *plan = nullptr;
    static std::once_flag once;
    std::call_once(once, [] { plan = tc_plan_create(DT_BF16, nullptr, nullptr, 1, 64, 0, 64); });
    if (!plan) return LLM_ERR_ARG;
    tc_plan_set_flag(plan, d_flag);
    if (!tc_gemm(plan, g, OUT_F32, d_C, ldc, nullptr, 0, 1, TC_EPI_NONE, s))
      return LLM_ERR_ARG;
  } else {
    gemm_simt(g, OUT_F32, d_C, ldc, nullptr, 0, 1, s);
  }
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}

extern "C" int llm_kernel_gemm_f32_scratch_floats(int M, int N, int K, int64_t *floats) {
  if (M < 1 || N < 1 || K < 1 || !floats) return LLM_ERR_ARG;
  *floats = gemm_tf32_scratch_floats(M, N, K);
  return LLM_OK;
}

extern "C" int llm_kernel_gemm_f32(int M, int N, int K, const float *d_A, int64_t lda,
                                   int a_kmajor, const float *d_B, int64_t ldb, int b_kmajor,
                                   float *d_C, int64_t ldc, int tensor_cores, float *d_scratch,
                                   int64_t scratch_floats, int *d_flag, void *stream) {
  if (M < 1 || N < 1 || K < 1 || !d_A || !d_B || !d_C || !d_flag) return LLM_ERR_ARG;
  if (lda < (a_kmajor ? K : M) || ldb < (b_kmajor ? K : N) || ldc < N) return LLM_ERR_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  GemmOperands g{M, N, K, d_A, lda, a_kmajor != 0, d_B, ldb, b_kmajor != 0, DT_F32};
  if (!claim_device(nullptr)) return LLM_ERR_ARG;  // one device per process
  g_launches = 0;
  if (tensor_cores) {
    if (!d_scratch || scratch_floats < gemm_tf32_scratch_floats(M, N, K) ||
        ((uintptr_t)d_scratch & 15))
      return LLM_ERR_ARG;
    if (!gemm_tf32(g, OUT_F32, d_C, ldc, nullptr, 0, 1, d_scratch, scratch_floats, d_flag, s))
      return LLM_ERR_ARG;
  } else {
    gemm_simt(g, OUT_F32, d_C, ldc, nullptr, 0, 1, s);
  }
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}

extern "C" int llm_kernel_embed_bwd_scratch_bytes(int64_t n_tokens, int vocab, int64_t *bytes) {
  if (!bytes || n_tokens < 1 || vocab < 1 || n_tokens > ((int64_t)1 << 30)) return LLM_ERR_ARG;
  *bytes = 4 * embed_bwd_scratch_ints(n_tokens, vocab);
  return LLM_OK;
}

extern "C" int llm_kernel_embed_bwd(const int32_t *d_tokens, const float *d_dx, float *d_dwte,
                                    int64_t n_tokens, int d_model, int vocab, void *d_scratch,
                                    int64_t scratch_bytes, void *stream) {
  if (!d_tokens || !d_dx || !d_dwte || !d_scratch || n_tokens < 1 || d_model < 1 || vocab < 1 ||
      n_tokens > ((int64_t)1 << 30) || ((uintptr_t)d_scratch & 15))
    return LLM_ERR_ARG;
  if (scratch_bytes < 4 * embed_bwd_scratch_ints(n_tokens, vocab)) return LLM_ERR_ARG;
  if (!claim_device(nullptr)) return LLM_ERR_ARG;  // one device per process
  g_launches = 0;
  embed_bwd(d_tokens, d_dx, d_dwte, n_tokens, d_model, vocab, (int32_t *)d_scratch,
            (cudaStream_t)stream);
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}

// Time-out flag of the tcgen05 attention kernels called through the kernel
// entries: one library-owned device word.
static int *attn_kernel_flag() {
  static int *flag = nullptr;
  static std::once_flag once;
  std::call_once(once, [] { cudaMalloc(&flag, sizeof(int)); cudaMemset(flag, 0, sizeof(int)); });
  return flag;
}

static bool attn_args_ok(const void *a, const void *b, int B, int T, int H, int Hkv, int hd) {
  return a && b && B >= 1 && T >= 1 && H >= 1 && Hkv >= 1 && H % Hkv == 0 && hd >= 2 &&
         hd % 2 == 0 && hd <= 128;
}

extern "C" int llm_kernel_attention_fwd_bf16(const void *d_qkv, void *d_o, float *d_lse,
                                             int batch, int ctx, int n_head, int n_kv_head,
                                             int head_dim, int tensor_cores, void *stream) {
  if (!attn_args_ok(d_qkv, d_o, batch, ctx, n_head, n_kv_head, head_dim) || !d_lse)
    return LLM_ERR_ARG;
  if (!claim_device(nullptr)) return LLM_ERR_ARG;  // one device per process
  g_launches = 0;
  cudaStream_t s = (cudaStream_t)stream;
  if (tensor_cores == 2) {
    int *flag = attn_kernel_flag();
    if (!flag || !attn_tc_covers(DT_BF16, head_dim, ctx) ||
        !attn_fwd_tc(d_qkv, d_o, d_lse, batch, ctx, n_head, n_kv_head, head_dim, flag, s))
      return LLM_ERR_ARG;
  } else if (tensor_cores == 1) {
    if (!attn_mma_covers(DT_BF16, head_dim)) return LLM_ERR_ARG;
    attn_fwd_mma(d_qkv, d_o, d_lse, batch, ctx, n_head, n_kv_head, head_dim, s);
  } else {
    attn_fwd_simt(d_qkv, d_o, d_lse, DT_BF16, batch, ctx, n_head, n_kv_head, head_dim, s);
  }
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}

extern "C" int llm_kernel_attention_fwd_f32(const float *d_qkv, float *d_o, float *d_lse, int batch,
                                            int ctx, int n_head, int n_kv_head, int head_dim,
                                            int tiled, void *stream) {
  if (!attn_args_ok(d_qkv, d_o, batch, ctx, n_head, n_kv_head, head_dim) || !d_lse)
    return LLM_ERR_ARG;
  if (!claim_device(nullptr)) return LLM_ERR_ARG;  // one device per process
  g_launches = 0;
  cudaStream_t s = (cudaStream_t)stream;
  if (tiled) {
    if (((uintptr_t)d_qkv | (uintptr_t)d_o) & 15) return LLM_ERR_ARG;
    if (!attn_fwd_f32_tiled(d_qkv, d_o, d_lse, batch, ctx, n_head, n_kv_head, head_dim, s))
      return LLM_ERR_ARG;
  } else {
    attn_fwd_rows(d_qkv, d_o, d_lse, DT_F32, batch, ctx, n_head, n_kv_head, head_dim, s,
                  DropArgs{});
  }
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}

extern "C" int llm_kernel_attention_bwd_f32(const float *d_qkv, const float *d_o,
                                            const float *d_dout, const float *d_lse, float *d_D,
                                            float *d_dqkv, int batch, int ctx, int n_head,
                                            int n_kv_head, int head_dim, int tiled,
                                            void *stream) {
  if (!attn_args_ok(d_qkv, d_o, batch, ctx, n_head, n_kv_head, head_dim) || !d_dout || !d_lse ||
      !d_D || !d_dqkv)
    return LLM_ERR_ARG;
  if (!claim_device(nullptr)) return LLM_ERR_ARG;  // one device per process
  g_launches = 0;
  cudaStream_t s = (cudaStream_t)stream;
  if (tiled) {
    if (((uintptr_t)d_qkv | (uintptr_t)d_o | (uintptr_t)d_dout | (uintptr_t)d_dqkv) & 15)
      return LLM_ERR_ARG;
    if (!attn_bwd_f32_tiled(d_qkv, d_o, d_dout, d_lse, d_D, d_dqkv, batch, ctx, n_head,
                            n_kv_head, head_dim, s))
      return LLM_ERR_ARG;
  } else {
    attn_bwd_rows(d_qkv, d_o, d_dout, d_lse, d_D, d_dqkv, DT_F32, batch, ctx, n_head, n_kv_head,
                  head_dim, s, DropArgs{});
  }
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}

extern "C" int llm_kernel_attention_bwd_bf16(const void *d_qkv, const void *d_o,
                                             const void *d_dout, const float *d_lse, float *d_D,
                                             void *d_dqkv, int batch, int ctx, int n_head,
                                             int n_kv_head, int head_dim, int tensor_cores,
                                             void *stream) {
  if (!attn_args_ok(d_qkv, d_o, batch, ctx, n_head, n_kv_head, head_dim) || !d_dout || !d_lse ||
      !d_D || !d_dqkv)
    return LLM_ERR_ARG;
  if (!claim_device(nullptr)) return LLM_ERR_ARG;  // one device per process
  g_launches = 0;
  cudaStream_t s = (cudaStream_t)stream;
  if (tensor_cores == 2) {
    int *flag = attn_kernel_flag();
    if (!flag || !attn_tc_covers(DT_BF16, head_dim, ctx) ||
        !attn_bwd_tc(d_qkv, d_o, d_dout, d_lse, d_D, d_dqkv, batch, ctx, n_head, n_kv_head,
                     head_dim, nullptr, nullptr, flag, s))
      return LLM_ERR_ARG;
  } else if (tensor_cores == 1) {
    if (!attn_mma_covers(DT_BF16, head_dim)) return LLM_ERR_ARG;
    attn_bwd_mma(d_qkv, d_o, d_dout, d_lse, d_D, d_dqkv, batch, ctx, n_head, n_kv_head, head_dim,
                 nullptr, nullptr, s);
  } else {
    attn_bwd_simt(d_qkv, d_o, d_dout, d_lse, d_D, d_dqkv, DT_BF16, batch, ctx, n_head, n_kv_head,
                  head_dim, s);
  }
  return cudaGetLastError() == cudaSuccess ? LLM_OK : LLM_ERR_CUDA;
}
