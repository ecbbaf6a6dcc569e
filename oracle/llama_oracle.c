/*
 * Plain float64 CPU oracle of one training step of a bias-free, pre-norm
 * Llama-style decoder: forward, hand-derived backward, AdamW.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes
 * or calls this file; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark use it.  It shares no code, header or table with the CUDA
 * path.
 *
 * Every function is the definition written out, in float64, with plain loops.
 * OpenMP splits independent output rows (or heads) across threads; each output
 * element is produced by one thread with a fixed summation order, so results
 * do not depend on the thread count ("Hephaistos", Design notes: threads only
 * write disjoint regions).
 *
 * Sources (page title, section):
 *   Hephaistos, "Architecture at a glance": pre-norm block, RMSNorm with cached
 *     rstd, RoPE on q/k inside attention, causal MHA with stable softmax,
 *     SwiGLU (silu(x W1) * x W3) W2, untied lm_head, AdamW with decoupled
 *     weight decay and bias correction.
 *   Hephaistos, "Design notes": flat parameter buffer with named offsets.
 *   Hephaistos, "Run your model in llama.cpp": the q/k layout is rotate-half.
 *   MicroGPT in Rust, "RMSNorm": eps 1e-5 added to the mean square.
 *   strata, capability table: fused causal attention takes n_head and
 *     n_kv_head independently (MHA/GQA/MQA); AdamW decoupled, bias-corrected.
 *   randyGPT, "Training (Metal GPU path)": cross-entropy over all positions.
 *
 * Readings taken where the pages are silent:
 *   - attention scale 1/sqrt(head_dim); the causal mask keeps the diagonal;
 *   - GQA groups are contiguous: query head hq uses kv head hq / (H/Hkv);
 *   - RoPE: theta_j = base^(-2j/hd), position = index within the sequence,
 *     pairs (j, j+hd/2);
 *   - loss = mean over all B*T positions, no ignore index;
 *   - AdamW: eps outside the sqrt, decay applied to every tensor.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Parallel regions only for work large enough to pay for the threads. */
#define OMP_MIN_WORK (1LL << 18)

typedef struct {
  int32_t V, d, L, H, Hkv, h, T, B;
  double rope_base, eps;
  double rope_scale; /* position interpolation: RoPE position = t / rope_scale */
} orc_cfg;

/* ----------------------------------------------------------------- dropout */
/* Inverted dropout (Hephaistos, Architecture at a glance: dropout on the
 * embeddings, the attention weights and the attention and MLP outputs; masks
 * drawn by the training forward and reused by its backward).  The masks come
 * from Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
 * easy as 1, 2, 3", SC 2011), whose one call gives four 32-bit words: the
 * elements are taken in groups of four consecutive indices, key = the seed's
 * two 32-bit halves, counter = (group index low word, group index high word,
 * site + 4 * layer, step), group index = element index / 4, with sites 0
 * embedding output [B*T, d], 1 attention probabilities [B, H, T, T],
 * 2 attention branch output [B*T, d], 3 MLP branch output [B*T, d] (element
 * index row-major over those shapes).  Element e is kept when output word
 * e mod 4 of its group's call is >= floor(p * 2^32); kept elements are scaled
 * by 1 / (1 - p).  The pages fix the rate and the sites, not the generator. */
void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3], k0 = key[0], k1 = key[1];
  for (int r = 0; r < 10; r++) {
    uint64_t p0 = (uint64_t)0xD2511F53u * c0, p1 = (uint64_t)0xCD9E8D57u * c2;
    uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0, n1 = (uint32_t)p1;
    uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1, n3 = (uint32_t)p0;
    c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

typedef struct {
  double p;       /* drop probability in [0, 1) */
  uint64_t seed;
  uint32_t step;  /* training forward number */
} orc_dropout;

/* 0 or 1/(1-p) for element e of (site, layer) */
static double drop_factor(const orc_dropout *dr, int site, int layer, uint64_t e) {
  const uint64_t g = e / 4;
  uint32_t ctr[4] = {(uint32_t)g, (uint32_t)(g >> 32), (uint32_t)(site + 4 * layer), dr->step};
  uint32_t key[2] = {(uint32_t)dr->seed, (uint32_t)(dr->seed >> 32)}, out[4];
  orc_philox4x32_10(ctr, key, out);
  const uint64_t thr = (uint64_t)floor(dr->p * 4294967296.0);
  return (uint64_t)out[e % 4] >= thr ? 1.0 / (1.0 - dr->p) : 0.0;
}

/* ------------------------------------------------------------------ layout */
/* Flat parameter buffer ("Hephaistos", Design notes: flat buffers, named
 * offsets).  Order: wte[V,d]; per layer g1[d], Wqkv[d, d+2kvd], Wo[d,d], g2[d],
 * W13[d,2h] (W1 = columns [0,h), W3 = columns [h,2h)), W2[h,d]; gf[d];
 * Wlm[d,V].  Matrices are [in, out] row-major so a projection is x W. */
static int64_t qkvw(const orc_cfg *c) { return (int64_t)c->d + 2LL * (c->d / c->H) * c->Hkv; }
static int64_t layer_size(const orc_cfg *c) {
  int64_t d = c->d, h = c->h;
  return d + d * qkvw(c) + d * d + d + d * 2 * h + h * d;
}
int64_t orc_n_params(const orc_cfg *c) {
  return (int64_t)c->V * c->d + c->L * layer_size(c) + c->d + (int64_t)c->d * c->V;
}
static int64_t off_layer(const orc_cfg *c, int l) { return (int64_t)c->V * c->d + l * layer_size(c); }
static int64_t off_g1(const orc_cfg *c, int l) { return off_layer(c, l); }
static int64_t off_wqkv(const orc_cfg *c, int l) { return off_g1(c, l) + c->d; }
static int64_t off_wo(const orc_cfg *c, int l) { return off_wqkv(c, l) + (int64_t)c->d * qkvw(c); }
static int64_t off_g2(const orc_cfg *c, int l) { return off_wo(c, l) + (int64_t)c->d * c->d; }
static int64_t off_w13(const orc_cfg *c, int l) { return off_g2(c, l) + c->d; }
static int64_t off_w2(const orc_cfg *c, int l) { return off_w13(c, l) + (int64_t)c->d * 2 * c->h; }
static int64_t off_gf(const orc_cfg *c) { return off_layer(c, c->L); }
static int64_t off_wlm(const orc_cfg *c) { return off_gf(c) + c->d; }

/* Writes (offset, rows, cols) for each tensor in layout order; returns count. */
int orc_param_layout(const orc_cfg *c, int64_t *offs, int64_t *rows, int64_t *cols) {
  int n = 0;
#define PUT(o, r, k) do { if (offs) { offs[n] = (o); rows[n] = (r); cols[n] = (k); } n++; } while (0)
  PUT(0, c->V, c->d);
  for (int l = 0; l < c->L; l++) {
    PUT(off_g1(c, l), 1, c->d);
    PUT(off_wqkv(c, l), c->d, qkvw(c));
    PUT(off_wo(c, l), c->d, c->d);
    PUT(off_g2(c, l), 1, c->d);
    PUT(off_w13(c, l), c->d, 2LL * c->h);
    PUT(off_w2(c, l), c->h, c->d);
  }
  PUT(off_gf(c), 1, c->d);
  PUT(off_wlm(c), c->d, c->V);
#undef PUT
  return n;
}

/* ------------------------------------------------------------------ matmul */
/* C[M,N] (=|+=) A[M,K] B[K,N]; leading dimensions given.  Plain definition. */
void orc_mm_nn(int M, int K, int N, const double *A, int64_t lda, const double *B, int64_t ldb,
               double *C, int64_t ldc, int accumulate) {
#pragma omp parallel for schedule(static) if ((int64_t)M * K * N > OMP_MIN_WORK)
  for (int i = 0; i < M; i++) {
    double *c = C + (int64_t)i * ldc;
    if (!accumulate) for (int j = 0; j < N; j++) c[j] = 0.0;
    for (int k = 0; k < K; k++) {
      double a = A[(int64_t)i * lda + k];
      const double *b = B + (int64_t)k * ldb;
      for (int j = 0; j < N; j++) c[j] += a * b[j];
    }
  }
}
/* C[M,N] (=|+=) A[K,M]^T B[K,N]. */
void orc_mm_tn(int M, int K, int N, const double *A, int64_t lda, const double *B, int64_t ldb,
               double *C, int64_t ldc, int accumulate) {
#pragma omp parallel for schedule(static) if ((int64_t)M * K * N > OMP_MIN_WORK)
  for (int i = 0; i < M; i++) {
    double *c = C + (int64_t)i * ldc;
    if (!accumulate) for (int j = 0; j < N; j++) c[j] = 0.0;
    for (int k = 0; k < K; k++) {
      double a = A[(int64_t)k * lda + i];
      const double *b = B + (int64_t)k * ldb;
      for (int j = 0; j < N; j++) c[j] += a * b[j];
    }
  }
}
/* C[M,N] (=|+=) A[M,K] B[N,K]^T. */
void orc_mm_nt(int M, int K, int N, const double *A, int64_t lda, const double *B, int64_t ldb,
               double *C, int64_t ldc, int accumulate) {
#pragma omp parallel for schedule(static) if ((int64_t)M * K * N > OMP_MIN_WORK)
  for (int i = 0; i < M; i++) {
    const double *a = A + (int64_t)i * lda;
    for (int j = 0; j < N; j++) {
      const double *b = B + (int64_t)j * ldb;
      double s = 0.0;
      for (int k = 0; k < K; k++) s += a[k] * b[k];
      C[(int64_t)i * ldc + j] = accumulate ? C[(int64_t)i * ldc + j] + s : s;
    }
  }
}

/* ----------------------------------------------------------------- RMSNorm */
/* Hephaistos, Architecture at a glance (Normalization): scale only, no mean,
 * no bias, rstd cached.  MicroGPT in Rust, RMSNorm: (mean(x^2) + eps)^-1/2. */
void orc_rmsnorm_fwd(int n, int d, const double *x, const double *g, double eps, double *y,
                     double *rstd) {
#pragma omp parallel for schedule(static) if ((int64_t)n * d > OMP_MIN_WORK)
  for (int i = 0; i < n; i++) {
    const double *xi = x + (int64_t)i * d;
    double ss = 0.0;
    for (int j = 0; j < d; j++) ss += xi[j] * xi[j];
    double r = 1.0 / sqrt(ss / d + eps);
    rstd[i] = r;
    for (int j = 0; j < d; j++) y[(int64_t)i * d + j] = g[j] * xi[j] * r;
  }
}
/* Backward of y = g * x * r(x):  dx = r (g*dy) - x r^3 (1/d) sum_j g_j dy_j x_j,
 * dg += sum_rows dy * x * r.  dx is written (accumulate=0) or added to. */
void orc_rmsnorm_bwd(int n, int d, const double *x, const double *rstd, const double *g,
                     const double *dy, double *dx, double *dg, int accumulate) {
#pragma omp parallel for schedule(static) if ((int64_t)n * d > OMP_MIN_WORK)
  for (int i = 0; i < n; i++) {
    const double *xi = x + (int64_t)i * d, *dyi = dy + (int64_t)i * d;
    double r = rstd[i], dot = 0.0;
    for (int j = 0; j < d; j++) dot += g[j] * dyi[j] * xi[j];
    for (int j = 0; j < d; j++) {
      double v = r * g[j] * dyi[j] - xi[j] * r * r * r * dot / d;
      dx[(int64_t)i * d + j] = accumulate ? dx[(int64_t)i * d + j] + v : v;
    }
  }
  for (int i = 0; i < n; i++)
    for (int j = 0; j < d; j++) dg[j] += dy[(int64_t)i * d + j] * x[(int64_t)i * d + j] * rstd[i];
}

/* -------------------------------------------------------------------- RoPE */
/* Rotate-half rotary embedding of one head vector u[hd] at position t
 * (Hephaistos: rotate-half layout; Architecture at a glance: applied to q/k).
 * theta_j = base^(-2j/hd); u'_j = u_j cos - u_{j+hd/2} sin,
 * u'_{j+hd/2} = u_{j+hd/2} cos + u_j sin.  sign = -1 applies the inverse
 * rotation (the backward of the forward rotation). */
/* Rotation at a (possibly fractional) position (strata, RoPE row: position
 * interpolation folds extended positions into the trained range, position
 * t / scale). */
void orc_rope_pos(double *u, int hd, double pos, double base, int sign) {
  int half = hd / 2;
  for (int j = 0; j < half; j++) {
    double theta = pow(base, -2.0 * j / hd);
    double phi = pos * theta;
    double c = cos(phi), s = sign * sin(phi);
    double a = u[j], b = u[j + half];
    u[j] = a * c - b * s;
    u[j + half] = b * c + a * s;
  }
}
void orc_rope(double *u, int hd, int t, double base, int sign) {
  orc_rope_pos(u, hd, (double)t, base, sign);
}

/* --------------------------------------------------------------- attention */
/* Causal attention of one sequence over all heads (Hephaistos: causal
 * multi-head self-attention, numerically stable softmax; strata: n_head and
 * n_kv_head independent).  qkv is [T, d+2kvd] (q heads, then k heads, then v
 * heads), RoPE already applied.  o is [T, d] (heads concatenated).
 * lse[H,T] (optional) is the log-sum-exp of each score row; P[H,T,T]
 * (optional) receives the probabilities (zero above the diagonal). */
static void attention_fwd_do(int T, int d, int H, int Hkv, const double *qkv, double *o,
                             double *lse, double *P, const orc_dropout *dr, int layer, int b);
void orc_attention_fwd(int T, int d, int H, int Hkv, const double *qkv, double *o, double *lse,
                       double *P) {
  attention_fwd_do(T, d, H, Hkv, qkv, o, lse, P, NULL, 0, 0);
}
/* With dr: o_i = sum_j P_ij f_ij v_j, f the dropout factor of probability
 * (b, head, i, j); P and lse stay the undropped softmax. */
static void attention_fwd_do(int T, int d, int H, int Hkv, const double *qkv, double *o,
                             double *lse, double *P, const orc_dropout *dr, int layer, int b) {
  int hd = d / H, grp = H / Hkv;
  int64_t w = (int64_t)d + 2LL * hd * Hkv;
  double scale = 1.0 / sqrt((double)hd);
#pragma omp parallel for collapse(2) schedule(static) if ((int64_t)H * T * T * hd > OMP_MIN_WORK)
  for (int hq = 0; hq < H; hq++) {
    for (int i = 0; i < T; i++) {
      int g = hq / grp;
      const double *q = qkv + (int64_t)i * w + (int64_t)hq * hd;
      double *s = (double *)malloc(sizeof(double) * (i + 1));
      double mx = -INFINITY;
      for (int j = 0; j <= i; j++) {
        const double *k = qkv + (int64_t)j * w + d + (int64_t)g * hd;
        double dot = 0.0;
        for (int e = 0; e < hd; e++) dot += q[e] * k[e];
        s[j] = dot * scale;
        if (s[j] > mx) mx = s[j];
      }
      double sum = 0.0;
      for (int j = 0; j <= i; j++) { s[j] = exp(s[j] - mx); sum += s[j]; }
      double *oi = o + (int64_t)i * d + (int64_t)hq * hd;
      for (int e = 0; e < hd; e++) oi[e] = 0.0;
      for (int j = 0; j <= i; j++) {
        double p = s[j] / sum;
        const double *v = qkv + (int64_t)j * w + d + (int64_t)hd * Hkv + (int64_t)g * hd;
        const double pd =
            dr ? p * drop_factor(dr, 1, layer, (((uint64_t)b * H + hq) * T + i) * T + j) : p;
        for (int e = 0; e < hd; e++) oi[e] += pd * v[e];
        if (P) P[((int64_t)hq * T + i) * T + j] = p;
      }
      if (P) for (int j = i + 1; j < T; j++) P[((int64_t)hq * T + i) * T + j] = 0.0;
      if (lse) lse[(int64_t)hq * T + i] = mx + log(sum);
      free(s);
    }
  }
}

/* Backward of orc_attention_fwd (strata: attention backward rule).  P is
 * recomputed from q and k.  dv_j = sum_i P_ij do_i; dP_ij = do_i . v_j;
 * dS = P (dP - rowsum(dP P)); dq = dS k / sqrt(hd); dk = dS^T q / sqrt(hd).
 * GQA: dk and dv sum over the query heads of the group, in head order.
 * dqkv [T, d+2kvd] is written. */
static void attention_bwd_do(int T, int d, int H, int Hkv, const double *qkv,
                             const double *dout, double *dqkv, const orc_dropout *dr, int layer,
                             int b);
void orc_attention_bwd(int T, int d, int H, int Hkv, const double *qkv, const double *dout,
                       double *dqkv) {
  attention_bwd_do(T, d, H, Hkv, qkv, dout, dqkv, NULL, 0, 0);
}
/* With dr (the mask of attention_fwd_do): dv_j = sum_i P_ij f_ij do_i;
 * dP_ij = f_ij (do_i . v_j); dS = P (dP - rowsum(dP P)). */
static void attention_bwd_do(int T, int d, int H, int Hkv, const double *qkv,
                             const double *dout, double *dqkv, const orc_dropout *dr, int layer,
                             int b) {
  int hd = d / H, grp = H / Hkv;
  int64_t w = (int64_t)d + 2LL * hd * Hkv;
  double scale = 1.0 / sqrt((double)hd);
  double *P = (double *)calloc((size_t)H * T * T, sizeof(double));
  double *dS = (double *)calloc((size_t)H * T * T, sizeof(double));
  double *F = NULL; /* dropout factors [H, T, T] */
  if (dr) {
    F = (double *)calloc((size_t)H * T * T, sizeof(double));
    for (int hq = 0; hq < H; hq++)
      for (int i = 0; i < T; i++)
        for (int j = 0; j <= i; j++)
          F[((int64_t)hq * T + i) * T + j] =
              drop_factor(dr, 1, layer, (((uint64_t)b * H + hq) * T + i) * T + j);
  }
  memset(dqkv, 0, sizeof(double) * (size_t)T * w);
  /* P and dS, one (query head, row) per iteration */
#pragma omp parallel for collapse(2) schedule(static) if ((int64_t)H * T * T * hd > OMP_MIN_WORK)
  for (int hq = 0; hq < H; hq++) {
    for (int i = 0; i < T; i++) {
      int g = hq / grp;
      double *Pi = P + ((int64_t)hq * T + i) * T, *dSi = dS + ((int64_t)hq * T + i) * T;
      const double *q = qkv + (int64_t)i * w + (int64_t)hq * hd;
      const double *doi = dout + (int64_t)i * d + (int64_t)hq * hd;
      double mx = -INFINITY;
      for (int j = 0; j <= i; j++) {
        const double *k = qkv + (int64_t)j * w + d + (int64_t)g * hd;
        double dot = 0.0;
        for (int e = 0; e < hd; e++) dot += q[e] * k[e];
        Pi[j] = dot * scale;
        if (Pi[j] > mx) mx = Pi[j];
      }
      double sum = 0.0;
      for (int j = 0; j <= i; j++) { Pi[j] = exp(Pi[j] - mx); sum += Pi[j]; }
      for (int j = 0; j <= i; j++) Pi[j] /= sum;
      double rs = 0.0;
      for (int j = 0; j <= i; j++) {
        const double *v = qkv + (int64_t)j * w + d + (int64_t)hd * Hkv + (int64_t)g * hd;
        double dp = 0.0;
        for (int e = 0; e < hd; e++) dp += doi[e] * v[e];
        if (F) dp *= F[((int64_t)hq * T + i) * T + j];
        dSi[j] = dp;
        rs += dp * Pi[j];
      }
      for (int j = 0; j <= i; j++) dSi[j] = Pi[j] * (dSi[j] - rs);
      /* dq_i = sum_j dS_ij k_j / sqrt(hd) */
      double *dq = dqkv + (int64_t)i * w + (int64_t)hq * hd;
      for (int j = 0; j <= i; j++) {
        const double *k = qkv + (int64_t)j * w + d + (int64_t)g * hd;
        for (int e = 0; e < hd; e++) dq[e] += dSi[j] * k[e] * scale;
      }
    }
  }
  /* dk_j, dv_j: one (kv head, key row) per iteration, summed over the group's
   * query heads in head order, then over i */
#pragma omp parallel for collapse(2) schedule(static) if ((int64_t)H * T * T * hd > OMP_MIN_WORK)
  for (int g = 0; g < Hkv; g++) {
    for (int j = 0; j < T; j++) {
      double *dk = dqkv + (int64_t)j * w + d + (int64_t)g * hd;
      double *dv = dqkv + (int64_t)j * w + d + (int64_t)hd * Hkv + (int64_t)g * hd;
      for (int hq = g * grp; hq < (g + 1) * grp; hq++) {
        for (int i = j; i < T; i++) {
          const double *q = qkv + (int64_t)i * w + (int64_t)hq * hd;
          const double *doi = dout + (int64_t)i * d + (int64_t)hq * hd;
          double ds = dS[((int64_t)hq * T + i) * T + j], p = P[((int64_t)hq * T + i) * T + j];
          if (F) p *= F[((int64_t)hq * T + i) * T + j];
          for (int e = 0; e < hd; e++) {
            dk[e] += ds * q[e] * scale;
            dv[e] += p * doi[e];
          }
        }
      }
    }
  }
  free(P);
  free(dS);
  free(F);
}

/* ------------------------------------------------------------------ SwiGLU */
/* Hephaistos, Architecture at a glance (Feed-forward): u = silu(a) * b with
 * a = x W1, b = x W3, silu(a) = a / (1 + e^-a). */
void orc_swiglu_fwd(int64_t n, const double *a, const double *b, double *u) {
#pragma omp parallel for schedule(static) if (n > OMP_MIN_WORK)
  for (int64_t i = 0; i < n; i++) u[i] = a[i] / (1.0 + exp(-a[i])) * b[i];
}
/* da = du * b * silu'(a), db = du * silu(a); silu'(a) = s (1 + a (1 - s)),
 * s = 1/(1+e^-a). */
void orc_swiglu_bwd(int64_t n, const double *a, const double *b, const double *du, double *da,
                    double *db) {
#pragma omp parallel for schedule(static) if (n > OMP_MIN_WORK)
  for (int64_t i = 0; i < n; i++) {
    double s = 1.0 / (1.0 + exp(-a[i]));
    da[i] = du[i] * b[i] * s * (1.0 + a[i] * (1.0 - s));
    db[i] = du[i] * a[i] * s;
  }
}

/* ---------------------------------------------------------- cross-entropy */
/* Softmax cross-entropy of rows z[n,V] against targets y[n]; returns the sum
 * of the row losses lse(z_i) - z_i[y_i].  dz (optional) = (softmax(z) -
 * onehot(y)) * inv_count. */
double orc_ce_fwd_bwd(int n, int V, const double *z, const int32_t *y, double inv_count,
                      double *dz) {
  double total = 0.0;
  double *row_loss = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
#pragma omp parallel for schedule(static) if ((int64_t)n * V > OMP_MIN_WORK)
  for (int i = 0; i < n; i++) {
    const double *zi = z + (int64_t)i * V;
    double mx = -INFINITY;
    for (int v = 0; v < V; v++) if (zi[v] > mx) mx = zi[v];
    double s = 0.0;
    for (int v = 0; v < V; v++) s += exp(zi[v] - mx);
    double lse = mx + log(s);
    row_loss[i] = lse - zi[y[i]];
    if (dz)
      for (int v = 0; v < V; v++)
        dz[(int64_t)i * V + v] = (exp(zi[v] - lse) - (v == y[i] ? 1.0 : 0.0)) * inv_count;
  }
  for (int i = 0; i < n; i++) total += row_loss[i];
  free(row_loss);
  return total;
}

/* ------------------------------------------------------- embedding bwd */
/* Gradient of the token-embedding gather (Hephaistos, Architecture at a
 * glance: token embedding): dwte[v,:] = sum over positions t with tok[t] = v
 * of dx[t,:], added in position order; rows of absent ids are zero. */
void orc_embed_bwd(int64_t n, int d, int V, const int32_t *tok, const double *dx, double *dwte) {
  memset(dwte, 0, sizeof(double) * (size_t)V * d);
  for (int64_t t = 0; t < n; t++) {
    double *gw = dwte + (int64_t)tok[t] * d;
    for (int j = 0; j < d; j++) gw[j] += dx[t * d + j];
  }
}

/* -------------------------------------------------------- the whole model */
typedef struct {
  double *x, *xn1, *rstd1, *qkv, *o, *x1, *xn2, *rstd2, *a, *b, *u;
} layer_acts;

/* Forward (and optionally backward) of one sequence.  Logits are written to
 * logits_out[T,V] if non-null; grads (if non-null) are accumulated with the
 * loss scale inv_count.  Returns the sum of this sequence's row losses. */
/* out[t, j] = x[t, j] + f(site, layer, (b*T + t)*d + j) * y[t, j] */
static void add_dropped(const orc_dropout *dr, int site, int layer, int b, int T, int d,
                        const double *x, const double *y, double *out) {
  for (int t = 0; t < T; t++)
    for (int j = 0; j < d; j++) {
      const int64_t i = (int64_t)t * d + j;
      out[i] = x[i] + drop_factor(dr, site, layer, ((uint64_t)b * T + t) * d + j) * y[i];
    }
}
/* dy[t, j] = f(site, layer, (b*T + t)*d + j) * dx[t, j] */
static void mask_rows(const orc_dropout *dr, int site, int layer, int b, int T, int d,
                      const double *dx, double *dy) {
  for (int t = 0; t < T; t++)
    for (int j = 0; j < d; j++) {
      const int64_t i = (int64_t)t * d + j;
      dy[i] = drop_factor(dr, site, layer, ((uint64_t)b * T + t) * d + j) * dx[i];
    }
}

static double seq_step(const orc_cfg *c, const double *p, const int32_t *tok, const int32_t *tgt,
                       double inv_count, double *logits_out, double *grads,
                       const orc_dropout *dr, int bseq) {
  const int T = c->T, d = c->d, L = c->L, H = c->H, Hkv = c->Hkv, h = c->h, V = c->V;
  const int hd = d / H;
  const int64_t w = qkvw(c);
  layer_acts *acts = (layer_acts *)calloc((size_t)(L > 0 ? L : 1), sizeof(layer_acts));
  double *x = (double *)malloc(sizeof(double) * (size_t)T * d);
  /* embedding gather (Hephaistos: token embedding, no positional table) */
  for (int t = 0; t < T; t++)
    memcpy(x + (int64_t)t * d, p + (int64_t)tok[t] * d, sizeof(double) * d);
  if (dr) mask_rows(dr, 0, 0, bseq, T, d, x, x);
  double *ybr = dr ? (double *)malloc(sizeof(double) * (size_t)T * d) : NULL;
  for (int l = 0; l < L; l++) {
    layer_acts *A = &acts[l];
    A->x = x;
    A->xn1 = (double *)malloc(sizeof(double) * (size_t)T * d);
    A->rstd1 = (double *)malloc(sizeof(double) * T);
    A->qkv = (double *)malloc(sizeof(double) * (size_t)T * w);
    A->o = (double *)malloc(sizeof(double) * (size_t)T * d);
    A->x1 = (double *)malloc(sizeof(double) * (size_t)T * d);
    A->xn2 = (double *)malloc(sizeof(double) * (size_t)T * d);
    A->rstd2 = (double *)malloc(sizeof(double) * T);
    A->a = (double *)malloc(sizeof(double) * (size_t)T * h);
    A->b = (double *)malloc(sizeof(double) * (size_t)T * h);
    A->u = (double *)malloc(sizeof(double) * (size_t)T * h);
    /* x1 = x + Attn(RMSNorm_g1(x)) */
    orc_rmsnorm_fwd(T, d, A->x, p + off_g1(c, l), c->eps, A->xn1, A->rstd1);
    orc_mm_nn(T, d, (int)w, A->xn1, d, p + off_wqkv(c, l), w, A->qkv, w, 0);
    for (int t = 0; t < T; t++) {
      const double pos = (double)t / c->rope_scale;
      for (int hq = 0; hq < H; hq++) orc_rope_pos(A->qkv + (int64_t)t * w + (int64_t)hq * hd, hd, pos, c->rope_base, 1);
      for (int g = 0; g < Hkv; g++) orc_rope_pos(A->qkv + (int64_t)t * w + d + (int64_t)g * hd, hd, pos, c->rope_base, 1);
    }
    attention_fwd_do(T, d, H, Hkv, A->qkv, A->o, NULL, NULL, dr, l, bseq);
    if (dr) {
      orc_mm_nn(T, d, d, A->o, d, p + off_wo(c, l), d, ybr, d, 0);
      add_dropped(dr, 2, l, bseq, T, d, A->x, ybr, A->x1);
    } else {
      memcpy(A->x1, A->x, sizeof(double) * (size_t)T * d);
      orc_mm_nn(T, d, d, A->o, d, p + off_wo(c, l), d, A->x1, d, 1);
    }
    /* x2 = x1 + SwiGLU(RMSNorm_g2(x1)) */
    orc_rmsnorm_fwd(T, d, A->x1, p + off_g2(c, l), c->eps, A->xn2, A->rstd2);
    const double *w13 = p + off_w13(c, l);
    orc_mm_nn(T, d, h, A->xn2, d, w13, 2LL * h, A->a, h, 0);
    orc_mm_nn(T, d, h, A->xn2, d, w13 + h, 2LL * h, A->b, h, 0);
    orc_swiglu_fwd((int64_t)T * h, A->a, A->b, A->u);
    double *x2 = (double *)malloc(sizeof(double) * (size_t)T * d);
    if (dr) {
      orc_mm_nn(T, h, d, A->u, h, p + off_w2(c, l), d, ybr, d, 0);
      add_dropped(dr, 3, l, bseq, T, d, A->x1, ybr, x2);
    } else {
      memcpy(x2, A->x1, sizeof(double) * (size_t)T * d);
      orc_mm_nn(T, h, d, A->u, h, p + off_w2(c, l), d, x2, d, 1);
    }
    x = x2;
  }
  /* final RMSNorm, untied lm_head, cross-entropy */
  double *xf = (double *)malloc(sizeof(double) * (size_t)T * d);
  double *rstdf = (double *)malloc(sizeof(double) * T);
  orc_rmsnorm_fwd(T, d, x, p + off_gf(c), c->eps, xf, rstdf);
  double *z = (double *)malloc(sizeof(double) * (size_t)T * V);
  orc_mm_nn(T, d, V, xf, d, p + off_wlm(c), V, z, V, 0);
  if (logits_out) memcpy(logits_out, z, sizeof(double) * (size_t)T * V);
  double *dz = grads ? (double *)malloc(sizeof(double) * (size_t)T * V) : NULL;
  double loss = tgt ? orc_ce_fwd_bwd(T, V, z, tgt, inv_count, dz) : 0.0;

  if (grads) {
    double *dx = (double *)malloc(sizeof(double) * (size_t)T * d);
    double *dxf = (double *)malloc(sizeof(double) * (size_t)T * d);
    /* lm_head: dWlm += xf^T dz, dxf = dz Wlm^T */
    orc_mm_tn(d, T, V, xf, d, dz, V, grads + off_wlm(c), V, 1);
    orc_mm_nt(T, V, d, dz, V, p + off_wlm(c), V, dxf, d, 0);
    orc_rmsnorm_bwd(T, d, x, rstdf, p + off_gf(c), dxf, dx, grads + off_gf(c), 0);
    double *dxn = (double *)malloc(sizeof(double) * (size_t)T * d);
    double *du = (double *)malloc(sizeof(double) * (size_t)T * h);
    double *da = (double *)malloc(sizeof(double) * (size_t)T * h);
    double *db = (double *)malloc(sizeof(double) * (size_t)T * h);
    double *dO = (double *)malloc(sizeof(double) * (size_t)T * d);
    double *dqkv = (double *)malloc(sizeof(double) * (size_t)T * w);
    for (int l = L - 1; l >= 0; l--) {
      layer_acts *A = &acts[l];
      /* dx holds d loss / d x2 (layer output). FFN branch (its output's
       * gradient is dx through the dropout mask): */
      const double *dyf = dx;
      if (dr) {
        mask_rows(dr, 3, l, bseq, T, d, dx, ybr);
        dyf = ybr;
      }
      orc_mm_tn(h, T, d, A->u, h, dyf, d, grads + off_w2(c, l), d, 1);
      orc_mm_nt(T, d, h, dyf, d, p + off_w2(c, l), d, du, h, 0);
      orc_swiglu_bwd((int64_t)T * h, A->a, A->b, du, da, db);
      double *g13 = grads + off_w13(c, l);
      const double *w13 = p + off_w13(c, l);
      orc_mm_tn(d, T, h, A->xn2, d, da, h, g13, 2LL * h, 1);
      orc_mm_tn(d, T, h, A->xn2, d, db, h, g13 + h, 2LL * h, 1);
      orc_mm_nt(T, h, d, da, h, w13, 2LL * h, dxn, d, 0);
      orc_mm_nt(T, h, d, db, h, w13 + h, 2LL * h, dxn, d, 1);
      /* residual: dx1 = dx2 + RMSNorm_bwd(dxn) */
      orc_rmsnorm_bwd(T, d, A->x1, A->rstd2, p + off_g2(c, l), dxn, dx, grads + off_g2(c, l), 1);
      /* attention branch */
      const double *dya = dx;
      if (dr) {
        mask_rows(dr, 2, l, bseq, T, d, dx, ybr);
        dya = ybr;
      }
      orc_mm_tn(d, T, d, A->o, d, dya, d, grads + off_wo(c, l), d, 1);
      orc_mm_nt(T, d, d, dya, d, p + off_wo(c, l), d, dO, d, 0);
      attention_bwd_do(T, d, H, Hkv, A->qkv, dO, dqkv, dr, l, bseq);
      for (int t = 0; t < T; t++) {
        const double pos = (double)t / c->rope_scale;
        for (int hq = 0; hq < H; hq++) orc_rope_pos(dqkv + (int64_t)t * w + (int64_t)hq * hd, hd, pos, c->rope_base, -1);
        for (int g = 0; g < Hkv; g++) orc_rope_pos(dqkv + (int64_t)t * w + d + (int64_t)g * hd, hd, pos, c->rope_base, -1);
      }
      orc_mm_tn(d, T, (int)w, A->xn1, d, dqkv, w, grads + off_wqkv(c, l), w, 1);
      orc_mm_nt(T, (int)w, d, dqkv, w, p + off_wqkv(c, l), w, dxn, d, 0);
      orc_rmsnorm_bwd(T, d, A->x, A->rstd1, p + off_g1(c, l), dxn, dx, grads + off_g1(c, l), 1);
    }
    /* embedding scatter-add: dwte[tok_t] += dx0_t, in token order (through
     * the embedding dropout mask) */
    if (dr) mask_rows(dr, 0, 0, bseq, T, d, dx, dx);
    for (int t = 0; t < T; t++) {
      double *gw = grads + (int64_t)tok[t] * d;
      for (int j = 0; j < d; j++) gw[j] += dx[(int64_t)t * d + j];
    }
    free(dx); free(dxf); free(dxn); free(du); free(da); free(db); free(dO); free(dqkv);
  }
  /* free activations; acts[0].x is the embedding output, acts[l].x for l>0
   * is the previous layer's x2 */
  for (int l = 0; l < L; l++) {
    layer_acts *A = &acts[l];
    free(A->x); free(A->xn1); free(A->rstd1); free(A->qkv); free(A->o); free(A->x1);
    free(A->xn2); free(A->rstd2); free(A->a); free(A->b); free(A->u);
  }
  free(x);
  if (L == 0) { /* x was never handed to a layer record */ }
  free(xf); free(rstdf); free(z); free(dz); free(acts); free(ybr);
  return loss;
}

/* Loss (mean over all B*T positions), logits[B*T, V] (optional) and grads[P]
 * (optional, overwritten) for tokens/targets [B, T] and params[P]. */
static double forward_backward(const orc_cfg *c, const double *params, const int32_t *tokens,
                               const int32_t *targets, double *logits, double *grads,
                               const orc_dropout *dr) {
  int64_t P = orc_n_params(c);
  int64_t N = (int64_t)c->B * c->T;
  if (grads) memset(grads, 0, sizeof(double) * (size_t)P);
  double total = 0.0;
  for (int b = 0; b < c->B; b++)
    total += seq_step(c, params, tokens + (int64_t)b * c->T, targets ? targets + (int64_t)b * c->T : NULL,
                      1.0 / (double)N, logits ? logits + (int64_t)b * c->T * c->V : NULL, grads,
                      dr, b);
  return total / (double)N;
}
double orc_forward_backward(const orc_cfg *c, const double *params, const int32_t *tokens,
                            const int32_t *targets, double *logits, double *grads) {
  return forward_backward(c, params, tokens, targets, logits, grads, NULL);
}
/* The training forward and backward with inverted dropout of rate p at the
 * four sites (see orc_philox4x32_10 above); masks keyed by seed and step. */
double orc_forward_backward_dropout(const orc_cfg *c, const double *params,
                                    const int32_t *tokens, const int32_t *targets,
                                    double *logits, double *grads, double p, uint64_t seed,
                                    uint32_t step) {
  orc_dropout dr = {p, seed, step};
  return forward_backward(c, params, tokens, targets, logits, grads, &dr);
}
/* Dropout factors (0 or 1/(1-p)) of elements [e0, e0 + n) of (site, layer). */
void orc_dropout_factors(double p, uint64_t seed, uint32_t step, int site, int layer,
                         uint64_t e0, int64_t n, double *out) {
  orc_dropout dr = {p, seed, step};
  for (int64_t i = 0; i < n; i++) out[i] = drop_factor(&dr, site, layer, e0 + (uint64_t)i);
}

/* ------------------------------------------------------------------- AdamW */
/* Hephaistos, Architecture at a glance (Optimizer): AdamW with decoupled
 * weight decay and bias correction; strata, capability table (AdamW).
 * m = b1 m + (1-b1) g;  v = b2 v + (1-b2) g^2;  mh = m/(1-b1^t);
 * vh = v/(1-b2^t);  p = p - lr wd p - lr mh/(sqrt(vh) + eps), t 1-based. */
void orc_adamw(int64_t n, double *p, const double *g, double *m, double *v, int64_t t, double lr,
               double wd, double b1, double b2, double eps) {
  double bc1 = 1.0 - pow(b1, (double)t), bc2 = 1.0 - pow(b2, (double)t);
#pragma omp parallel for schedule(static) if (n > OMP_MIN_WORK)
  for (int64_t i = 0; i < n; i++) {
    m[i] = b1 * m[i] + (1.0 - b1) * g[i];
    v[i] = b2 * v[i] + (1.0 - b2) * g[i] * g[i];
    double mh = m[i] / bc1, vh = v[i] / bc2;
    p[i] = p[i] - lr * wd * p[i] - lr * mh / (sqrt(vh) + eps);
  }
}
