// Single-token decode against the key/value cache, and the token sampler.
//
// Hephaistos, feature list ("True KV Cache"): the prompt is run once, then each
// new position costs one pass of every projection over a single row per
// sequence; strata, model table: the cached keys are stored already rotated.
// The cache is the forward pass's own [B*T, q|k|v] activation buffer of every
// layer (RoPE applied to q and k), so a forward over the prompt is the prefill
// and a decode call writes row (b, pos) of it.
//
// With B rows per call the projections are matrix-vector products bound by
// reading the weights once: k_gemv streams W in 128-column blocks split over
// K (one wave of two blocks per SM), each thread multiplying 8 columns of W by the
// block's B rows held in shared memory, with the RMSNorm of the input row
// applied while the rows are staged.  The K slices' partial sums are added in
// slice order by the last block of a column block to finish (a counter per
// column block), which then applies the epilogue: RoPE + cache store for the
// q|k|v projection, residual add, SwiGLU, or the fp32 logits.  Attention of
// the new query against positions 0..pos is split over 128-key chunks staged
// in shared memory by asynchronous copies; the last chunk of a (sequence,
// key/value head) to finish merges them in order.
// Every sum has a fixed order: a decode call is bit-reproducible.
#include <limits.h>
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace llm {

namespace {

constexpr int GV_THREADS = 256;
constexpr int GV_COLS = 128;     // columns of W per block
constexpr int GV_CG = 16;        // column groups of 8 per block
constexpr int GV_KL = 16;        // k lanes per block (GV_THREADS / GV_CG)
constexpr int GV_MB = 8;         // rows of A per pass
constexpr int GV_UNROLL = 4;     // W rows in flight per thread
constexpr int GV_KSLICE_MAX = 1024;
constexpr int GV_KS_MAX = 16;    // K slices (partials the finishing block adds)
constexpr int GV_SMEM_FLOATS = GV_MB * GV_KSLICE_MAX;  // A slice, then the warp partials
static_assert(GV_SMEM_FLOATS >= (GV_THREADS / 32) * GV_MB * GV_COLS, "reduction space");
static_assert(GV_CG * GV_KL == GV_THREADS && 8 * GV_CG == GV_COLS, "thread layout");

constexpr int AT_KEYS = 128;     // keys per attention block (one per thread when scoring)
constexpr int AT_THREADS = 128;

constexpr int SP_THREADS = 1024;
constexpr int SP_PEN_BYTES = 64 * 1024;  // history bitmap of the penalty: ids < 524288

inline unsigned cdiv(int64_t a, int64_t b) { return (unsigned)((a + b - 1) / b); }

// Programmatic dependent launch: the next kernel of the stream may be
// scheduled once every block of this one has passed pdl_release(); it runs
// its independent prologue (weight loads) and then pdl_wait() blocks until
// this grid has completed and its writes are visible.  Without the launch
// attribute both are no-ops.
LLM_DEV void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
LLM_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

LLM_DEV void bf16x8(uint4 q, float (&f)[8]) {
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&q);
#pragma unroll
  for (int k = 0; k < 4; k++) {
    const float2 t = __bfloat1622float2(h[k]);
    f[2 * k] = t.x;
    f[2 * k + 1] = t.y;
  }
}
// 8 consecutive values from p; one or two 16-byte loads when vec (aligned
// and all 8 inside the row), else element by element up to n.
LLM_DEV void load8(const __nv_bfloat16 *p, bool vec, int n, float (&w)[8]) {
  if (vec && n >= 8) {
    bf16x8(__ldg(reinterpret_cast<const uint4 *>(p)), w);
  } else {
#pragma unroll
    for (int k = 0; k < 8; k++) w[k] = k < n ? __bfloat162float(p[k]) : 0.f;
  }
}
LLM_DEV void load8(const float *p, bool vec, int n, float (&w)[8]) {
  if (vec && n >= 8) {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
    const float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else {
#pragma unroll
    for (int k = 0; k < 8; k++) w[k] = k < n ? p[k] : 0.f;
  }
}

// Epilogue of rows [b0, b0 + mb) x columns [n0, n0 + 128) whose sums are in
// v[r * GV_COLS + c].
template <typename A>
LLM_DEV void gemv_epilogue(const GemvArgs &a, const float *v, int b0, int mb, int n0) {
  for (int idx = threadIdx.x; idx < GV_MB * GV_COLS; idx += GV_THREADS) {
    const int r = idx / GV_COLS, c = idx % GV_COLS, n = n0 + c;
    if (r >= mb) continue;
    const int64_t b = b0 + r;
    const float y = v[idx];
    if (a.epi == DEC_QKV) {
      // Hephaistos, Architecture at a glance (Positions): q and k of head
      // columns rotate pairs (j, j + hd/2) by pos * theta_j; heads do not
      // straddle the block (hd divides 128).
      if (n >= a.nvalid) continue;
      const int t = *a.pos;
      float o = y;
      if (n < a.rot_cols) {
        const int half = a.hd / 2, e = n % a.hd, j = e % half, cb = c - e;
        const float cs = a.cos_t[(int64_t)t * half + j], sn = a.sin_t[(int64_t)t * half + j];
        const float x0 = v[r * GV_COLS + cb + j], x1 = v[r * GV_COLS + cb + j + half];
        o = e < half ? x0 * cs - x1 * sn : x1 * cs + x0 * sn;
      }
      reinterpret_cast<A *>(a.out)[b * a.ldo + (int64_t)t * a.pos_stride + n] = from_f<A>(o);
    } else if (a.epi == DEC_RESID) {
      if (n < a.nvalid) reinterpret_cast<float *>(a.out)[b * a.ldo + n] += y;
    } else if (a.epi == DEC_SWIGLU) {
      // interleaved W1|W3 blocks of 64 columns: a in the first half of the
      // block, its b 64 columns further (Hephaistos, Architecture at a
      // glance: u = silu(a) * b); a and b rounded like the saved activations
      if (c >= SWIGLU_BLOCK) continue;
      const int64_t j = (int64_t)(n0 / (2 * SWIGLU_BLOCK)) * SWIGLU_BLOCK + c;
      if (j >= a.nvalid) continue;
      const float av = to_f(from_f<A>(y)), bv = to_f(from_f<A>(v[idx + SWIGLU_BLOCK]));
      reinterpret_cast<A *>(a.out)[b * a.ldo + j] = from_f<A>(av * sigmoidf_(av) * bv);
    } else {  // DEC_LOGITS
      if (n < a.nvalid) reinterpret_cast<float *>(a.out)[b * a.ldo + n] = y;
    }
  }
}

// y[b, n] = sum_k A[b, k] W[k, n] for B rows; grid (column blocks, K slices).
template <typename A>
__global__ void __launch_bounds__(GV_THREADS) k_gemv(const GemvArgs a) {
  __shared__ __align__(16) float sm[GV_SMEM_FLOATS];
  __shared__ float rs[GV_MB];
  __shared__ int last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cg = tid % GV_CG, kl = tid / GV_CG;
  const int n0 = blockIdx.x * GV_COLS, ksi = blockIdx.y;
  const int k0 = ksi * a.kslice, k1 = min(a.K, k0 + a.kslice), kn = k1 - k0;
  const int nc = n0 + 8 * cg;
  const int ncols = max(0, min(8, a.N - nc));
  const A *W = reinterpret_cast<const A *>(a.W);
  const bool vec = a.vec != 0;
  float w[GV_UNROLL][8];
  auto load_w = [&](int k) {
#pragma unroll
    for (int u = 0; u < GV_UNROLL; u++) {
      const int kk = k + u * GV_KL;
      if (kk < k1 && ncols > 0) {
        load8(W + (int64_t)kk * a.ldw + nc, vec, ncols, w[u]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; j++) w[u][j] = 0.f;
      }
    }
  };
  pdl_release();
  // the weights are never written by the kernels before this one: the first
  // batch of this thread's rows is in flight before waiting for them
  load_w(k0 + kl);
  pdl_wait();
  for (int b0 = 0; b0 < a.B; b0 += GV_MB) {
    const int mb = min(GV_MB, a.B - b0);
    // ---- the rows' K slice in shared memory, in operand precision
    if (a.gain) {
      // Hephaistos, Architecture at a glance (Normalization): r = (mean x^2 +
      // eps)^-1/2, A = g * x * r, over the whole row (K = d)
      // (x rows are 16-byte aligned and K = d is a multiple of 4)
      if (warp < mb) {
        const float4 *xr = reinterpret_cast<const float4 *>(a.x + (int64_t)(b0 + warp) * a.ldx);
        float ss = 0.f;
#pragma unroll 8
        for (int j = lane; j < a.K / 4; j += 32) {
          const float4 v = xr[j];
          ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
        }
        ss = warp_sum(ss);
        if (lane == 0) rs[warp] = 1.0f / sqrtf(ss / (float)a.K + a.eps);
      }
      __syncthreads();
    }
#pragma unroll 4
    for (int i = tid; i < GV_MB * kn; i += GV_THREADS) {
      const int r = i / kn, k = k0 + i % kn;
      float v = 0.f;
      if (r < mb) {
        const int64_t row = b0 + r;
        v = a.gain ? to_f(from_f<A>(a.gain[k] * a.x[row * a.ldx + k] * rs[r]))
                   : to_f(reinterpret_cast<const A *>(a.xa)[row * a.ldxa + k]);
      }
      sm[i] = v;
    }
    __syncthreads();
    // ---- products: this thread's 8 columns over rows k0 + kl, + 16, ...
    float acc[GV_MB][8];
#pragma unroll
    for (int r = 0; r < GV_MB; r++)
#pragma unroll
      for (int j = 0; j < 8; j++) acc[r][j] = 0.f;
    for (int k = k0 + kl; k < k1; k += GV_KL * GV_UNROLL) {
      if (b0 > 0 || k > k0 + kl) load_w(k);  // the first batch was loaded up front
#pragma unroll
      for (int u = 0; u < GV_UNROLL; u++) {
        const int kk = k + u * GV_KL;
        if (kk < k1) {
#pragma unroll
          for (int r = 0; r < GV_MB; r++) {
            const float xv = sm[r * kn + (kk - k0)];
#pragma unroll
            for (int j = 0; j < 8; j++) acc[r][j] = fmaf(xv, w[u][j], acc[r][j]);
          }
        }
      }
    }
    __syncthreads();  // the A slice is no longer read: its space takes the partials
    // ---- k lanes: the two of a warp by shuffle, then the 8 warps in order
#pragma unroll
    for (int r = 0; r < GV_MB; r++)
#pragma unroll
      for (int j = 0; j < 8; j++) acc[r][j] += __shfl_xor_sync(0xffffffffu, acc[r][j], 16);
    if (lane < 16) {
#pragma unroll
      for (int r = 0; r < GV_MB; r++)
#pragma unroll
        for (int j = 0; j < 8; j++) sm[(warp * GV_MB + r) * GV_COLS + 8 * cg + j] = acc[r][j];
    }
    __syncthreads();
    float fin[GV_MB * GV_COLS / GV_THREADS];
#pragma unroll
    for (int i = 0; i < GV_MB * GV_COLS / GV_THREADS; i++) {
      const int idx = tid + GV_THREADS * i, r = idx / GV_COLS, c = idx % GV_COLS;
      float s = 0.f;
#pragma unroll
      for (int w8 = 0; w8 < GV_THREADS / 32; w8++) s += sm[(w8 * GV_MB + r) * GV_COLS + c];
      fin[i] = s;
    }
    __syncthreads();
    if (a.ks == 1) {
#pragma unroll
      for (int i = 0; i < GV_MB * GV_COLS / GV_THREADS; i++) sm[tid + GV_THREADS * i] = fin[i];
      __syncthreads();
      gemv_epilogue<A>(a, sm, b0, mb, n0);
    } else {
#pragma unroll
      for (int i = 0; i < GV_MB * GV_COLS / GV_THREADS; i++) {
        const int idx = tid + GV_THREADS * i, r = idx / GV_COLS, c = idx % GV_COLS;
        if (r < mb && n0 + c < a.N)
          a.part[((int64_t)ksi * a.B + b0 + r) * a.N + n0 + c] = fin[i];
      }
    }
    __syncthreads();
  }
  if (a.ks == 1) return;
  // ---- the last K slice of this column block to finish adds the partials
  // in slice order and applies the epilogue
  __threadfence();
  __syncthreads();
  if (tid == 0) last = atomicAdd(&a.count[blockIdx.x], 1u) == (unsigned)(a.ks - 1);
  __syncthreads();
  if (!last) return;
  __threadfence();
  constexpr int PER = GV_MB * GV_COLS / GV_THREADS;
  const int64_t qstride = (int64_t)a.B * a.N;
  for (int b0 = 0; b0 < a.B; b0 += GV_MB) {
    const int mb = min(GV_MB, a.B - b0);
    const float *pp[PER];
    bool ok[PER];
    float sum[PER];
#pragma unroll
    for (int i = 0; i < PER; i++) {
      const int idx = tid + GV_THREADS * i, r = idx / GV_COLS, c = idx % GV_COLS;
      ok[i] = r < mb && n0 + c < a.N;
      pp[i] = a.part + ((int64_t)b0 + r) * a.N + n0 + c;
      sum[i] = 0.f;
    }
    // every slice of this thread's outputs in flight at once, then added in
    // slice order (past the last slice a zero is added: the sum is unchanged)
    float v[PER][GV_KS_MAX];
#pragma unroll
    for (int i = 0; i < PER; i++)
#pragma unroll
      for (int q = 0; q < GV_KS_MAX; q++)
        v[i][q] = (ok[i] && q < a.ks) ? __ldcg(pp[i] + q * qstride) : 0.f;
#pragma unroll
    for (int i = 0; i < PER; i++)
#pragma unroll
      for (int q = 0; q < GV_KS_MAX; q++) sum[i] += v[i][q];
#pragma unroll
    for (int i = 0; i < PER; i++) sm[tid + GV_THREADS * i] = sum[i];
    __syncthreads();
    gemv_epilogue<A>(a, sm, b0, mb, n0);
    __syncthreads();
  }
  if (tid == 0) a.count[blockIdx.x] = 0u;  // ready for the next launch
}

// ----------------------------------------------------------- attention
// Hephaistos, Architecture at a glance (Attention): the query of position pos
// attends to keys 0..pos with weights softmax(q.k / sqrt(hd)); strata: query
// head h reads key/value head h / (H / H_kv).  Block (chunk c of 128 keys,
// key/value head g, sequence b).  The chunk's key and value rows are staged in
// shared memory (rows padded by 16 bytes) by asynchronous 16-byte copies: the
// rows before pos were written by earlier calls, so their copies are issued
// before waiting for the kernel before (which writes q and row pos).  The
// group's query heads go in passes of GT; scores are kept in base 2 (q
// pre-scaled by log2(e) / sqrt(hd)).  Each block writes per head its chunk
// maximum m, sum l of 2^(s - m) and o = sum 2^(s - m) v; the last chunk of
// (b, g) to finish merges the chunks in order:
// o = sum_c 2^(m_c - M) o_c / sum_c 2^(m_c - M) l_c.
constexpr int AT_HDMAX = 128;
constexpr int AT_MERGE = 16;  // chunks whose records are loaded together in the merge

LLM_DEV uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
LLM_DEV void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src)
               : "memory");
}
LLM_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// 8 values of a staged row (16-byte aligned when vec), element by element up to n
LLM_DEV void smem8(const __nv_bfloat16 *p, bool vec, int n, float (&w)[8]) {
  if (vec && n >= 8) {
    bf16x8(*reinterpret_cast<const uint4 *>(p), w);
  } else {
#pragma unroll
    for (int k = 0; k < 8; k++) w[k] = k < n ? __bfloat162float(p[k]) : 0.f;
  }
}
LLM_DEV void smem8(const float *p, bool vec, int n, float (&w)[8]) {
  if (vec && n >= 8) {
    const float4 a = reinterpret_cast<const float4 *>(p)[0];
    const float4 b = reinterpret_cast<const float4 *>(p)[1];
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else {
#pragma unroll
    for (int k = 0; k < 8; k++) w[k] = k < n ? p[k] : 0.f;
  }
}
// Bytes of one staged row (a multiple of 16, plus 16 so rows fall on
// different banks) and of the block's dynamic shared memory.
__host__ __device__ inline int attn_row_bytes(int hd, int esz) {
  return (hd * esz + 15) / 16 * 16 + 16;
}

template <typename A, int GT>
__global__ void __launch_bounds__(AT_THREADS, 4)
    k_attn_decode(const A *__restrict__ qkv, int64_t qkvw, int T, const int *__restrict__ pos_p,
                  int H, int Hkv, int hd, int nch, int vec, float *__restrict__ part,
                  unsigned *__restrict__ count, A *__restrict__ out) {
  extern __shared__ __align__(16) uint8_t kv_sm[];
  __shared__ __align__(16) float qs[GT][AT_HDMAX];
  __shared__ float ps[GT][AT_KEYS];
  __shared__ float wm[AT_THREADS / 32][GT], wl[AT_THREADS / 32][GT];
  __shared__ int last;
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  pdl_release();
  // the position word is written before the decode kernels start
  const int pos = *pos_p;
  const int j0 = c * AT_KEYS;
  if (j0 > pos) return;
  const int nk = min(AT_KEYS, pos + 1 - j0);
  const int nold = min(nk, pos - j0);  // rows of this chunk written by earlier calls
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = H / Hkv, d = H * hd, kvd = Hkv * hd;
  const int esz = (int)sizeof(A), RS = attn_row_bytes(hd, esz);
  uint8_t *Ks = kv_sm, *Vs = kv_sm + AT_KEYS * RS;
  const A *kb = qkv + ((int64_t)b * T + j0) * qkvw + d + (int64_t)g * hd;
  const A *vb = kb + kvd;
  const int cpr = hd * esz / 16;  // 16-byte pieces of a row (vec)
  auto stage = [&](int ja, int jb) {  // rows [ja, jb) of the chunk
    if (vec) {
      for (int i = tid; i < (jb - ja) * cpr; i += AT_THREADS) {
        const int j = ja + i / cpr, q = i % cpr;
        cp_async16(Ks + j * RS + 16 * q, reinterpret_cast<const uint8_t *>(kb + (int64_t)j * qkvw) + 16 * q);
        cp_async16(Vs + j * RS + 16 * q, reinterpret_cast<const uint8_t *>(vb + (int64_t)j * qkvw) + 16 * q);
      }
    } else {
      for (int i = tid; i < (jb - ja) * hd; i += AT_THREADS) {
        const int j = ja + i / hd, e = i % hd;
        reinterpret_cast<A *>(Ks + j * RS)[e] = kb[(int64_t)j * qkvw + e];
        reinterpret_cast<A *>(Vs + j * RS)[e] = vb[(int64_t)j * qkvw + e];
      }
    }
  };
  stage(0, nold);
  pdl_wait();  // q and row pos come from the kernel before
  stage(nold, nk);
  cp_async_wait_all();
  const float scale = 1.4426950408889634f / sqrtf((float)hd);
  const A *rowq = qkv + ((int64_t)b * T + pos) * qkvw;
  for (int r0 = 0; r0 < G; r0 += GT) {
    const int nr = min(GT, G - r0);
    for (int i = tid; i < GT * hd; i += AT_THREADS) {
      const int r = i / hd, e = i % hd;
      qs[r][e] = r < nr ? to_f(rowq[(int64_t)(g * G + r0 + r) * hd + e]) * scale : 0.f;
    }
    __syncthreads();  // q, and every thread's staged rows
    // scores: one key per thread
    float s[GT];
#pragma unroll
    for (int r = 0; r < GT; r++) s[r] = 0.f;
    if (tid < nk) {
      const A *kr = reinterpret_cast<const A *>(Ks + tid * RS);
      for (int e = 0; e < hd; e += 8) {
        float kv[8];
        smem8(kr + e, vec != 0, hd - e, kv);
#pragma unroll
        for (int r = 0; r < GT; r++) {
          float t = s[r];
#pragma unroll
          for (int q = 0; q < 8; q++)
            if (e + q < hd) t = fmaf(qs[r][e + q], kv[q], t);
          s[r] = t;
        }
      }
    }
    // chunk maximum and sum per query head (warps, then the 4 warps in order)
#pragma unroll
    for (int r = 0; r < GT; r++) {
      const float m = warp_max(tid < nk ? s[r] : -INFINITY);
      if (lane == 0) wm[warp][r] = m;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < GT; r++) {
      const float m = fmaxf(fmaxf(wm[0][r], wm[1][r]), fmaxf(wm[2][r], wm[3][r]));
      const float p = tid < nk ? exp2f(s[r] - m) : 0.f;
      ps[r][tid] = p;
      const float l = warp_sum(p);
      if (lane == 0) wl[warp][r] = l;
    }
    __syncthreads();
    // o[r][e] = sum_j p_j v_j[e], keys in order, one output per thread
    for (int idx = tid; idx < nr * hd; idx += AT_THREADS) {
      const int r = idx / hd, e = idx % hd;
      const uint8_t *vc = Vs + e * esz;
      float o = 0.f;
#pragma unroll 8
      for (int jj = 0; jj < nk; jj++)
        o = fmaf(ps[r][jj], to_f(*reinterpret_cast<const A *>(vc + jj * RS)), o);
      float *rec = part + ((((int64_t)b * Hkv + g) * nch + c) * G + r0 + r) * (hd + 2);
      rec[2 + e] = o;
      if (e == 0) {
        rec[0] = fmaxf(fmaxf(wm[0][r], wm[1][r]), fmaxf(wm[2][r], wm[3][r]));
        rec[1] = ((wl[0][r] + wl[1][r]) + wl[2][r]) + wl[3][r];
      }
    }
    __syncthreads();
  }
  // ---- the last chunk of (b, g) to finish merges the chunks in order
  const int nc = pos / AT_KEYS + 1;
  __threadfence();
  __syncthreads();
  if (tid == 0) last = atomicAdd(&count[b * Hkv + g], 1u) == (unsigned)(nc - 1);
  __syncthreads();
  if (!last) return;
  __threadfence();
  const int64_t stride = (int64_t)G * (hd + 2);
  for (int idx = tid; idx < G * hd; idx += AT_THREADS) {
    const int r = idx / hd, e = idx % hd;
    const float *rec0 = part + (((int64_t)b * Hkv + g) * nch * G + r) * (hd + 2);
    float M = -INFINITY;
    for (int c0 = 0; c0 < nc; c0 += AT_MERGE) {
      float mv[AT_MERGE];
#pragma unroll
      for (int u = 0; u < AT_MERGE; u++)
        mv[u] = c0 + u < nc ? __ldcg(rec0 + (c0 + u) * stride) : -INFINITY;
#pragma unroll
      for (int u = 0; u < AT_MERGE; u++) M = fmaxf(M, mv[u]);
    }
    float L = 0.f, o = 0.f;
    for (int c0 = 0; c0 < nc; c0 += AT_MERGE) {
      float mv[AT_MERGE], lv[AT_MERGE], ov[AT_MERGE];
#pragma unroll
      for (int u = 0; u < AT_MERGE; u++) {
        const bool in = c0 + u < nc;
        const float *rc = rec0 + (c0 + u) * stride;
        mv[u] = in ? __ldcg(rc) : 0.f;
        lv[u] = in ? __ldcg(rc + 1) : 0.f;
        ov[u] = in ? __ldcg(rc + 2 + e) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < AT_MERGE; u++) {
        if (c0 + u < nc) {
          const float f = exp2f(mv[u] - M);
          L = fmaf(f, lv[u], L);
          o = fmaf(f, ov[u], o);
        }
      }
    }
    out[(int64_t)b * H * hd + (int64_t)(g * G + r) * hd + e] = from_f<A>(o / L);
  }
  if (tid == 0) count[b * Hkv + g] = 0u;  // ready for the next launch
}

// ------------------------------------------------------------- sampling
// Hephaistos, Sampling (temperature + top-k).  Readings: temperature <= 0 or
// top_k == 1 is greedy (lowest id among equal maxima); the top-k set is the
// first k ids ordered by (logit descending, id ascending); weights
// exp((z - max z) / temperature); the draw is the smallest id of the set, in
// increasing id order, whose cumulative weight exceeds u * total.  One block
// per row; thread t owns the contiguous ids [t*chunk, (t+1)*chunk).
LLM_DEV uint32_t order_key(float f) {  // unsigned order = float order
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
LLM_DEV float sample_weight(float z, float zmax, float temperature) {
  return expf((z - zmax) / temperature);
}
// Extensions (llm_sample_ex), applied only by the EXT instantiation
// (Transformer-In-Rust, sampling pipeline: repetition penalty, temperature,
// top-k, top-p; strata and randyGPT: top-p).  The penalty divides a positive
// logit of an id present in the row's history by `penalty` and multiplies a
// negative one, before everything else (float32, the logits' precision).  Top-p
// keeps, inside the top-k set walked in (logit descending, id ascending)
// order, the shortest prefix whose weight reaches top_p of the set's total;
// the set is sorted in shared memory, so top_k <= SP_NUC_MAX.
constexpr int SP_NUC_MAX = 1024;
struct SampleExt {
  float top_p = 1.f;
  float penalty = 1.f;
  const int32_t *hist = nullptr;
  int64_t hist_ld = 0;
  int hist_len = 0;
};
LLM_DEV unsigned long long sort_composite(uint32_t key, int id) {  // (key desc, id asc) = desc
  return ((unsigned long long)key << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)id);
}

template <bool EXT>
__global__ void __launch_bounds__(SP_THREADS)
    k_sample(const float *__restrict__ logits, int64_t ld, int V, float temperature, int top_k,
             const float *__restrict__ uni, int32_t *__restrict__ out, const SampleExt ext) {
  extern __shared__ uint32_t pen_bits[];  // EXT with a penalty: one bit per id of the history
  __shared__ float sv[32];
  __shared__ int si[32];
  __shared__ unsigned hist[256];
  __shared__ unsigned s_prefix, s_rem;
  __shared__ unsigned eqc[SP_THREADS];
  __shared__ float wsum[SP_THREADS];
  __shared__ int s_owner;
  __shared__ float s_tl;
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float *z = logits + (int64_t)b * ld;
  const int chunk = (V + SP_THREADS - 1) / SP_THREADS;
  const int lo = min(V, tid * chunk), hi = min(V, lo + chunk);
  bool pen = false;
  if constexpr (EXT) {
    pen = ext.penalty != 1.f && ext.hist_len > 0;
    if (pen) {
      for (int w = tid; w < (V + 31) / 32; w += SP_THREADS) pen_bits[w] = 0u;
      __syncthreads();
      const int32_t *h = ext.hist + (int64_t)b * ext.hist_ld;
      for (int j = tid; j < ext.hist_len; j += SP_THREADS) {
        const int id = h[j];
        if (id >= 0 && id < V) atomicOr(&pen_bits[id >> 5], 1u << (id & 31));
      }
      __syncthreads();
    }
  }
  auto zval = [&](int i) -> float {  // the (penalised) logit of id i
    float v = z[i];
    if constexpr (EXT) {
      if (pen && ((pen_bits[i >> 5] >> (i & 31)) & 1u))
        v = v > 0.f ? v / ext.penalty : v * ext.penalty;
    }
    return v;
  };
  // maximum and its lowest id
  float bv = -INFINITY;
  int bi = INT_MAX;
  for (int i = lo; i < hi; i++) {
    const float v = zval(i);
    if (bi == INT_MAX || v > bv) { bv = v; bi = i; }
  }
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
  }
  if (lane == 0) { sv[warp] = bv; si[warp] = bi; }
  __syncthreads();
  if (warp == 0) {
    bv = sv[lane];
    bi = si[lane];
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if (lane == 0) { sv[0] = bv; si[0] = bi; }
  }
  __syncthreads();
  const float zmax = sv[0];
  if (!(temperature > 0.f) || top_k == 1 || V == 1) {
    if (tid == 0) out[b] = si[0];
    return;
  }
  // top-k cut: the k-th largest key by an 8-bit-digit radix select (most
  // significant digit first); the set is every key above it plus the first
  // `rem` ids holding it
  const bool all = top_k <= 0 || top_k >= V;
  uint32_t thr = 0u;
  unsigned rem = 0u;
  if (!all) {
    uint32_t prefix = 0u, mask = 0u;
    unsigned remaining = (unsigned)top_k;
    for (int shift = 24; shift >= 0; shift -= 8) {
      if (tid < 256) hist[tid] = 0u;
      __syncthreads();
      for (int i = lo; i < hi; i++) {
        const uint32_t k = order_key(zval(i));
        if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (tid == 0) {
        unsigned cum = 0u;
        int dsel = 0;
        for (int dg = 255; dg >= 0; dg--) {
          if (cum + hist[dg] >= remaining) { dsel = dg; break; }
          cum += hist[dg];
        }
        s_prefix = prefix | ((uint32_t)dsel << shift);
        s_rem = remaining - cum;
      }
      __syncthreads();
      prefix = s_prefix;
      remaining = s_rem;
      mask |= 255u << shift;
      __syncthreads();
    }
    thr = prefix;
    rem = remaining;
  }
  // rank of this thread's first id among the ids holding the cut key
  unsigned myeq = 0u;
  if (!all)
    for (int i = lo; i < hi; i++) myeq += order_key(zval(i)) == thr;
  eqc[tid] = myeq;
  __syncthreads();
  if (tid == 0) {
    unsigned run = 0u;
    for (int t = 0; t < SP_THREADS; t++) {
      const unsigned n = eqc[t];
      eqc[t] = run;
      run += n;
    }
  }
  __syncthreads();
  const unsigned eq0 = eqc[tid];
  // top-p: the composites of the top-k set sorted descending; members are the
  // composites >= the cut (0: no cut)
  unsigned long long cut = 0ull;
  if constexpr (EXT) {
    if (ext.top_p < 1.f) {
      __shared__ unsigned long long sortv[SP_NUC_MAX];
      __shared__ unsigned scnt[SP_THREADS];
      __shared__ unsigned s_n;
      __shared__ unsigned long long s_cut;
      unsigned cnt = 0u;
      {
        unsigned eq = eq0;
        for (int i = lo; i < hi; i++) {
          const uint32_t k = order_key(zval(i));
          cnt += all || k > thr || (k == thr && eq < rem);
          if (!all) eq += k == thr;
        }
      }
      scnt[tid] = cnt;
      __syncthreads();
      if (tid == 0) {
        unsigned run = 0u;
        for (int t = 0; t < SP_THREADS; t++) {
          const unsigned n = scnt[t];
          scnt[t] = run;
          run += n;
        }
        s_n = run;  // <= SP_NUC_MAX: top_k <= SP_NUC_MAX, or V itself when top_k >= V
      }
      __syncthreads();
      const int n = (int)s_n;
      {
        unsigned pos = scnt[tid], eq = eq0;
        for (int i = lo; i < hi; i++) {
          const uint32_t k = order_key(zval(i));
          const bool in = all || k > thr || (k == thr && eq < rem);
          if (!all) eq += k == thr;
          if (in) sortv[pos++] = sort_composite(k, i);
        }
      }
      int n2 = 1;
      while (n2 < n) n2 <<= 1;
      for (int t = n + tid; t < n2; t += SP_THREADS) sortv[t] = 0ull;  // below every member
      __syncthreads();
      // bitonic sort, descending
      for (int size = 2; size <= n2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          for (int t = tid; t < n2; t += SP_THREADS) {
            const int q = t ^ stride;
            if (q > t) {
              const unsigned long long x = sortv[t], y = sortv[q];
              if (((t & size) == 0) ? (x < y) : (x > y)) { sortv[t] = y; sortv[q] = x; }
            }
          }
          __syncthreads();
        }
      }
      // weights along the walk (one per thread), then the prefix by one thread
      for (int t = tid; t < n; t += SP_THREADS) {
        const int id = (int)(0xFFFFFFFFu - (uint32_t)sortv[t]);
        wsum[t] = sample_weight(zval(id), zmax, temperature);
      }
      __syncthreads();
      if (tid == 0) {
        float W = 0.f;
        for (int t = 0; t < n; t++) W += wsum[t];
        const float goal = ext.top_p * W;
        float c = 0.f;
        int m = n;
        for (int t = 0; t < n; t++) {
          c += wsum[t];
          if (c >= goal) { m = t + 1; break; }
        }
        s_cut = sortv[m - 1];
      }
      __syncthreads();
      cut = s_cut;
    }
  }
  auto member = [&](int i, unsigned &eq) -> bool {  // in the top-k set (and the nucleus)
    bool in = all;
    uint32_t k = 0u;
    if (!all || EXT) k = order_key(zval(i));
    if (!all) {
      in = k > thr || (k == thr && eq < rem);
      eq += k == thr;
    }
    if constexpr (EXT) in = in && sort_composite(k, i) >= cut;
    return in;
  };
  // this thread's weight, ids in increasing order
  float my = 0.f;
  {
    unsigned eq = eq0;
    for (int i = lo; i < hi; i++)
      if (member(i, eq)) my += sample_weight(zval(i), zmax, temperature);
  }
  __syncthreads();  // the top-p walk's weights are no longer read
  wsum[tid] = my;
  __syncthreads();
  if (tid == 0) {
    float W = 0.f;
    for (int t = 0; t < SP_THREADS; t++) W += wsum[t];
    const float u = fminf(fmaxf(uni[b], 0.f), 0.99999994f);
    const float target = u * W;
    float c = 0.f, tl = 0.f;
    int owner = -1;
    for (int t = 0; t < SP_THREADS; t++) {
      const float cn = c + wsum[t];
      if (wsum[t] > 0.f && target < cn) { owner = t; tl = target - c; break; }
      c = cn;
    }
    if (owner < 0)  // rounding put the target past the end: the last weighted id
      for (int t = SP_THREADS - 1; t >= 0; t--)
        if (wsum[t] > 0.f) { owner = t; tl = wsum[t]; break; }
    s_owner = owner;
    s_tl = tl;
  }
  __syncthreads();
  if (tid == s_owner) {
    float c = 0.f;
    int pick = -1, lastin = -1;
    unsigned eq = eq0;
    for (int i = lo; i < hi; i++) {
      if (!member(i, eq)) continue;
      c += sample_weight(zval(i), zmax, temperature);
      lastin = i;
      if (c > s_tl) { pick = i; break; }
    }
    out[b] = pick >= 0 ? pick : lastin;
  }
}

__global__ void k_set_int(int *p, int v) { *p = v; }

}  // namespace

void gemv_plan(int64_t K, int64_t N, int *ks, int *kslice) {
  const int64_t cb = (N + GV_COLS - 1) / GV_COLS;
  // one wave: two blocks of this kernel fit on each of the 148 SMs
  const int64_t want = std::max<int64_t>(1, (2 * 148) / cb);
  const int64_t ks_max = std::min<int64_t>(GV_KS_MAX, std::max<int64_t>(1, (K + 63) / 64));
  const int64_t ks_min = (K + GV_KSLICE_MAX - 1) / GV_KSLICE_MAX;
  // (measured: more slices than one wave, or slices under 128 rows bought
  // with a second wave, made the W13 and lm_head products slower)
  int64_t s = std::max(std::min(want, ks_max), ks_min);
  int64_t sl = (K + s - 1) / s;
  sl = std::min<int64_t>(GV_KSLICE_MAX, (sl + 15) / 16 * 16);
  *kslice = (int)sl;
  *ks = (int)((K + sl - 1) / sl);
}

int gemv_col_blocks(int64_t N) { return (int)cdiv(N, GV_COLS); }

bool gemv_fits(int64_t K, int64_t N) {
  int ks = 0, sl = 0;
  gemv_plan(K, N, &ks, &sl);
  return ks >= 1 && ks <= GV_KS_MAX && sl >= 1 && sl <= GV_KSLICE_MAX;
}

// Launch with programmatic stream serialisation (see pdl_release / pdl_wait).
template <typename... P, typename... Q>
static void launch_pdl(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Q... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kernel, args...);
}

void gemv(const GemvArgs &a, DType dt, cudaStream_t s) {
  dim3 grid(cdiv(a.N, GV_COLS), a.ks);
  if (dt == DT_BF16) launch_pdl(k_gemv<__nv_bfloat16>, grid, dim3(GV_THREADS), 0, s, a);
  else launch_pdl(k_gemv<float>, grid, dim3(GV_THREADS), 0, s, a);
  count_launch();
}

int attn_decode_chunks(int T) { return (int)cdiv(T, AT_KEYS); }

template <typename A, int GT>
static void attn_launch(dim3 grid, size_t smem, cudaStream_t s, const void *qkv, int64_t qkvw,
                        int T, const int *pos, int H, int Hkv, int hd, int nch, int vec,
                        float *part, unsigned *count, void *o) {
  // room for the largest staged tile (a refusal fails the launch)
  smem_optin((const void *)k_attn_decode<A, GT>, (int)(2 * AT_KEYS * attn_row_bytes(AT_HDMAX, 4)));
  launch_pdl(k_attn_decode<A, GT>, grid, dim3(AT_THREADS), smem, s, (const A *)qkv, qkvw, T, pos,
             H, Hkv, hd, nch, vec, part, count, (A *)o);
}
template <typename A>
static void attn_dispatch(int G, dim3 grid, size_t smem, cudaStream_t s, const void *qkv,
                          int64_t qkvw, int T, const int *pos, int H, int Hkv, int hd, int nch,
                          int vec, float *part, unsigned *count, void *o) {
  if (G <= 1) attn_launch<A, 1>(grid, smem, s, qkv, qkvw, T, pos, H, Hkv, hd, nch, vec, part, count, o);
  else if (G <= 2) attn_launch<A, 2>(grid, smem, s, qkv, qkvw, T, pos, H, Hkv, hd, nch, vec, part, count, o);
  else if (G <= 4) attn_launch<A, 4>(grid, smem, s, qkv, qkvw, T, pos, H, Hkv, hd, nch, vec, part, count, o);
  else attn_launch<A, 8>(grid, smem, s, qkv, qkvw, T, pos, H, Hkv, hd, nch, vec, part, count, o);
}

void attn_decode(const void *qkv, int64_t qkvw, int B, int T, const int *pos, int H, int Hkv,
                 int hd, float *part, unsigned *count, void *o, DType dt, cudaStream_t s) {
  const int nch = attn_decode_chunks(T), d = H * hd, kvd = Hkv * hd;
  const int esz = dt == DT_BF16 ? 2 : 4, ve = 16 / esz;
  // 16-byte copies: whole pieces per row, every row start 16-byte aligned
  const int vec = ((hd * esz) % 16 == 0 && qkvw % ve == 0 && d % ve == 0 && kvd % ve == 0 &&
                   ((uintptr_t)qkv & 15) == 0) ? 1 : 0;
  const size_t smem = 2 * (size_t)AT_KEYS * attn_row_bytes(hd, esz);
  dim3 grid(nch, Hkv, B);
  if (dt == DT_BF16)
    attn_dispatch<__nv_bfloat16>(H / Hkv, grid, smem, s, qkv, qkvw, T, pos, H, Hkv, hd, nch, vec,
                                 part, count, o);
  else
    attn_dispatch<float>(H / Hkv, grid, smem, s, qkv, qkvw, T, pos, H, Hkv, hd, nch, vec, part,
                         count, o);
  count_launch();
}

void sample_tokens(const float *logits, int64_t ld, int rows, int V, float temperature, int top_k,
                   const float *uni, int32_t *out, cudaStream_t s) {
  k_sample<false><<<rows, SP_THREADS, 0, s>>>(logits, ld, V, temperature, top_k, uni, out,
                                              SampleExt{});
  count_launch();
}

int sample_ex_max_top_k() { return SP_NUC_MAX; }
int64_t sample_ex_max_vocab_penalty() { return (int64_t)SP_PEN_BYTES * 8; }

void sample_tokens_ex(const float *logits, int64_t ld, int rows, int V, float temperature,
                      int top_k, float top_p, float penalty, const int32_t *hist,
                      int64_t hist_ld, int hist_len, const float *uni, int32_t *out,
                      cudaStream_t s) {
  smem_optin((const void *)k_sample<true>, SP_PEN_BYTES);  // room for the largest history bitmap
  SampleExt e;
  e.top_p = top_p;
  e.penalty = penalty;
  e.hist = hist;
  e.hist_ld = hist_ld;
  e.hist_len = hist_len;
  const bool pen = penalty != 1.f && hist_len > 0;
  const size_t smem = pen ? (size_t)((V + 31) / 32) * 4 : 0;
  k_sample<true><<<rows, SP_THREADS, smem, s>>>(logits, ld, V, temperature, top_k, uni, out, e);
  count_launch();
}

void set_device_int(int *p, int v, cudaStream_t s) {
  k_set_int<<<1, 1, 0, s>>>(p, v);
  count_launch();
}

}  // namespace llm
