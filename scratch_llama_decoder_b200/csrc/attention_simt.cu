// CUDA-core causal attention, forward and backward, for any head size.  Used
// by the float32 configurations (head sizes 4 and 32; the tiled kernels below
// take head sizes 32 and 64 without dropout) and as the plain reference of the
// tensor-core kernels.  One warp per query row (forward, dq)
// or per key row (dk, dv); the softmax is the online (running max and sum)
// form of strata's flash-style attention, and only the row log-sum-exp is
// saved for the backward.  With dropout (drop.on) the value sums use the
// dropped probabilities P f while the softmax statistics stay those of P
// (Hephaistos: inverted dropout on the attention weights).
#include "common.cuh"
#include "internal.h"

namespace llm {

constexpr int MAXR = 4;  // head sizes up to 128 (4 values per lane)

// Hephaistos, Architecture at a glance (Attention): causal multi-head
// attention with a numerically stable softmax; strata: n_head and n_kv_head
// independent.  Query head hq reads kv head hq / (H/Hkv).
// s_ij = q_i . k_j / sqrt(hd) for j <= i; o_i = sum_j softmax_j(s_ij) v_j.
template <typename A>
__global__ void k_attn_fwd_simt(const A *__restrict__ qkv, A *__restrict__ o,
                                float *__restrict__ lse, int B, int T, int H, int Hkv, int hd,
                                const DropArgs drop) {
  int64_t wid = blockIdx.x * (int64_t)(blockDim.x / 32) + threadIdx.x / 32;
  int lane = threadIdx.x & 31;
  if (wid >= (int64_t)B * H * T) return;
  int i = (int)(wid % T);
  int hq = (int)((wid / T) % H);
  int b = (int)(wid / ((int64_t)T * H));
  int d = H * hd, kvd = Hkv * hd, g = hq / (H / Hkv);
  int64_t w = d + 2 * kvd;
  float scale = 1.0f / sqrtf((float)hd);
  const A *qr = qkv + ((int64_t)b * T + i) * w + (int64_t)hq * hd;
  float q[MAXR], acc[MAXR];
#pragma unroll
  for (int r = 0; r < MAXR; r++) {
    int e = lane + 32 * r;
    q[r] = (e < hd) ? to_f(qr[e]) : 0.f;
    acc[r] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const uint32_t step = drop.on ? (uint32_t)*drop.step : 0u;
  const uint64_t erow = (((uint64_t)b * H + hq) * T + i) * T;
  for (int j = 0; j <= i; j++) {
    const A *kr = qkv + ((int64_t)b * T + j) * w + d + (int64_t)g * hd;
    const A *vr = kr + kvd;
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < MAXR; r++) {
      int e = lane + 32 * r;
      if (e < hd) s += q[r] * to_f(kr[e]);
    }
    s = warp_sum(s) * scale;
    float mn = fmaxf(m, s);
    float corr = expf(m - mn), p = expf(s - mn);
    l = l * corr + p;
    const float pv = drop.on ? p * drop_factor(drop, erow + j, step) : p;
#pragma unroll
    for (int r = 0; r < MAXR; r++) {
      int e = lane + 32 * r;
      acc[r] = acc[r] * corr + ((e < hd) ? pv * to_f(vr[e]) : 0.f);
    }
    m = mn;
  }
  A *orow = o + ((int64_t)b * T + i) * d + (int64_t)hq * hd;
#pragma unroll
  for (int r = 0; r < MAXR; r++) {
    int e = lane + 32 * r;
    if (e < hd) orow[e] = from_f<A>(acc[r] / l);
  }
  if (lane == 0) lse[((int64_t)b * H + hq) * T + i] = m + logf(l);
}

// Backward (strata: attention backward; P recomputed from the saved lse):
// D_i = do_i . o_i; P_ij = exp(s_ij - lse_i); dP_ij = do_i . v_j;
// dS_ij = P_ij (dP_ij - D_i); dq_i = sum_j dS_ij k_j / sqrt(hd).
// With dropout, dP_ij = f_ij (do_i . v_j) and D_i = do_i . o_i still equals
// sum_j P_ij dP_ij.
template <typename A>
__global__ void k_attn_bwd_dq_simt(const A *__restrict__ qkv, const A *__restrict__ o,
                                   const A *__restrict__ dout, const float *__restrict__ lse,
                                   float *__restrict__ Dbuf, A *__restrict__ dqkv, int B, int T,
                                   int H, int Hkv, int hd, const DropArgs drop) {
  int64_t wid = blockIdx.x * (int64_t)(blockDim.x / 32) + threadIdx.x / 32;
  int lane = threadIdx.x & 31;
  if (wid >= (int64_t)B * H * T) return;
  int i = (int)(wid % T);
  int hq = (int)((wid / T) % H);
  int b = (int)(wid / ((int64_t)T * H));
  int d = H * hd, kvd = Hkv * hd, g = hq / (H / Hkv);
  int64_t w = d + 2 * kvd;
  float scale = 1.0f / sqrtf((float)hd);
  int64_t row = (int64_t)b * T + i;
  const A *qr = qkv + row * w + (int64_t)hq * hd;
  const A *dor = dout + row * d + (int64_t)hq * hd;
  const A *orow = o + row * d + (int64_t)hq * hd;
  float q[MAXR], dov[MAXR], dq[MAXR];
  float D = 0.f;
#pragma unroll
  for (int r = 0; r < MAXR; r++) {
    int e = lane + 32 * r;
    q[r] = (e < hd) ? to_f(qr[e]) : 0.f;
    dov[r] = (e < hd) ? to_f(dor[e]) : 0.f;
    D += (e < hd) ? dov[r] * to_f(orow[e]) : 0.f;
    dq[r] = 0.f;
  }
  D = warp_sum(D);
  float L = lse[((int64_t)b * H + hq) * T + i];
  if (lane == 0) Dbuf[((int64_t)b * H + hq) * T + i] = D;
  const uint32_t step = drop.on ? (uint32_t)*drop.step : 0u;
  const uint64_t erow = (((uint64_t)b * H + hq) * T + i) * T;
  for (int j = 0; j <= i; j++) {
    const A *kr = qkv + ((int64_t)b * T + j) * w + d + (int64_t)g * hd;
    const A *vr = kr + kvd;
    float s = 0.f, dp = 0.f;
#pragma unroll
    for (int r = 0; r < MAXR; r++) {
      int e = lane + 32 * r;
      if (e < hd) { s += q[r] * to_f(kr[e]); dp += dov[r] * to_f(vr[e]); }
    }
    s = warp_sum(s) * scale;
    dp = warp_sum(dp);
    if (drop.on) dp *= drop_factor(drop, erow + j, step);
    float p = expf(s - L);
    float ds = p * (dp - D) * scale;
#pragma unroll
    for (int r = 0; r < MAXR; r++) {
      int e = lane + 32 * r;
      if (e < hd) dq[r] += ds * to_f(kr[e]);
    }
  }
  A *dqr = dqkv + row * w + (int64_t)hq * hd;
#pragma unroll
  for (int r = 0; r < MAXR; r++) {
    int e = lane + 32 * r;
    if (e < hd) dqr[e] = from_f<A>(dq[r]);
  }
}

// dk_j = sum over the group's query heads, then i >= j, of dS_ij q_i / sqrt(hd);
// dv_j = the same sum of P_ij do_i.  Needs Dbuf from the dq kernel.
template <typename A>
__global__ void k_attn_bwd_dkv_simt(const A *__restrict__ qkv, const A *__restrict__ dout,
                                    const float *__restrict__ lse, const float *__restrict__ Dbuf,
                                    A *__restrict__ dqkv, int B, int T, int H, int Hkv, int hd,
                                    const DropArgs drop) {
  int64_t wid = blockIdx.x * (int64_t)(blockDim.x / 32) + threadIdx.x / 32;
  int lane = threadIdx.x & 31;
  if (wid >= (int64_t)B * Hkv * T) return;
  int j = (int)(wid % T);
  int g = (int)((wid / T) % Hkv);
  int b = (int)(wid / ((int64_t)T * Hkv));
  int d = H * hd, kvd = Hkv * hd, grp = H / Hkv;
  int64_t w = d + 2 * kvd;
  float scale = 1.0f / sqrtf((float)hd);
  const A *kr = qkv + ((int64_t)b * T + j) * w + d + (int64_t)g * hd;
  const A *vr = kr + kvd;
  float k[MAXR], v[MAXR], dk[MAXR], dv[MAXR];
#pragma unroll
  for (int r = 0; r < MAXR; r++) {
    int e = lane + 32 * r;
    k[r] = (e < hd) ? to_f(kr[e]) : 0.f;
    v[r] = (e < hd) ? to_f(vr[e]) : 0.f;
    dk[r] = dv[r] = 0.f;
  }
  const uint32_t step = drop.on ? (uint32_t)*drop.step : 0u;
  for (int hq = g * grp; hq < (g + 1) * grp; hq++) {
    for (int i = j; i < T; i++) {
      int64_t row = (int64_t)b * T + i;
      const A *qr = qkv + row * w + (int64_t)hq * hd;
      const A *dor = dout + row * d + (int64_t)hq * hd;
      float s = 0.f, dp = 0.f;
      float qv[MAXR], dov[MAXR];
#pragma unroll
      for (int r = 0; r < MAXR; r++) {
        int e = lane + 32 * r;
        qv[r] = (e < hd) ? to_f(qr[e]) : 0.f;
        dov[r] = (e < hd) ? to_f(dor[e]) : 0.f;
        s += qv[r] * k[r];
        dp += dov[r] * v[r];
      }
      s = warp_sum(s) * scale;
      dp = warp_sum(dp);
      int64_t li = ((int64_t)b * H + hq) * T + i;
      float p = expf(s - lse[li]);
      float pv = p;  // the probability the forward multiplied v by
      if (drop.on) {
        const float f = drop_factor(drop, (uint64_t)li * T + j, step);
        dp *= f;
        pv = p * f;
      }
      float ds = p * (dp - Dbuf[li]) * scale;
#pragma unroll
      for (int r = 0; r < MAXR; r++) {
        dk[r] += ds * qv[r];
        dv[r] += pv * dov[r];
      }
    }
  }
  A *dkr = dqkv + ((int64_t)b * T + j) * w + d + (int64_t)g * hd;
  A *dvr = dkr + kvd;
#pragma unroll
  for (int r = 0; r < MAXR; r++) {
    int e = lane + 32 * r;
    if (e < hd) { dkr[e] = from_f<A>(dk[r]); dvr[e] = from_f<A>(dv[r]); }
  }
}


// ------------------------------------------------------------- tiled fp32
// float32 attention for head sizes 32 and 64 without dropout: the same
// quantities as the kernels above, with 64-query x 64-key tiles in shared
// memory and 4 x 4 register tiles per thread (256 threads: tx = thread % 16
// picks 4 columns of a tile, ty = thread / 16 picks 4 rows; the 16 threads of
// a row group are one half-warp, so row reductions are 4 shuffles).  Operands
// of a tile product sit transposed ([head column][row], padded rows) so a
// thread reads its 4 rows and its 4 columns as two float4 per head column;
// probability tiles sit as [column][row] float4 slots, slot ty of row k at
// ty ^ (k / 4) so that the float4 stores of a half-warp hit distinct banks.
constexpr int TB = 64;       // query and key tile
constexpr int TLD = TB + 4;  // padded row of a transposed operand
constexpr int TNT = 256;

LLM_DEV int pslot(int k, int g4) { return k * TB + ((g4 ^ (k >> 2)) & 15) * 4; }

// acc[r][c] += sum_e A[e][ty*4 + r] B[e][tx*4 + c] over HD head columns.
template <int HD>
LLM_DEV void tile_dot(const float *At, const float *Bt, int tx, int ty, float (&acc)[4][4]) {
#pragma unroll 8
  for (int e = 0; e < HD; e++) {
    const float4 a = *reinterpret_cast<const float4 *>(At + e * TLD + ty * 4);
    const float4 b = *reinterpret_cast<const float4 *>(Bt + e * TLD + tx * 4);
    const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int r = 0; r < 4; r++)
#pragma unroll
      for (int c = 0; c < 4; c++) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
  }
}
// out[r][c] += sum_k P[k][ty*4 + r] M[k][tx*CW + c] over the 64 tile rows k of
// a probability tile P (float4 slots) and a row-major [64][HD] operand M.
template <int HD>
LLM_DEV void tile_acc(const float *P, const float *M, int tx, int ty, float (&out)[4][HD / 16]) {
  constexpr int CW = HD / 16;
#pragma unroll 4
  for (int k = 0; k < TB; k++) {
    const float4 p = *reinterpret_cast<const float4 *>(P + pslot(k, ty));
    const float pv[4] = {p.x, p.y, p.z, p.w};
    float mv[CW];
    if constexpr (CW == 4) {
      const float4 m = *reinterpret_cast<const float4 *>(M + k * HD + tx * 4);
      mv[0] = m.x; mv[1] = m.y; mv[2] = m.z; mv[3] = m.w;
    } else {
      const float2 m = *reinterpret_cast<const float2 *>(M + k * HD + tx * 2);
      mv[0] = m.x; mv[1] = m.y;
    }
#pragma unroll
    for (int r = 0; r < 4; r++)
#pragma unroll
      for (int c = 0; c < CW; c++) out[r][c] = fmaf(pv[r], mv[c], out[r][c]);
  }
}
// Rows row0.. of a [rows, ld] float32 matrix at column col0, HD columns, into
// a transposed tile At[e][row] (times mul; rows >= nrows give 0) and, when Mr
// is given, a row-major copy Mr[row][e].
template <int HD>
LLM_DEV void tile_load(const float *src, int64_t ld, int64_t row0, int nrows, int64_t col0,
                       float mul, float *At, float *Mr) {
  for (int idx = threadIdx.x; idx < TB * HD / 4; idx += TNT) {
    const int row = idx / (HD / 4), c4 = idx % (HD / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row < nrows) v = *reinterpret_cast<const float4 *>(src + (row0 + row) * ld + col0 + c4 * 4);
    v.x *= mul; v.y *= mul; v.z *= mul; v.w *= mul;
    At[(c4 * 4 + 0) * TLD + row] = v.x;
    At[(c4 * 4 + 1) * TLD + row] = v.y;
    At[(c4 * 4 + 2) * TLD + row] = v.z;
    At[(c4 * 4 + 3) * TLD + row] = v.w;
    if (Mr) *reinterpret_cast<float4 *>(Mr + row * HD + c4 * 4) = v;
  }
}
LLM_DEV float half_max(float v) {
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
LLM_DEV float half_sum(float v) {
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Dropout factors of the keys key0 .. key0 + 3 (key0 % 4 == 0) of query q,
// element (hrow + q) T + key of the probability site: one generator group
// when T % 4 == 0, else one group per element.
LLM_DEV void drop_keys4(const DropArgs &drop, uint64_t hrow, int T, int q, int key0,
                        uint32_t step, float (&f)[4]) {
  const uint64_t e = (hrow + q) * (uint64_t)T + key0;
  if ((T & 3) == 0) {  // drop.e0, a multiple of H T^2, keeps the group aligned
    const uint32_t keep = drop_bits4(drop, (drop.e0 + e) >> 2, step);
#pragma unroll
    for (int j = 0; j < 4; j++) f[j] = (keep >> j) & 1u ? drop.scale : 0.f;
  } else {
#pragma unroll
    for (int j = 0; j < 4; j++) f[j] = drop_factor(drop, e + j, step);
  }
}

// Forward: grid (query tiles, B*H), last query tiles first.
template <int HD, bool DROP>
__global__ void __launch_bounds__(TNT) k_attn_fwd_tile(const float *__restrict__ qkv,
                                                        float *__restrict__ o,
                                                        float *__restrict__ lse, int T, int H,
                                                        int Hkv, const DropArgs drop) {
  constexpr int CW = HD / 16;
  extern __shared__ float4 sm4[];
  float *Qt = reinterpret_cast<float *>(sm4), *Kt = Qt + HD * TLD, *Vs = Kt + HD * TLD,
        *Pt = Vs + TB * HD;
  const uint32_t dstep = DROP ? (uint32_t)*drop.step : 0u;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int qb = gridDim.x - 1 - blockIdx.x, b = blockIdx.y / H, h = blockIdx.y % H;
  const int g = h / (H / Hkv), d = H * HD, kvd = Hkv * HD;
  const int64_t w = d + 2 * kvd, row0 = (int64_t)b * T;
  const int q0 = qb * TB;
  tile_load<HD>(qkv, w, row0 + q0, min(TB, T - q0), (int64_t)h * HD, (1.0f / sqrtf((float)HD)), Qt,
                nullptr);
  float m[4], lp[4], acc[4][CW];
#pragma unroll
  for (int r = 0; r < 4; r++) {
    m[r] = -INFINITY;
    lp[r] = 0.f;
#pragma unroll
    for (int c = 0; c < CW; c++) acc[r][c] = 0.f;
  }
  for (int kb = 0; kb <= qb; kb++) {
    __syncthreads();  // the previous tile's products are done with Kt, Vs, Pt
    const int k0 = kb * TB, nk = min(TB, T - k0);
    tile_load<HD>(qkv, w, row0 + k0, nk, d + (int64_t)g * HD, 1.f, Kt, nullptr);
    for (int idx = threadIdx.x; idx < TB * HD / 4; idx += TNT) {
      const int row = idx / (HD / 4), c4 = idx % (HD / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (row < nk)
        v = *reinterpret_cast<const float4 *>(qkv + (row0 + k0 + row) * w + d + kvd + g * HD + c4 * 4);
      *reinterpret_cast<float4 *>(Vs + row * HD + c4 * 4) = v;
    }
    __syncthreads();
    float sv[4][4] = {};
    tile_dot<HD>(Qt, Kt, tx, ty, sv);
    if (kb == qb) {  // the diagonal tile: keys above the row (and past T) masked
#pragma unroll
      for (int r = 0; r < 4; r++)
#pragma unroll
        for (int c = 0; c < 4; c++) {
          const int key = k0 + tx * 4 + c;
          if (key > q0 + ty * 4 + r || key >= T) sv[r][c] = -INFINITY;
        }
    }
    float pt[4][4];
#pragma unroll
    for (int r = 0; r < 4; r++) {
      const float bm = half_max(fmaxf(fmaxf(sv[r][0], sv[r][1]), fmaxf(sv[r][2], sv[r][3])));
      const float mn = fmaxf(m[r], bm);
      const float corr = expf(m[r] - mn);  // 0 on the first tile (m = -inf)
      float ps = 0.f;
#pragma unroll
      for (int c = 0; c < 4; c++) {
        pt[c][r] = expf(sv[r][c] - mn);
        ps += pt[c][r];
      }
      lp[r] = lp[r] * corr + ps;
      m[r] = mn;
#pragma unroll
      for (int c = 0; c < CW; c++) acc[r][c] *= corr;
    }
    if constexpr (DROP) {  // P V with the dropped probabilities P f; the sums lp keep P's
#pragma unroll
      for (int r = 0; r < 4; r++) {
        float f[4];
        drop_keys4(drop, ((uint64_t)b * H + h) * T, T, q0 + ty * 4 + r, k0 + tx * 4, dstep, f);
#pragma unroll
        for (int c = 0; c < 4; c++) pt[c][r] *= f[c];
      }
    }
#pragma unroll
    for (int c = 0; c < 4; c++)
      *reinterpret_cast<float4 *>(Pt + pslot(tx * 4 + c, ty)) =
          make_float4(pt[c][0], pt[c][1], pt[c][2], pt[c][3]);
    __syncthreads();
    tile_acc<HD>(Pt, Vs, tx, ty, acc);
  }
#pragma unroll
  for (int r = 0; r < 4; r++) {
    const float l = half_sum(lp[r]);
    const int q = q0 + ty * 4 + r;
    if (q < T) {
      float *orow = o + (row0 + q) * d + (int64_t)h * HD + tx * CW;
#pragma unroll
      for (int c = 0; c < CW; c++) orow[c] = acc[r][c] / l;
      if (tx == 0) lse[((int64_t)b * H + h) * T + q] = m[r] + logf(l);
    }
  }
}

// dQ (and D = rowsum(dO o O) into Dbuf): grid (query tiles, B*H).
template <int HD, bool DROP>
__global__ void __launch_bounds__(TNT) k_attn_dq_tile(const float *__restrict__ qkv,
                                                       const float *__restrict__ o,
                                                       const float *__restrict__ dout,
                                                       const float *__restrict__ lse,
                                                       float *__restrict__ Dbuf,
                                                       float *__restrict__ dqkv, int T, int H,
                                                       int Hkv, const DropArgs drop) {
  constexpr int CW = HD / 16;
  const uint32_t dstep = DROP ? (uint32_t)*drop.step : 0u;
  extern __shared__ float4 sm4[];
  float *Qt = reinterpret_cast<float *>(sm4), *dOt = Qt + HD * TLD, *Kt = dOt + HD * TLD,
        *Vt = Kt + HD * TLD, *Kr = Vt + HD * TLD, *dSt = Kr + TB * HD;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int qb = gridDim.x - 1 - blockIdx.x, b = blockIdx.y / H, h = blockIdx.y % H;
  const int g = h / (H / Hkv), d = H * HD, kvd = Hkv * HD;
  const int64_t w = d + 2 * kvd, row0 = (int64_t)b * T;
  const int q0 = qb * TB, nq = min(TB, T - q0);
  const float scale = (1.0f / sqrtf((float)HD));
  tile_load<HD>(qkv, w, row0 + q0, nq, (int64_t)h * HD, scale, Qt, nullptr);
  tile_load<HD>(dout, d, row0 + q0, nq, (int64_t)h * HD, 1.f, dOt, nullptr);
  // D and L of this thread's 4 rows
  float Dr[4], Lr[4];
#pragma unroll
  for (int r = 0; r < 4; r++) {
    const int q = q0 + ty * 4 + r;
    float part = 0.f;
    if (q < T) {
      const float *orow = o + (row0 + q) * d + (int64_t)h * HD + tx * CW;
      const float *drow = dout + (row0 + q) * d + (int64_t)h * HD + tx * CW;
#pragma unroll
      for (int c = 0; c < CW; c++) part += orow[c] * drow[c];
    }
    Dr[r] = half_sum(part);
    Lr[r] = q < T ? lse[((int64_t)b * H + h) * T + q] : INFINITY;
    if (tx == 0 && q < T) Dbuf[((int64_t)b * H + h) * T + q] = Dr[r];
  }
  float dq[4][CW];
#pragma unroll
  for (int r = 0; r < 4; r++)
#pragma unroll
    for (int c = 0; c < CW; c++) dq[r][c] = 0.f;
  for (int kb = 0; kb <= qb; kb++) {
    __syncthreads();
    const int k0 = kb * TB, nk = min(TB, T - k0);
    tile_load<HD>(qkv, w, row0 + k0, nk, d + (int64_t)g * HD, 1.f, Kt, Kr);
    tile_load<HD>(qkv, w, row0 + k0, nk, d + kvd + (int64_t)g * HD, 1.f, Vt, nullptr);
    __syncthreads();
    float sv[4][4] = {}, dp[4][4] = {};
    tile_dot<HD>(Qt, Kt, tx, ty, sv);
    tile_dot<HD>(dOt, Vt, tx, ty, dp);
    float ds[4][4];
#pragma unroll
    for (int r = 0; r < 4; r++) {
      // with dropout dP = f (dO . v), the forward having multiplied v by P f
      float f[4] = {1.f, 1.f, 1.f, 1.f};
      if constexpr (DROP)
        drop_keys4(drop, ((uint64_t)b * H + h) * T, T, q0 + ty * 4 + r, k0 + tx * 4, dstep, f);
#pragma unroll
      for (int c = 0; c < 4; c++) {
        const int key = k0 + tx * 4 + c;
        const bool masked = kb == qb && (key > q0 + ty * 4 + r || key >= T);
        const float p = masked ? 0.f : expf(sv[r][c] - Lr[r]);
        ds[c][r] = p * (dp[r][c] * f[c] - Dr[r]);
      }
    }
#pragma unroll
    for (int c = 0; c < 4; c++)
      *reinterpret_cast<float4 *>(dSt + pslot(tx * 4 + c, ty)) =
          make_float4(ds[c][0], ds[c][1], ds[c][2], ds[c][3]);
    __syncthreads();
    tile_acc<HD>(dSt, Kr, tx, ty, dq);
  }
#pragma unroll
  for (int r = 0; r < 4; r++) {
    const int q = q0 + ty * 4 + r;
    if (q < T) {
      float *dst = dqkv + (row0 + q) * w + (int64_t)h * HD + tx * CW;
#pragma unroll
      for (int c = 0; c < CW; c++) dst[c] = dq[r][c] * scale;
    }
  }
}

// dK, dV: grid (key tiles, B*Hkv), first key tiles first; steps over the
// group's query heads and the query tiles at or after the key tile.
template <int HD, bool DROP>
__global__ void __launch_bounds__(TNT) k_attn_dkv_tile(const float *__restrict__ qkv,
                                                        const float *__restrict__ dout,
                                                        const float *__restrict__ lse,
                                                        const float *__restrict__ Dbuf,
                                                        float *__restrict__ dqkv, int T, int H,
                                                        int Hkv, const DropArgs drop) {
  constexpr int CW = HD / 16;
  const uint32_t dstep = DROP ? (uint32_t)*drop.step : 0u;
  extern __shared__ float4 sm4[];
  float *Kt = reinterpret_cast<float *>(sm4), *Vt = Kt + HD * TLD, *Qt = Vt + HD * TLD,
        *dOt = Qt + HD * TLD, *Qr = dOt + HD * TLD, *dOr = Qr + TB * HD, *Ps = dOr + TB * HD,
        *dSs = Ps + TB * TB, *sL = dSs + TB * TB, *sD = sL + TB;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int kb = blockIdx.x, b = blockIdx.y / Hkv, g = blockIdx.y % Hkv;
  const int grp = H / Hkv, d = H * HD, kvd = Hkv * HD;
  const int64_t w = d + 2 * kvd, row0 = (int64_t)b * T;
  const int k0 = kb * TB, nk = min(TB, T - k0), nqt = (T + TB - 1) / TB;
  const float scale = (1.0f / sqrtf((float)HD));
  tile_load<HD>(qkv, w, row0 + k0, nk, d + (int64_t)g * HD, 1.f, Kt, nullptr);
  tile_load<HD>(qkv, w, row0 + k0, nk, d + kvd + (int64_t)g * HD, 1.f, Vt, nullptr);
  float dk[4][CW], dv[4][CW];
#pragma unroll
  for (int r = 0; r < 4; r++)
#pragma unroll
    for (int c = 0; c < CW; c++) dk[r][c] = dv[r][c] = 0.f;
  for (int hq = g * grp; hq < (g + 1) * grp; hq++) {
    for (int qb = kb; qb < nqt; qb++) {
      __syncthreads();
      const int q0 = qb * TB, nq = min(TB, T - q0);
      tile_load<HD>(qkv, w, row0 + q0, nq, (int64_t)hq * HD, scale, Qt, Qr);
      tile_load<HD>(dout, d, row0 + q0, nq, (int64_t)hq * HD, 1.f, dOt, dOr);
      if (threadIdx.x < TB) {
        const int q = q0 + threadIdx.x;
        const int64_t li = ((int64_t)b * H + hq) * T + q;
        sL[threadIdx.x] = q < T ? lse[li] : INFINITY;  // queries past T: P = 0
        sD[threadIdx.x] = q < T ? Dbuf[li] : 0.f;
      }
      __syncthreads();
      float sv[4][4] = {}, dp[4][4] = {};
      tile_dot<HD>(Kt, Qt, tx, ty, sv);  // S^T: rows keys, columns queries
      tile_dot<HD>(Vt, dOt, tx, ty, dp);
      // the forward multiplied v by P f: dV takes P f, dP takes f (fk[c][r]:
      // query q0 + 4 tx + c, key k0 + 4 ty + r)
      float fk[4][4];
#pragma unroll
      for (int c = 0; c < 4; c++) {
        if constexpr (DROP)
          drop_keys4(drop, ((uint64_t)b * H + hq) * T, T, q0 + tx * 4 + c, k0 + ty * 4, dstep,
                     fk[c]);
        else
          fk[c][0] = fk[c][1] = fk[c][2] = fk[c][3] = 1.f;
      }
      float pq[4][4], dq[4][4];
#pragma unroll
      for (int r = 0; r < 4; r++)
#pragma unroll
        for (int c = 0; c < 4; c++) {
          const int key = k0 + ty * 4 + r, q = q0 + tx * 4 + c;
          const bool masked = qb == kb && key > q;
          const float p = masked ? 0.f : expf(sv[r][c] - sL[tx * 4 + c]);
          pq[c][r] = p * fk[c][r];
          dq[c][r] = p * (dp[r][c] * fk[c][r] - sD[tx * 4 + c]);
        }
#pragma unroll
      for (int c = 0; c < 4; c++) {
        *reinterpret_cast<float4 *>(Ps + pslot(tx * 4 + c, ty)) =
            make_float4(pq[c][0], pq[c][1], pq[c][2], pq[c][3]);
        *reinterpret_cast<float4 *>(dSs + pslot(tx * 4 + c, ty)) =
            make_float4(dq[c][0], dq[c][1], dq[c][2], dq[c][3]);
      }
      __syncthreads();
      tile_acc<HD>(Ps, dOr, tx, ty, dv);
      tile_acc<HD>(dSs, Qr, tx, ty, dk);  // Qr holds q / sqrt(hd)
    }
  }
#pragma unroll
  for (int r = 0; r < 4; r++) {
    const int key = k0 + ty * 4 + r;
    if (key < T) {
      float *dkr = dqkv + (row0 + key) * w + d + (int64_t)g * HD + tx * CW;
      float *dvr = dkr + kvd;
#pragma unroll
      for (int c = 0; c < CW; c++) {
        dkr[c] = dk[r][c];
        dvr[c] = dv[r][c];
      }
    }
  }
}

template <int HD> constexpr int fwd_tile_smem() { return (2 * HD * TLD + TB * HD + TB * TB) * 4; }
template <int HD> constexpr int dq_tile_smem() { return (4 * HD * TLD + TB * HD + TB * TB) * 4; }
template <int HD>
constexpr int dkv_tile_smem() { return (4 * HD * TLD + 2 * TB * HD + 2 * TB * TB + 2 * TB) * 4; }

// The tiled float32 path: head size 32 or 64, 16-byte aligned
// rows (every row stride a multiple of 4 floats).
static bool tile_covers(DType dt, int hd) { return dt == DT_F32 && (hd == 32 || hd == 64); }
bool attn_tile_covers(int hd) { return hd == 32 || hd == 64; }
template <int HD>
static bool attn_fwd_tile(const float *qkv, float *o, float *lse, int B, int T, int H, int Hkv,
                          cudaStream_t s, const DropArgs &drop) {
  auto kern = drop.on ? k_attn_fwd_tile<HD, true> : k_attn_fwd_tile<HD, false>;
  if (!smem_optin((const void *)kern, fwd_tile_smem<HD>())) return false;
  kern<<<dim3((T + TB - 1) / TB, B * H), TNT, fwd_tile_smem<HD>(), s>>>(qkv, o, lse, T, H, Hkv,
                                                                      drop);
  count_launch();
  return true;
}
template <int HD>
static bool attn_bwd_tile(const float *qkv, const float *o, const float *dout, const float *lse,
                          float *Dbuf, float *dqkv, int B, int T, int H, int Hkv, cudaStream_t s,
                          const DropArgs &drop) {
  auto kdq = drop.on ? k_attn_dq_tile<HD, true> : k_attn_dq_tile<HD, false>;
  auto kdkv = drop.on ? k_attn_dkv_tile<HD, true> : k_attn_dkv_tile<HD, false>;
  if (!smem_optin((const void *)kdq, dq_tile_smem<HD>()) ||
      !smem_optin((const void *)kdkv, dkv_tile_smem<HD>()))
    return false;
  const int nt = (T + TB - 1) / TB;
  kdq<<<dim3(nt, B * H), TNT, dq_tile_smem<HD>(), s>>>(qkv, o, dout, lse, Dbuf, dqkv, T, H, Hkv,
                                                       drop);
  kdkv<<<dim3(nt, B * Hkv), TNT, dkv_tile_smem<HD>(), s>>>(qkv, dout, lse, Dbuf, dqkv, T, H, Hkv,
                                                           drop);
  count_launch(2);
  return true;
}

bool attn_fwd_f32_tiled(const float *qkv, float *o, float *lse, int B, int T, int H, int Hkv,
                        int hd, cudaStream_t s, DropArgs drop) {
  if (!attn_tile_covers(hd)) return false;
  return hd == 32 ? attn_fwd_tile<32>(qkv, o, lse, B, T, H, Hkv, s, drop)
                  : attn_fwd_tile<64>(qkv, o, lse, B, T, H, Hkv, s, drop);
}
bool attn_bwd_f32_tiled(const float *qkv, const float *o, const float *dout, const float *lse,
                        float *Dbuf, float *dqkv, int B, int T, int H, int Hkv, int hd,
                        cudaStream_t s, DropArgs drop) {
  if (!attn_tile_covers(hd)) return false;
  return hd == 32 ? attn_bwd_tile<32>(qkv, o, dout, lse, Dbuf, dqkv, B, T, H, Hkv, s, drop)
                  : attn_bwd_tile<64>(qkv, o, dout, lse, Dbuf, dqkv, B, T, H, Hkv, s, drop);
}
// The one-warp-per-row kernels alone (any head size).
void attn_fwd_rows(const void *qkv, void *o, float *lse, DType dt, int B, int T, int H, int Hkv,
                   int hd, cudaStream_t s, DropArgs drop);
void attn_bwd_rows(const void *qkv, const void *o, const void *dout, const float *lse, float *Dbuf,
                   void *dqkv, DType dt, int B, int T, int H, int Hkv, int hd, cudaStream_t s,
                   DropArgs drop);

void attn_fwd_simt(const void *qkv, void *o, float *lse, DType dt, int B, int T, int H, int Hkv,
                   int hd, cudaStream_t s, DropArgs drop) {
  if (tile_covers(dt, hd) &&
      attn_fwd_f32_tiled((const float *)qkv, (float *)o, lse, B, T, H, Hkv, hd, s, drop))
    return;
  attn_fwd_rows(qkv, o, lse, dt, B, T, H, Hkv, hd, s, drop);
}
void attn_bwd_simt(const void *qkv, const void *o, const void *dout, const float *lse, float *Dbuf,
                   void *dqkv, DType dt, int B, int T, int H, int Hkv, int hd, cudaStream_t s,
                   DropArgs drop) {
  if (tile_covers(dt, hd) &&
      attn_bwd_f32_tiled((const float *)qkv, (const float *)o, (const float *)dout, lse, Dbuf,
                         (float *)dqkv, B, T, H, Hkv, hd, s, drop))
    return;
  attn_bwd_rows(qkv, o, dout, lse, Dbuf, dqkv, dt, B, T, H, Hkv, hd, s, drop);
}

void attn_fwd_rows(const void *qkv, void *o, float *lse, DType dt, int B, int T, int H, int Hkv,
                   int hd, cudaStream_t s, DropArgs drop) {
  int64_t warps = (int64_t)B * H * T;
  unsigned grid = (unsigned)((warps + 7) / 8);
  if (dt == DT_BF16)
    k_attn_fwd_simt<<<grid, 256, 0, s>>>((const __nv_bfloat16 *)qkv, (__nv_bfloat16 *)o, lse, B, T,
                                         H, Hkv, hd, drop);
  else
    k_attn_fwd_simt<<<grid, 256, 0, s>>>((const float *)qkv, (float *)o, lse, B, T, H, Hkv, hd,
                                         drop);
  count_launch();
}

void attn_bwd_rows(const void *qkv, const void *o, const void *dout, const float *lse, float *Dbuf,
                   void *dqkv, DType dt, int B, int T, int H, int Hkv, int hd, cudaStream_t s,
                   DropArgs drop) {
  unsigned g1 = (unsigned)(((int64_t)B * H * T + 7) / 8);
  unsigned g2 = (unsigned)(((int64_t)B * Hkv * T + 7) / 8);
  if (dt == DT_BF16) {
    using T_ = __nv_bfloat16;
    k_attn_bwd_dq_simt<<<g1, 256, 0, s>>>((const T_ *)qkv, (const T_ *)o, (const T_ *)dout, lse,
                                          Dbuf, (T_ *)dqkv, B, T, H, Hkv, hd, drop);
    k_attn_bwd_dkv_simt<<<g2, 256, 0, s>>>((const T_ *)qkv, (const T_ *)dout, lse, Dbuf,
                                           (T_ *)dqkv, B, T, H, Hkv, hd, drop);
  } else {
    k_attn_bwd_dq_simt<<<g1, 256, 0, s>>>((const float *)qkv, (const float *)o,
                                          (const float *)dout, lse, Dbuf, (float *)dqkv, B, T, H,
                                          Hkv, hd, drop);
    k_attn_bwd_dkv_simt<<<g2, 256, 0, s>>>((const float *)qkv, (const float *)dout, lse, Dbuf,
                                           (float *)dqkv, B, T, H, Hkv, hd, drop);
  }
  count_launch(2);
}

}  // namespace llm
