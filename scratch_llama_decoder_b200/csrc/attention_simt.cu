// CUDA-core causal attention, forward and backward, for any head size.  Used
// by the float32 configurations (head sizes 4 and 32) and as the plain
// reference of the tensor-core kernels.  One warp per query row (forward, dq)
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

void attn_fwd_simt(const void *qkv, void *o, float *lse, DType dt, int B, int T, int H, int Hkv,
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

void attn_bwd_simt(const void *qkv, const void *o, const void *dout, const float *lse, float *Dbuf,
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
