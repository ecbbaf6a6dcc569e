// Tensor-core causal attention (bf16 operands, fp32 softmax and accumulators)
// for head sizes 32 and 64: the flash-style forward and backward of strata's
// online-softmax attention (no T x T scores in memory; the forward saves only
// the row log-sum-exp), on warp-level mma.m16n8k16 tiles.
//
// Layout: qkv [B*T, qkvw] row-major with the q heads, then k heads, then v
// heads of each token; query head h reads kv head h / (H/Hkv).  o [B*T, H*hd].
// lse, D: [B, H, T] float32 (natural log).
//
// Kernels (64 x 64 tiles, 4 warps, 16 rows per warp):
//   fwd : one CTA per (b, h, 64 queries); loops over key blocks up to the
//         diagonal; online softmax in registers; P goes from the S
//         accumulator straight into the A fragments of P.V.
//   dq  : one CTA per (b, h, 64 queries): D_i = sum_e dO_ie O_ie (saved for
//         dkv), recompute P from lse, dP = dO V^T, dS = P (dP - D),
//         dQ += dS K.
//   dkv : one CTA per (b, kv head, 64 keys): loops over the group's query
//         heads and the query blocks at or after the keys, in a fixed order:
//         dV += P^T dO, dK += dS^T Q.  No atomics: deterministic.
// With cos/sin tables given, dq and dk leave through the inverse RoPE
// rotation (Hephaistos: RoPE on q and k), so the gradient reaching the QKV
// projection is with respect to the un-rotated q and k.
#include "common.cuh"
#include "gemm_tc.h"
#include "tcgen05.cuh"

namespace llm {
namespace attn {

constexpr int BQ = 64, BKV = 64, NW = 4, NT = NW * 32;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

LLM_DEV uint32_t sm(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// 16-byte async copy, zero-filled when !valid.
LLM_DEV void cp16(uint32_t dst, const void *src, bool valid) {
  int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n)
               : "memory");
}
LLM_DEV void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
LLM_DEV void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

LLM_DEV void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
LLM_DEV void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D (16x8 fp32) += A (16x16 bf16, row) . B (16x8 bf16, col)
LLM_DEV void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
LLM_DEV uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

// Shared-memory tile of 64 rows x HD bf16, rows padded by 8 elements (16 B)
// so the 8 row addresses of an ldmatrix fall in distinct banks.
template <int HD>
struct Tile {
  static constexpr int LD = HD + 8;
  __nv_bfloat16 v[64 * LD];
};

// Async load of rows [r0, r0+64) of a [rows_total, ld] bf16 matrix, columns
// [c0, c0+HD); rows >= rows_total are zero-filled.
template <int HD>
LLM_DEV void load_tile(Tile<HD> &t, const __nv_bfloat16 *base, int64_t ld, int r0, int rows_total,
                       int64_t row_offset) {
  constexpr int CH = HD / 8;  // 16-byte chunks per row
  for (int i = threadIdx.x; i < 64 * CH; i += NT) {
    int r = i / CH, c = i % CH;
    bool ok = r0 + r < rows_total;
    const __nv_bfloat16 *src = base + (row_offset + (ok ? r0 + r : 0)) * ld + c * 8;
    cp16(sm(&t.v[r * Tile<HD>::LD + c * 8]), src, ok);
  }
}

// A fragments (16 rows x HD) of rows [w*16, w*16+16) of a tile.
template <int HD>
LLM_DEV void load_afrag(const Tile<HD> &t, int w, uint32_t (&f)[HD / 16][4]) {
  int lane = threadIdx.x & 31;
  int row = w * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
  for (int k = 0; k < HD / 16; k++) {
    int col = k * 16 + (lane >> 4) * 8;
    ldsm_x4(sm(&t.v[row * Tile<HD>::LD + col]), f[k][0], f[k][1], f[k][2], f[k][3]);
  }
}

// acc[16 x 8*NT] += A[16 x HD] . X^T over rows [x0, x0 + 8*NT) of a 64 x HD
// tile X (rows = n): B(k, n) = X[x0 + n][k], loaded without transpose.
template <int HD, int NT = 8>
LLM_DEV void mma_abt(float (&acc)[NT][4], const uint32_t (&a)[HD / 16][4], const Tile<HD> &x,
                     int x0 = 0) {
  int lane = threadIdx.x & 31;
#pragma unroll
  for (int np = 0; np < NT / 2; np++) {  // pairs of 8-wide n tiles
    int row = x0 + np * 16 + (lane & 7) + (lane >> 4) * 8;
#pragma unroll
    for (int k = 0; k < HD / 16; k++) {
      int col = k * 16 + ((lane >> 3) & 1) * 8;
      uint32_t b0, b1, b2, b3;
      ldsm_x4(sm(&x.v[row * Tile<HD>::LD + col]), b0, b1, b2, b3);
      mma16816(acc[2 * np], a[k], b0, b1);
      mma16816(acc[2 * np + 1], a[k], b2, b3);
    }
  }
}

// acc[16 x HD] += P[16 x 16*KS] . Y over rows [y0, y0 + 16*KS) of a 64 x HD
// tile Y (rows = k): B(k, n) = Y[y0 + k][n], loaded with transpose.
// p: A fragments of P (KS k-steps).
template <int HD, int KS = 4>
LLM_DEV void mma_ab(float (&acc)[HD / 8][4], const uint32_t (&p)[KS][4], const Tile<HD> &y,
                    int y0 = 0) {
  int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 0; k < KS; k++) {
    int row = y0 + k * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
    for (int np = 0; np < HD / 16; np++) {
      int col = np * 16 + (lane >> 4) * 8;
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(sm(&y.v[row * Tile<HD>::LD + col]), b0, b1, b2, b3);
      mma16816(acc[2 * np], p[k], b0, b1);
      mma16816(acc[2 * np + 1], p[k], b2, b3);
    }
  }
}

// C fragments of a 16 x 8*NT fp32 tile -> A fragments (bf16) over its columns.
template <int NT = 8>
LLM_DEV void c_to_a(const float (&s)[NT][4], uint32_t (&p)[NT / 2][4]) {
#pragma unroll
  for (int k = 0; k < NT / 2; k++) {
    p[k][0] = pack2(s[2 * k][0], s[2 * k][1]);
    p[k][1] = pack2(s[2 * k][2], s[2 * k][3]);
    p[k][2] = pack2(s[2 * k + 1][0], s[2 * k + 1][1]);
    p[k][3] = pack2(s[2 * k + 1][2], s[2 * k + 1][3]);
  }
}

// Rotate one accumulator row (r) of a 16 x HD tile by -angle(pos): columns j
// and j + HD/2 (n tiles i and i + HD/16) pair up; the backward of the
// rotate-half RoPE.
template <int HD>
LLM_DEV void rope_bwd_row(float (&acc)[HD / 8][4], int r, const float *ct, const float *st) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < HD / 16; i++)
#pragma unroll
    for (int e = 0; e < 2; e++) {
      int j = 8 * i + 2 * (lane & 3) + e;
      float c = ct[j], sn = st[j];
      float x = acc[i][2 * r + e], y = acc[i + HD / 16][2 * r + e];
      acc[i][2 * r + e] = x * c + y * sn;
      acc[i + HD / 16][2 * r + e] = y * c - x * sn;
    }
}

// ------------------------------------------------------------------ dropout
// Factors of the probabilities (element (hrow + i) T + j of the site, hrow =
// (b H + h) T) a thread holds in one 8-column tile of a warp's 16-row tile.
// With T % 4 == 0 the keys 4m .. 4m + 3 of a query are one generator group
// (the context's offset drop.e0, a multiple of H T^2, keeps them aligned),
// so the warp's 32 groups of the tile are drawn once each, one per lane, and
// the keep bits go to their holders by shuffles; otherwise every element
// draws its own group.
//
// Query-row tiles (forward, dQ): rows r0 + 0..15 are queries, columns k8 +
// 0..7 keys; a thread holds rows (lane >> 2) + 8 (e >> 1), columns
// 2 (lane & 3) + (e & 1).  Lane x draws row (x >> 2) + 8 (x & 1), keys
// 4 ((x >> 1) & 1) .. + 3, so element e's bits are in lane (lane & ~1) |
// (e >> 1), at bit 2 (lane & 1) + (e & 1).
LLM_DEV void drop_q_tile(const DropArgs &drop, uint64_t hrow, int T, int r0, int k8, int lane,
                         uint32_t step, float (&f)[4]) {
  if ((T & 3) == 0) {
    const int rx = r0 + (lane >> 2) + (lane & 1) * 8, kx = k8 + ((lane >> 1) & 1) * 4;
    const uint32_t mine = drop_bits4(drop, (drop.e0 + (hrow + rx) * (uint64_t)T + kx) >> 2, step);
    const uint32_t lo = __shfl_sync(0xffffffffu, mine, lane & ~1);
    const uint32_t hi = __shfl_sync(0xffffffffu, mine, lane | 1);
    const int sh = (lane & 1) * 2;
#pragma unroll
    for (int e = 0; e < 4; e++)
      f[e] = (((e >> 1) ? hi : lo) >> (sh + (e & 1))) & 1u ? drop.scale : 0.f;
  } else {
#pragma unroll
    for (int e = 0; e < 4; e++) {
      const int qi = r0 + (lane >> 2) + (e >> 1) * 8, kj = k8 + (lane & 3) * 2 + (e & 1);
      f[e] = drop_factor(drop, (hrow + qi) * (uint64_t)T + kj, step);
    }
  }
}
// Key-row tiles (dK/dV): rows kr0 + 0..15 are keys, columns q8 + 0..7
// queries; a thread holds keys (lane >> 2) + 8 (e >> 1), queries
// 2 (lane & 3) + (e & 1).  Lane x draws query x >> 2, keys 4 (x & 3) .. + 3,
// so element e's bits are in lane 4 (2 (lane & 3) + (e & 1)) + (lane >> 4) +
// 2 (e >> 1), at bit (lane >> 2) & 3.
LLM_DEV void drop_k_tile(const DropArgs &drop, uint64_t hrow, int T, int kr0, int q8, int lane,
                         uint32_t step, float (&f)[4]) {
  if ((T & 3) == 0) {
    const int qx = q8 + (lane >> 2), kx = kr0 + (lane & 3) * 4;
    const uint32_t mine = drop_bits4(drop, (drop.e0 + (hrow + qx) * (uint64_t)T + kx) >> 2, step);
    const int sh = (lane >> 2) & 3;
#pragma unroll
    for (int e = 0; e < 4; e++) {
      const int src = 4 * ((lane & 3) * 2 + (e & 1)) + (lane >> 4) + 2 * (e >> 1);
      f[e] = (__shfl_sync(0xffffffffu, mine, src) >> sh) & 1u ? drop.scale : 0.f;
    }
  } else {
#pragma unroll
    for (int e = 0; e < 4; e++) {
      const int kj = kr0 + (lane >> 2) + (e >> 1) * 8, qi = q8 + (lane & 3) * 2 + (e & 1);
      f[e] = drop_factor(drop, (hrow + qi) * (uint64_t)T + kj, step);
    }
  }
}

// ------------------------------------------------------------------ forward
template <int HD, bool DROP>
__global__ void __launch_bounds__(NT) k_attn_fwd(const __nv_bfloat16 *__restrict__ qkv,
                                                 __nv_bfloat16 *__restrict__ o,
                                                 float *__restrict__ lse, int T, int H, int Hkv,
                                                 float scale, const DropArgs drop) {
  __shared__ Tile<HD> Qs, Ks[2], Vs[2];
  const uint32_t dstep = DROP ? (uint32_t)*drop.step : 0u;
  // grid (H, B, query blocks): blocks are dispatched x-fastest, so the last
  // (longest) query blocks of every head start first
  const int nqb = gridDim.z;
  const int qb = nqb - 1 - blockIdx.z;
  const int h = blockIdx.x, b = blockIdx.y;
  const int g = h / (H / Hkv);
  const int d = H * HD, kvd = Hkv * HD;
  const int64_t ld = d + 2 * kvd;
  const int w = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int q0 = qb * BQ;
  const __nv_bfloat16 *qbase = qkv + h * HD, *kbase = qkv + d + g * HD,
                      *vbase = qkv + d + kvd + g * HD;
  const int64_t roff = (int64_t)b * T;
  load_tile<HD>(Qs, qbase, ld, q0, T, roff);
  load_tile<HD>(Ks[0], kbase, ld, 0, T, roff);
  load_tile<HD>(Vs[0], vbase, ld, 0, T, roff);
  cp_commit();
  const float sl2 = scale * LOG2E;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  float acc[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; i++) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  uint32_t qf[HD / 16][4];
  const int row0 = q0 + w * 16 + (lane >> 2);  // this thread's rows: row0, row0 + 8
  for (int kb = 0; kb <= qb; kb++) {
    const int cur = kb & 1;
    if (kb < qb) {
      load_tile<HD>(Ks[cur ^ 1], kbase, ld, (kb + 1) * BKV, T, roff);
      load_tile<HD>(Vs[cur ^ 1], vbase, ld, (kb + 1) * BKV, T, roff);
    }
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    if (kb == 0) load_afrag<HD>(Qs, w, qf);
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; i++) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
    mma_abt<HD>(s, qf, Ks[cur]);
    // scale to log2 units, causal / length mask
    const int k0 = kb * BKV;
#pragma unroll
    for (int nt = 0; nt < 8; nt++) {
#pragma unroll
      for (int e = 0; e < 4; e++) {
        int qi = row0 + (e >> 1) * 8;
        int kj = k0 + nt * 8 + (lane & 3) * 2 + (e & 1);
        float v = s[nt][e] * sl2;
        s[nt][e] = (kj > qi || kj >= T) ? -INFINITY : v;
      }
    }
    // online softmax per row (a quad of lanes shares a row)
#pragma unroll
    for (int r = 0; r < 2; r++) {
      float mx = m[r];
#pragma unroll
      for (int nt = 0; nt < 8; nt++) mx = fmaxf(mx, fmaxf(s[nt][2 * r], s[nt][2 * r + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      float corr = (m[r] == -INFINITY) ? 0.f : tc::ex2(m[r] - mx);
      float rs = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; nt++) {
        float p0 = (mx == -INFINITY) ? 0.f : tc::ex2(s[nt][2 * r] - mx);
        float p1 = (mx == -INFINITY) ? 0.f : tc::ex2(s[nt][2 * r + 1] - mx);
        s[nt][2 * r] = p0;
        s[nt][2 * r + 1] = p1;
        rs += p0 + p1;
      }
      l[r] = l[r] * corr + rs;
      m[r] = mx;
#pragma unroll
      for (int i = 0; i < HD / 8; i++) {
        acc[i][2 * r] *= corr;
        acc[i][2 * r + 1] *= corr;
      }
    }
    if constexpr (DROP) {  // P V with the dropped probabilities P f; l keeps P's sums
      const uint64_t hrow = ((uint64_t)b * H + h) * T;
#pragma unroll
      for (int nt = 0; nt < 8; nt++) {
        float f[4];
        drop_q_tile(drop, hrow, T, q0 + w * 16, k0 + nt * 8, lane, dstep, f);
#pragma unroll
        for (int e = 0; e < 4; e++) s[nt][e] *= f[e];  // masked entries are 0 already
      }
    }
    uint32_t pf[4][4];
    c_to_a(s, pf);
    mma_ab<HD>(acc, pf, Vs[cur]);
    __syncthreads();  // buffer cur is refilled in the next iteration
  }
  // row sums across the quad, normalise, store
#pragma unroll
  for (int r = 0; r < 2; r++) {
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
  }
#pragma unroll
  for (int r = 0; r < 2; r++) {
    int qi = row0 + r * 8;
    if (qi >= T) continue;
    float inv = 1.f / l[r];
    __nv_bfloat16 *orow = o + ((int64_t)b * T + qi) * d + h * HD + (lane & 3) * 2;
#pragma unroll
    for (int i = 0; i < HD / 8; i++)
      *reinterpret_cast<uint32_t *>(orow + i * 8) = pack2(acc[i][2 * r] * inv, acc[i][2 * r + 1] * inv);
    if ((lane & 3) == 0) lse[((int64_t)b * H + h) * T + qi] = (m[r] + log2f(l[r])) * LN2;
  }
}

// ---------------------------------------------------------------- backward
template <int HD, bool DROP>
__global__ void __launch_bounds__(NT) k_attn_dq(const __nv_bfloat16 *__restrict__ qkv,
                                                const __nv_bfloat16 *__restrict__ o,
                                                const __nv_bfloat16 *__restrict__ dout,
                                                const float *__restrict__ lse,
                                                float *__restrict__ Dv,
                                                __nv_bfloat16 *__restrict__ dqkv,
                                                const float *__restrict__ cos_t,
                                                const float *__restrict__ sin_t, int T, int H,
                                                int Hkv, float scale, const DropArgs drop) {
  __shared__ Tile<HD> Ks[2], Vs[2];
  __shared__ float Dsh[64];
  const uint32_t dstep = DROP ? (uint32_t)*drop.step : 0u;
  const int nqb = gridDim.z;
  const int qb = nqb - 1 - blockIdx.z;
  const int h = blockIdx.x, b = blockIdx.y;
  const int g = h / (H / Hkv);
  const int d = H * HD, kvd = Hkv * HD;
  const int64_t ld = d + 2 * kvd;
  const int w = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int q0 = qb * BQ;
  const int64_t roff = (int64_t)b * T;
  const __nv_bfloat16 *kbase = qkv + d + g * HD, *vbase = qkv + d + kvd + g * HD;
  // Q and dO pass through the second K/V buffers into registers first.
  load_tile<HD>(Ks[1], qkv + h * HD, ld, q0, T, roff);
  load_tile<HD>(Vs[1], dout + h * HD, d, q0, T, roff);
  load_tile<HD>(Ks[0], kbase, ld, 0, T, roff);
  load_tile<HD>(Vs[0], vbase, ld, 0, T, roff);
  cp_commit();
  cp_wait<0>();
  __syncthreads();
  uint32_t qf[HD / 16][4], df[HD / 16][4];
  load_afrag<HD>(Ks[1], w, qf);
  load_afrag<HD>(Vs[1], w, df);
  {
    // D_i = sum_e dO_ie O_ie: two threads per row, halves combined by shuffle
    const int r = threadIdx.x >> 1, half = threadIdx.x & 1;
    const int qi = q0 + r;
    float acc_d = 0.f;
    if (qi < T) {
      const __nv_bfloat16 *orow = o + (roff + qi) * d + h * HD + half * (HD / 2);
      const __nv_bfloat16 *drow = &Vs[1].v[r * Tile<HD>::LD + half * (HD / 2)];
#pragma unroll
      for (int e = 0; e < HD / 2; e += 8) {
        uint4 a = *reinterpret_cast<const uint4 *>(orow + e);
        uint4 c = *reinterpret_cast<const uint4 *>(drow + e);
        const __nv_bfloat162 *ha = reinterpret_cast<const __nv_bfloat162 *>(&a);
        const __nv_bfloat162 *hc = reinterpret_cast<const __nv_bfloat162 *>(&c);
#pragma unroll
        for (int k = 0; k < 4; k++) {
          float2 fa = __bfloat1622float2(ha[k]), fc = __bfloat1622float2(hc[k]);
          acc_d += fa.x * fc.x + fa.y * fc.y;
        }
      }
    }
    acc_d += __shfl_xor_sync(0xffffffffu, acc_d, 1);
    if (half == 0) {
      Dsh[r] = acc_d;
      if (qi < T) Dv[((int64_t)b * H + h) * T + qi] = acc_d;
    }
  }
  __syncthreads();
  const float sl2 = scale * LOG2E;
  const int row0 = q0 + w * 16 + (lane >> 2);
  float L2[2], Dr[2];
#pragma unroll
  for (int r = 0; r < 2; r++) {
    int qi = row0 + r * 8;
    bool ok = qi < T;
    L2[r] = ok ? lse[((int64_t)b * H + h) * T + qi] * LOG2E : 0.f;
    Dr[r] = Dsh[w * 16 + (lane >> 2) + r * 8];
  }
  float acc[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; i++) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  for (int kb = 0; kb <= qb; kb++) {
    const int cur = kb & 1;
    if (kb < qb) {
      load_tile<HD>(Ks[cur ^ 1], kbase, ld, (kb + 1) * BKV, T, roff);
      load_tile<HD>(Vs[cur ^ 1], vbase, ld, (kb + 1) * BKV, T, roff);
    }
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    float s[8][4], dp[8][4];
#pragma unroll
    for (int i = 0; i < 8; i++)
#pragma unroll
      for (int e = 0; e < 4; e++) s[i][e] = dp[i][e] = 0.f;
    mma_abt<HD>(s, qf, Ks[cur]);
    mma_abt<HD>(dp, df, Vs[cur]);
    const int k0 = kb * BKV;
#pragma unroll
    for (int nt = 0; nt < 8; nt++) {
      float f[4];
      if constexpr (DROP)
        drop_q_tile(drop, ((uint64_t)b * H + h) * T, T, q0 + w * 16, k0 + nt * 8, lane, dstep, f);
#pragma unroll
      for (int e = 0; e < 4; e++) {
        int r = e >> 1;
        int qi = row0 + r * 8;
        int kj = k0 + nt * 8 + (lane & 3) * 2 + (e & 1);
        const bool valid = !(kj > qi || kj >= T || qi >= T);
        float p = valid ? tc::ex2(s[nt][e] * sl2 - L2[r]) : 0.f;
        float dpv = dp[nt][e];
        // with dropout dP = f (dO . v), the forward having multiplied v by P f
        if constexpr (DROP) dpv *= f[e];
        s[nt][e] = p * (dpv - Dr[r]);  // dS
      }
    }
    uint32_t sf[4][4];
    c_to_a(s, sf);
    mma_ab<HD>(acc, sf, Ks[cur]);
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 2; r++) {
    int qi = row0 + r * 8;
    if (qi >= T) continue;
    if (cos_t) rope_bwd_row<HD>(acc, r, cos_t + (int64_t)qi * (HD / 2), sin_t + (int64_t)qi * (HD / 2));
    __nv_bfloat16 *dst = dqkv + ((int64_t)b * T + qi) * ld + h * HD + (lane & 3) * 2;
#pragma unroll
    for (int i = 0; i < HD / 8; i++)
      *reinterpret_cast<uint32_t *>(dst + i * 8) =
          pack2(acc[i][2 * r] * scale, acc[i][2 * r + 1] * scale);
  }
}

template <int HD, bool DROP>
__global__ void __launch_bounds__(NT) k_attn_dkv(const __nv_bfloat16 *__restrict__ qkv,
                                                 const __nv_bfloat16 *__restrict__ dout,
                                                 const float *__restrict__ lse,
                                                 const float *__restrict__ Dv,
                                                 __nv_bfloat16 *__restrict__ dqkv,
                                                 const float *__restrict__ cos_t,
                                                 const float *__restrict__ sin_t, int T, int H,
                                                 int Hkv, float scale, const DropArgs drop) {
  __shared__ Tile<HD> KVs, Qs[2], dOs[2];
  const uint32_t dstep = DROP ? (uint32_t)*drop.step : 0u;
  __shared__ float Ls[2][64], Ds[2][64];
  // grid (Hkv, B, key blocks): the first key blocks see the most query
  // blocks, and blocks are dispatched x-fastest, so they start first
  const int nkb = gridDim.z;
  const int kb = blockIdx.z;
  const int g = blockIdx.x, b = blockIdx.y;
  const int grp = H / Hkv;
  const int d = H * HD, kvd = Hkv * HD;
  const int64_t ld = d + 2 * kvd;
  const int w = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int k0 = kb * BKV;
  const int64_t roff = (int64_t)b * T;
  const float sl2 = scale * LOG2E;
  const int nqb = nkb;
  uint32_t kf[HD / 16][4], vf[HD / 16][4];
  // K tile -> fragments, then V tile -> fragments (one shared buffer)
  load_tile<HD>(KVs, qkv + d + g * HD, ld, k0, T, roff);
  cp_commit();
  cp_wait<0>();
  __syncthreads();
  load_afrag<HD>(KVs, w, kf);
  __syncthreads();
  load_tile<HD>(KVs, qkv + d + kvd + g * HD, ld, k0, T, roff);
  cp_commit();
  cp_wait<0>();
  __syncthreads();
  load_afrag<HD>(KVs, w, vf);
  float dk[HD / 8][4], dv[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; i++)
#pragma unroll
    for (int e = 0; e < 4; e++) dk[i][e] = dv[i][e] = 0.f;
  const int key0 = k0 + w * 16 + (lane >> 2);  // this thread's keys: key0, key0 + 8
  // (query head, query block) pairs in order: heads of the group, then blocks >= kb
  const int nsteps = grp * (nqb - kb);
  auto issue = [&](int step, int buf) {
    int hq = g * grp + step / (nqb - kb);
    int qb = kb + step % (nqb - kb);
    load_tile<HD>(Qs[buf], qkv + hq * HD, ld, qb * BQ, T, roff);
    load_tile<HD>(dOs[buf], dout + hq * HD, d, qb * BQ, T, roff);
    for (int i = threadIdx.x; i < 64; i += NT) {
      int qi = qb * BQ + i;
      bool ok = qi < T;
      Ls[buf][i] = ok ? lse[((int64_t)b * H + hq) * T + qi] * LOG2E : 0.f;
      Ds[buf][i] = ok ? Dv[((int64_t)b * H + hq) * T + qi] : 0.f;
    }
  };
  issue(0, 0);
  cp_commit();
  for (int step = 0; step < nsteps; step++) {
    const int cur = step & 1;
    const int qb = kb + step % (nqb - kb), hq = g * grp + step / (nqb - kb);
    if (step + 1 < nsteps) issue(step + 1, cur ^ 1);
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    // Two halves of 32 queries: S^T = K Q^T and dP^T = V dO^T (16 keys x 32
    // queries per warp), then dV += P^T dO and dK += dS^T Q over that half.
    const int q0 = qb * BQ;
#pragma unroll
    for (int hf = 0; hf < 2; hf++) {
      float s[4][4], dp[4][4];
#pragma unroll
      for (int i = 0; i < 4; i++)
#pragma unroll
        for (int e = 0; e < 4; e++) s[i][e] = dp[i][e] = 0.f;
      mma_abt<HD, 4>(s, kf, Qs[cur], hf * 32);
      mma_abt<HD, 4>(dp, vf, dOs[cur], hf * 32);
#pragma unroll
      for (int nt = 0; nt < 4; nt++) {
        // the forward multiplied v by P f: dV takes P f, dP takes f
        float f[4] = {1.f, 1.f, 1.f, 1.f};
        if constexpr (DROP)
          drop_k_tile(drop, ((uint64_t)b * H + hq) * T, T, k0 + w * 16, q0 + hf * 32 + nt * 8,
                      lane, dstep, f);
#pragma unroll
        for (int e = 0; e < 4; e++) {
          int kj = key0 + (e >> 1) * 8;
          int col = hf * 32 + nt * 8 + (lane & 3) * 2 + (e & 1);
          int qi = q0 + col;
          const bool valid = !(kj > qi || qi >= T || kj >= T);
          float p = valid ? tc::ex2(s[nt][e] * sl2 - Ls[cur][col]) : 0.f;
          s[nt][e] = p * f[e];                                // (P f)^T
          dp[nt][e] = p * (dp[nt][e] * f[e] - Ds[cur][col]);  // dS^T
        }
      }
      uint32_t pf[2][4], sf[2][4];
      c_to_a<4>(s, pf);
      c_to_a<4>(dp, sf);
      mma_ab<HD, 2>(dv, pf, dOs[cur], hf * 32);
      mma_ab<HD, 2>(dk, sf, Qs[cur], hf * 32);
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 2; r++) {
    int kj = key0 + r * 8;
    if (kj >= T) continue;
    if (cos_t) rope_bwd_row<HD>(dk, r, cos_t + (int64_t)kj * (HD / 2), sin_t + (int64_t)kj * (HD / 2));
    __nv_bfloat16 *dkr = dqkv + ((int64_t)b * T + kj) * ld + d + g * HD + (lane & 3) * 2;
    __nv_bfloat16 *dvr = dkr + kvd;
#pragma unroll
    for (int i = 0; i < HD / 8; i++) {
      *reinterpret_cast<uint32_t *>(dkr + i * 8) = pack2(dk[i][2 * r] * scale, dk[i][2 * r + 1] * scale);
      *reinterpret_cast<uint32_t *>(dvr + i * 8) = pack2(dv[i][2 * r], dv[i][2 * r + 1]);
    }
  }
}

}  // namespace attn

bool attn_mma_covers(DType dt, int hd) { return dt == DT_BF16 && (hd == 32 || hd == 64); }

void attn_fwd_mma(const void *qkv, void *o, float *lse, int B, int T, int H, int Hkv, int hd,
                  cudaStream_t s, DropArgs drop) {
  using namespace attn;
  dim3 grid(H, B, (T + BQ - 1) / BQ);
  float scale = 1.0f / sqrtf((float)hd);
  auto launch = [&](auto kern) {
    kern<<<grid, NT, 0, s>>>((const __nv_bfloat16 *)qkv, (__nv_bfloat16 *)o, lse, T, H, Hkv, scale,
                             drop);
  };
  if (hd == 64) drop.on ? launch(k_attn_fwd<64, true>) : launch(k_attn_fwd<64, false>);
  else drop.on ? launch(k_attn_fwd<32, true>) : launch(k_attn_fwd<32, false>);
  count_launch();
}

void attn_bwd_mma(const void *qkv, const void *o, const void *dout, const float *lse, float *Dbuf,
                  void *dqkv, int B, int T, int H, int Hkv, int hd, const float *cos_t,
                  const float *sin_t, cudaStream_t s, DropArgs drop) {
  using namespace attn;
  float scale = 1.0f / sqrtf((float)hd);
  const __nv_bfloat16 *q = (const __nv_bfloat16 *)qkv, *oo = (const __nv_bfloat16 *)o,
                      *dO = (const __nv_bfloat16 *)dout;
  __nv_bfloat16 *dq = (__nv_bfloat16 *)dqkv;
  dim3 gq(H, B, (T + BQ - 1) / BQ), gkv(Hkv, B, (T + BKV - 1) / BKV);
  auto launch = [&](auto kdq, auto kdkv) {
    kdq<<<gq, NT, 0, s>>>(q, oo, dO, lse, Dbuf, dq, cos_t, sin_t, T, H, Hkv, scale, drop);
    kdkv<<<gkv, NT, 0, s>>>(q, dO, lse, Dbuf, dq, cos_t, sin_t, T, H, Hkv, scale, drop);
  };
  if (hd == 64)
    drop.on ? launch(k_attn_dq<64, true>, k_attn_dkv<64, true>)
            : launch(k_attn_dq<64, false>, k_attn_dkv<64, false>);
  else
    drop.on ? launch(k_attn_dq<32, true>, k_attn_dkv<32, true>)
            : launch(k_attn_dq<32, false>, k_attn_dkv<32, false>);
  count_launch(2);
}

}  // namespace llm
