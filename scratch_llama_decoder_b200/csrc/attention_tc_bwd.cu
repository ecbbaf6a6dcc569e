// tcgen05 flash-attention backward for head size 64 (bf16 operands, fp32
// scores and accumulators).  With the forward's saved row log-sum-exp L and
// D_i = sum_e dO_ie O_ie, the causal softmax backward of strata's flash
// attention is, per (query i, key j) pair,
//     P_ij  = exp(scale * q_i.k_j - L_i)          (0 above the diagonal)
//     dS_ij = P_ij (dO_i.v_j - D_i)
//     dQ = scale * dS K,   dK = scale * dS^T Q,   dV = P^T dO,
// recomputed block by block so no T x T matrix reaches memory.  Two kernels,
// both with 128 x 128 blocks, one CTA per SM (512 TMEM columns), 19 warps:
//   warp 0      TMA producer (Q/dO or K/V once, the other pair through a
//               2-deep ring);
//   warps 1, 18 MMA issuers A and B (whole converged warps, one elected lane;
//               one warp issues a tcgen05.mma only every ~127 cycles whatever
//               N is, so the products are split between two warps); warp 1
//               also allocates TMEM;
//   warps 2..17 elementwise warps, four per TMEM lane quarter: thread = one
//               row of the block (TMEM lane) and one column group (32 of the
//               block's 128 columns); four groups per row keep enough warps
//               in flight to cover the TMEM, SFU and shared-memory latencies.
// dQ kernel (grid H x B x query blocks, longest rows first), per key block j:
//   S = Q K_j^T (issuer A) and dP = dO V_j^T (issuer B) (M 128, N 128, K 64;
//   operands K-major in shared memory) into TMEM; the elementwise warps read
//   both rows, release them (so the next block's products start), form dS in
//   bf16 and put it back into TMEM; dQ_a += dS[:, 0:64] K_j[0:64] (A) and
//   dQ_b += dS[:, 64:128] K_j[64:128] (B) (M 128, N 64, K 64; A = dS from
//   TMEM, B = K_j MN-major), dQ = dQ_a + dQ_b at the end, so each key half
//   of the elementwise warps runs its own pipeline.  The same kernel first
//   forms D (one dot product per row) and stores it for the second kernel.
// dK/dV kernel (grid Hkv x B x key blocks, first key blocks first), per (query
//   head of the group, query block >= this key block):
//   S^T = K Q^T (A) and dP^T = V dO^T (B) into TMEM; P^T and dS^T back into
//   TMEM as bf16; dV += P^T dO (A) and dK += dS^T Q (B) (A operands from
//   TMEM, B = dO / Q MN-major).
//   The per-query L and D of each step travel with its Q/dO tiles.
// dQ and dK leave through the backward of the rotate-half RoPE (when tables
// are given), then scale, bf16.  No atomics: every output element is written
// once by the CTA that owns its row.  Every wait is bounded (FLAG_TIMEOUT,
// then drain and free TMEM).
#include "common.cuh"
#include "gemm_tc.h"
#include "tcgen05.cuh"

namespace llm {
namespace attn_tc_bwd {

using namespace tc;

constexpr int BQ = 128, BK = 128, HD = 64;
constexpr int TILE_BYTES = 128 * HD * 2;  // 16 KB: 128 rows x 64 bf16, 128-byte swizzle
constexpr int STAGES = 4;  // streamed-operand rings: deep enough to cover the TMA latency
constexpr int EW_WARPS = 16;  // elementwise warps: 4 lane quarters x NCQ column groups
constexpr int NCQ = EW_WARPS / 4;  // column groups of a row (2 or 4)
constexpr int CW = 128 / NCQ;      // score columns per thread
constexpr int HW = 32 / NCQ;       // head columns per thread in each RoPE half
constexpr int MMA_B_WARP = 2 + EW_WARPS;  // second MMA-issuing warp
constexpr int NTHREADS = 32 * (MMA_B_WARP + 1);
constexpr int TMEM_COLS = 512;
constexpr float LOG2E = 1.4426950408889634f;

// dQ kernel: TMEM columns; shared memory Q | dO | K[2] | V[2] | barriers | red
constexpr int DQ_COL_S = 0, DQ_COL_DP = 128, DQ_COL_DS = 256, DQ_COL_DQA = 320, DQ_COL_DQB = 384;
constexpr int BAR_BYTES = 512;  // 48 mbarrier slots, then the TMEM address and abort words
constexpr int DQ_SMEM = (2 + 2 * STAGES) * TILE_BYTES + 1024 + BAR_BYTES + NCQ * 128 * 4;
// dK/dV kernel: TMEM columns; shared memory K | V | Q[2] | dO[2] | L[2] | D[2] | barriers
constexpr int KV_COL_S = 0, KV_COL_DP = 128, KV_COL_P = 256, KV_COL_DS = 320, KV_COL_DV = 384,
              KV_COL_DK = 448;
constexpr int KV_SMEM = (2 + 2 * STAGES) * TILE_BYTES + 2 * STAGES * 128 * 4 + BAR_BYTES + 1024;

// Named barrier of the elementwise warps (id 1).
LLM_DEV void ew_sync() { asm volatile("bar.sync 1, %0;" ::"n"(32 * EW_WARPS) : "memory"); }

// Backward of the rotate-half RoPE on N column pairs (c, c + 32) of one row:
// (x, y) <- (x cos + y sin, y cos - x sin), angle table entries ct[i], st[i].
template <int N>
LLM_DEV void rope_bwd_n(float (&x)[N], float (&y)[N], const float *ct, const float *st) {
#pragma unroll
  for (int i = 0; i < N; i += 4) {
    const float4 c = *reinterpret_cast<const float4 *>(ct + i);
    const float4 s = *reinterpret_cast<const float4 *>(st + i);
    const float cv[4] = {c.x, c.y, c.z, c.w}, sv[4] = {s.x, s.y, s.z, s.w};
#pragma unroll
    for (int e = 0; e < 4; e++) {
      const float a = x[i + e], b = y[i + e];
      x[i + e] = a * cv[e] + b * sv[e];
      y[i + e] = b * cv[e] - a * sv[e];
    }
  }
}

// N consecutive bf16 values (v * mul, N a multiple of 8) to a 16-byte
// aligned address.
template <int N>
LLM_DEV void store_n(__nv_bfloat16 *dst, const float (&v)[N], float mul) {
#pragma unroll
  for (int i = 0; i < N; i += 8)
    reinterpret_cast<uint4 *>(dst)[i / 8] =
        make_uint4(pack_bf16(v[i] * mul, v[i + 1] * mul), pack_bf16(v[i + 2] * mul, v[i + 3] * mul),
                   pack_bf16(v[i + 4] * mul, v[i + 5] * mul), pack_bf16(v[i + 6] * mul, v[i + 7] * mul));
}

LLM_DEV void tmem_alloc_512(uint32_t *dst) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(TMEM_COLS)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
LLM_DEV void tmem_free_512(uint32_t tmem) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS)
               : "memory");
}
// Bounded wait used only on the way out (the copies / MMAs of this thread).
LLM_DEV void drain_wait(uint32_t bar, uint32_t parity) {
  const unsigned long long t0 = gtimer();
  while (!mbar_try(bar, parity) && gtimer() - t0 < WAIT_NS) {
  }
}

// ------------------------------------------------------------------- dQ
__global__ void __launch_bounds__(NTHREADS, 1)
    k_attn_dq_tc(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_do,
                 const __nv_bfloat16 *__restrict__ o, const __nv_bfloat16 *__restrict__ dout,
                 const float *__restrict__ lse, float *__restrict__ Dv,
                 __nv_bfloat16 *__restrict__ dqkv, const float *__restrict__ cos_t,
                 const float *__restrict__ sin_t, int T, int H, int Hkv, float scale, int *gflag) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *sQ = smem, *sdO = smem + TILE_BYTES, *sK = smem + 2 * TILE_BYTES,
          *sV = sK + STAGES * TILE_BYTES;
  uint64_t *bars = (uint64_t *)(sV + STAGES * TILE_BYTES);
  uint32_t *tmem_sh = (uint32_t *)(bars + 48);
  volatile int *abort_sh = (volatile int *)(tmem_sh + 1);
  float *red = (float *)(bars + BAR_BYTES / 8);  // [NCQ][128] partial dot products
  const uint32_t b0 = smem_u32(bars);
  const uint32_t q_full = b0, k_full = b0 + 8, k_empty = k_full + 8 * STAGES,
                 v_full = k_empty + 8 * STAGES, v_empty = v_full + 8 * STAGES,
                 s_full = v_empty + 8 * STAGES, s_free = s_full + 8,
                 ds_full = s_free + 8,   // [2]: key half a, b
                 dq_done = ds_full + 16, // [2]
                 drain = dq_done + 16;   // [2]: one per MMA warp
  static_assert(3 + 4 * STAGES + 6 <= 48, "barriers overlap the TMEM address word");
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int nqb = gridDim.z, qb = nqb - 1 - blockIdx.z;
  const int h = blockIdx.x, b = blockIdx.y;
  const int g = h / (H / Hkv), d = H * HD, kvd = Hkv * HD;
  const int64_t ld = d + 2 * kvd;
  const int q0 = qb * BQ;
  const int nj = qb + 1;  // causal: key blocks 0..qb (block qb holds the diagonal)
  const int row_base = b * T;

  if (threadIdx.x == 0) {
    *abort_sh = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < STAGES; s++) {
      mbar_init(k_full + 8 * s, 1);
      mbar_init(k_empty + 8 * s, 2);  // dQ_a and dQ_b read K_j
      mbar_init(v_full + 8 * s, 1);
      mbar_init(v_empty + 8 * s, 1);
    }
    mbar_init(s_full, 2);  // S and dP
    mbar_init(s_free, EW_WARPS);
    for (int x = 0; x < 2; x++) {
      mbar_init(ds_full + 8 * x, EW_WARPS / 2);
      mbar_init(dq_done + 8 * x, 1);
      mbar_init(drain + 8 * x, 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc_512(tmem_sh);
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_sh;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      int issued = 0;
      mbar_arrive_expect_tx(q_full, 2 * TILE_BYTES);
      tma_load_2d(smem_u32(sQ), &tm_qkv, h * HD, row_base + q0, q_full);
      tma_load_2d(smem_u32(sdO), &tm_do, h * HD, row_base + q0, q_full);
      for (int j = 0; j < nj; j++) {
        const int s = j % STAGES;
        const uint32_t ph = (j / STAGES) & 1;
        if (!mbar_wait(k_empty + 8 * s, ph ^ 1, abort_sh, gflag)) break;
        if (!mbar_wait(v_empty + 8 * s, ph ^ 1, abort_sh, gflag)) break;
        mbar_arrive_expect_tx(k_full + 8 * s, TILE_BYTES);
        tma_load_2d(smem_u32(sK + s * TILE_BYTES), &tm_qkv, d + g * HD, row_base + j * BK,
                    k_full + 8 * s);
        mbar_arrive_expect_tx(v_full + 8 * s, TILE_BYTES);
        tma_load_2d(smem_u32(sV + s * TILE_BYTES), &tm_qkv, d + kvd + g * HD, row_base + j * BK,
                    v_full + 8 * s);
        issued = j + 1;
      }
      // every copy this thread issued has landed before the CTA may exit
      drain_wait(q_full, 0);
      for (int j = max(0, issued - STAGES); j < issued; j++) {
        drain_wait(k_full + 8 * (j % STAGES), (j / STAGES) & 1);
        drain_wait(v_full + 8 * (j % STAGES), (j / STAGES) & 1);
      }
    }
  } else if (warp == 1 || warp == MMA_B_WARP) {
    // ------------------------------------- MMA issuers (whole warps)
    // A: S = Q K_j^T, dQ_a += dS_a K_j[0:64];  B: dP = dO V_j^T, dQ_b += dS_b K_j[64:128]
    const int x = warp == 1 ? 0 : 1;
    constexpr uint32_t ID_S = idesc_mn(128, BK, false, false);
    constexpr uint32_t ID_DQ = idesc_mn(128, HD, false, true);
    const uint64_t ad = sdesc(smem_u32(x ? sdO : sQ), 16, 1024);
    uint8_t *sB = x ? sV : sK;
    const uint32_t b_full = x ? v_full : k_full;
    const uint32_t col = x ? DQ_COL_DP : DQ_COL_S;
    auto issue_prod = [&](int j) {
      const int s = j % STAGES;
      const uint64_t bd = sdesc(smem_u32(sB + s * TILE_BYTES), 16, 1024);
#pragma unroll
      for (int kk = 0; kk < HD / 16; kk++)
        mma_bf16_e(tmem + col, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), ID_S,
                   kk > 0 ? 1u : 0u);
      mma_commit_e(s_full);
      if (x) mma_commit_e(v_empty + 8 * s);  // V_j is not read again
    };
    bool ok = warp_wait(q_full, 0, abort_sh, gflag) && warp_wait(b_full, 0, abort_sh, gflag);
    if (ok) {
      fence_after();
      issue_prod(0);
    }
    for (int j = 0; j < nj && ok; j++) {
      const int s = j % STAGES;
      const uint32_t ph = (j / STAGES) & 1;
      if (j + 1 < nj) {
        // next block's products once the elementwise warps have read S, dP
        const int s1 = (j + 1) % STAGES;
        const uint32_t ph1 = ((j + 1) / STAGES) & 1;
        if (!warp_wait(b_full + 8 * s1, ph1, abort_sh, gflag) ||
            !warp_wait(s_free, j & 1, abort_sh, gflag)) {
          ok = false;
          break;
        }
        fence_after();
        issue_prod(j + 1);
      }
      if (!warp_wait(ds_full + 8 * x, j & 1, abort_sh, gflag) ||
          (x && !warp_wait(k_full + 8 * s, ph, abort_sh, gflag))) {
        ok = false;
        break;
      }
      fence_after();
      const uint64_t kmd = sdesc(smem_u32(sK + s * TILE_BYTES), 8192, 1024);
#pragma unroll
      for (int kk = 0; kk < 4; kk++)
        mma_ts_e(tmem + (x ? DQ_COL_DQB : DQ_COL_DQA), tmem + DQ_COL_DS + x * 32 + kk * 8,
                 kmd + (uint64_t)((x * 4 + kk) * 128), ID_DQ, (j > 0 || kk > 0) ? 1u : 0u);
      mma_commit_e(k_empty + 8 * s);
      mma_commit_e(dq_done + 8 * x);
    }
    mma_commit_e(drain + 8 * x);
    if (lane == 0) drain_wait(drain + 8 * x, 0);
    __syncwarp();
  } else {
    // --------------------------------------------------------- elementwise
    const int quarter = warp & 3;
    const int cq = (warp - 2) >> 2;  // column group: keys [cq CW, cq CW + CW) of the block
    const int x = cq / (NCQ / 2);    // key half (dQ_a or dQ_b) this group feeds
    const int r = quarter * 32 + lane;
    const int qi = q0 + r;
    const bool valid = qi < T;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float sl2 = scale * LOG2E;
    // D_i = dO_i . O_i, each thread over 64 / NCQ of the 64 head columns
    float dpart = 0.f;
    if (valid) {
      const int64_t off = ((int64_t)row_base + qi) * d + h * HD + cq * (HD / NCQ);
      const uint4 *po = reinterpret_cast<const uint4 *>(o + off);
      const uint4 *pd = reinterpret_cast<const uint4 *>(dout + off);
#pragma unroll
      for (int e = 0; e < HD / NCQ / 8; e++) {
        const uint4 a = po[e], c = pd[e];
        const __nv_bfloat162 *ha = reinterpret_cast<const __nv_bfloat162 *>(&a);
        const __nv_bfloat162 *hc = reinterpret_cast<const __nv_bfloat162 *>(&c);
#pragma unroll
        for (int k = 0; k < 4; k++) {
          const float2 fa = __bfloat1622float2(ha[k]), fc = __bfloat1622float2(hc[k]);
          dpart += fa.x * fc.x + fa.y * fc.y;
        }
      }
    }
    red[cq * 128 + r] = dpart;
    ew_sync();
    float Di = 0.f;
#pragma unroll
    for (int c = 0; c < NCQ; c++) Di += red[c * 128 + r];
    // rows past T get L = +inf, so every P of theirs is 0
    const float L2 = valid ? lse[((int64_t)b * H + h) * T + qi] * LOG2E : INFINITY;
    if (cq == 0 && valid) Dv[((int64_t)b * H + h) * T + qi] = Di;
    bool ok = true;
    for (int j = 0; j < nj && ok; j++) {
      if (!warp_wait(s_full, j & 1, abort_sh, gflag)) {
        ok = false;
        break;
      }
      fence_after();
      float sv[CW], dv[CW];
      tmem_ldn<CW>(tmem + lane_off + DQ_COL_S + cq * CW, sv);
      tmem_ldn<CW>(tmem + lane_off + DQ_COL_DP + cq * CW, dv);
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);  // the MMA warps may overwrite S and dP now
      const int k0 = j * BK + cq * CW;
      const bool diag = (j == qb);  // only the diagonal block masks (keys >= T lie above it)
      uint32_t w[CW / 2];
      if (diag) {  // the causal mask only on the diagonal block
#pragma unroll
        for (int i = 0; i < CW; i += 2) {
          float p0 = ex2(fmaf(sv[i], sl2, -L2)), p1 = ex2(fmaf(sv[i + 1], sl2, -L2));
          if (k0 + i > qi) p0 = 0.f;
          if (k0 + i + 1 > qi) p1 = 0.f;
          w[i / 2] = pack_bf16(p0 * (dv[i] - Di), p1 * (dv[i + 1] - Di));
        }
      } else {
#pragma unroll
        for (int i = 0; i < CW; i += 2) {
          const float p0 = ex2(fmaf(sv[i], sl2, -L2)), p1 = ex2(fmaf(sv[i + 1], sl2, -L2));
          w[i / 2] = pack_bf16(p0 * (dv[i] - Di), p1 * (dv[i + 1] - Di));
        }
      }
      // this half's dS of the previous block is free once its dQ product completed
      if (j > 0) {
        if (!warp_wait(dq_done + 8 * x, (j - 1) & 1, abort_sh, gflag)) {
          ok = false;
          break;
        }
        fence_after();
      }
#pragma unroll
      for (int c = 0; c < CW / 2; c += 16)
        tmem_stn<(CW / 2 < 16 ? CW / 2 : 16)>(tmem + lane_off + DQ_COL_DS + cq * (CW / 2) + c, w + c);
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_full + 8 * x);
    }
    if (ok)
      ok = warp_wait(dq_done, (nj - 1) & 1, abort_sh, gflag) &&
           warp_wait(dq_done + 8, (nj - 1) & 1, abort_sh, gflag);
    if (ok) {
      fence_after();
      // column pairs (c, c + 32) of RoPE: this group takes c in [cq HW, cq HW + HW)
      float xa[HW], ya[HW], xb[HW], yb[HW];
      tmem_ldn<HW>(tmem + lane_off + DQ_COL_DQA + cq * HW, xa);
      tmem_ldn<HW>(tmem + lane_off + DQ_COL_DQA + 32 + cq * HW, ya);
      tmem_ldn<HW>(tmem + lane_off + DQ_COL_DQB + cq * HW, xb);
      tmem_ldn<HW>(tmem + lane_off + DQ_COL_DQB + 32 + cq * HW, yb);
#pragma unroll
      for (int i = 0; i < HW; i++) {
        xa[i] += xb[i];
        ya[i] += yb[i];
      }
      if (valid) {
        if (cos_t)
          rope_bwd_n<HW>(xa, ya, cos_t + (int64_t)qi * (HD / 2) + cq * HW,
                         sin_t + (int64_t)qi * (HD / 2) + cq * HW);
        __nv_bfloat16 *dst = dqkv + ((int64_t)row_base + qi) * ld + h * HD + cq * HW;
        store_n<HW>(dst, xa, scale);
        store_n<HW>(dst + 32, ya, scale);
      }
    }
  }
  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) tmem_free_512(tmem);
}

// ---------------------------------------------------------------- dK, dV
__global__ void __launch_bounds__(NTHREADS, 1)
    k_attn_dkv_tc(const __grid_constant__ CUtensorMap tm_qkv,
                  const __grid_constant__ CUtensorMap tm_do, const float *__restrict__ lse,
                  const float *__restrict__ Dv, __nv_bfloat16 *__restrict__ dqkv,
                  const float *__restrict__ cos_t, const float *__restrict__ sin_t, int T, int H,
                  int Hkv, float scale, int *gflag) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *sK = smem, *sV = smem + TILE_BYTES, *sQ = smem + 2 * TILE_BYTES,
          *sdO = sQ + STAGES * TILE_BYTES;
  float *sL = (float *)(sdO + STAGES * TILE_BYTES);  // [STAGES][128] L * log2(e)
  float *sD = sL + STAGES * 128;                      // [STAGES][128] D
  uint64_t *bars = (uint64_t *)(sD + STAGES * 128);
  uint32_t *tmem_sh = (uint32_t *)(bars + 48);
  volatile int *abort_sh = (volatile int *)(tmem_sh + 1);
  const uint32_t b0 = smem_u32(bars);
  const uint32_t kv_full = b0, q_full = b0 + 8, q_empty = q_full + 8 * STAGES,
                 ld_full = q_empty + 8 * STAGES, s_full = ld_full + 8 * STAGES,
                 s_free = s_full + 8, p_full = s_free + 8, pv_done = p_full + 8,
                 drain = pv_done + 8;  // drain [2]: one per MMA warp
  static_assert(1 + 3 * STAGES + 6 <= 48, "barriers overlap the TMEM address word");
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int nkb = gridDim.z, kb = blockIdx.z;
  const int g = blockIdx.x, b = blockIdx.y;
  const int grp = H / Hkv, d = H * HD, kvd = Hkv * HD;
  const int64_t ld = d + 2 * kvd;
  const int k0 = kb * BK;
  const int nq = nkb - kb;       // query blocks kb..nkb-1 see this key block
  const int nsteps = grp * nq;   // (query head of the group, query block) pairs
  const int row_base = b * T;

  if (threadIdx.x == 0) {
    *abort_sh = 0;
    mbar_init(kv_full, 1);
    for (int s = 0; s < STAGES; s++) {
      mbar_init(q_full + 8 * s, 1);
      mbar_init(q_empty + 8 * s, 2);  // both MMA warps read Q_s and dO_s
      mbar_init(ld_full + 8 * s, 32);
    }
    mbar_init(s_full, 2);   // S^T and dP^T
    mbar_init(s_free, EW_WARPS);
    mbar_init(p_full, EW_WARPS);
    mbar_init(pv_done, 2);  // dV and dK
    mbar_init(drain, 1);
    mbar_init(drain + 8, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc_512(tmem_sh);
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_sh;

  if (warp == 0) {
    // ---------------------------------------------- TMA producer (warp)
    if (lane == 0) {
      mbar_arrive_expect_tx(kv_full, 2 * TILE_BYTES);
      tma_load_2d(smem_u32(sK), &tm_qkv, d + g * HD, row_base + k0, kv_full);
      tma_load_2d(smem_u32(sV), &tm_qkv, d + kvd + g * HD, row_base + k0, kv_full);
    }
    int issued = 0;
    for (int st = 0; st < nsteps; st++) {
      const int s = st % STAGES;
      const uint32_t ph = (st / STAGES) & 1;
      const int hq = g * grp + st / nq, qb = kb + st % nq;
      // the slot (tiles and L, D) of step st - 2 is free once its products completed
      if (!warp_wait(q_empty + 8 * s, ph ^ 1, abort_sh, gflag)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(q_full + 8 * s, 2 * TILE_BYTES);
        tma_load_2d(smem_u32(sQ + s * TILE_BYTES), &tm_qkv, hq * HD, row_base + qb * BQ,
                    q_full + 8 * s);
        tma_load_2d(smem_u32(sdO + s * TILE_BYTES), &tm_do, hq * HD, row_base + qb * BQ,
                    q_full + 8 * s);
      }
      const int64_t base = ((int64_t)b * H + hq) * T;
#pragma unroll
      for (int i = lane; i < BQ; i += 32) {
        const int qi = qb * BQ + i;
        // queries past T get L = +inf, so every P of theirs is 0
        sL[s * 128 + i] = qi < T ? lse[base + qi] * LOG2E : INFINITY;
        sD[s * 128 + i] = qi < T ? Dv[base + qi] : 0.f;
      }
      mbar_arrive(ld_full + 8 * s);
      issued = st + 1;
    }
    if (lane == 0) {
      drain_wait(kv_full, 0);
      for (int st = max(0, issued - STAGES); st < issued; st++)
        drain_wait(q_full + 8 * (st % STAGES), (st / STAGES) & 1);
    }
  } else if (warp == 1 || warp == MMA_B_WARP) {
    // ------------------------------------- MMA issuers (whole warps)
    // A: S^T = K Q^T, dV += P^T dO;  B: dP^T = V dO^T, dK += dS^T Q
    const int x = warp == 1 ? 0 : 1;
    constexpr uint32_t ID_S = idesc_mn(128, BQ, false, false);
    constexpr uint32_t ID_KV = idesc_mn(128, HD, false, true);
    const uint64_t ad = sdesc(smem_u32(x ? sV : sK), 16, 1024);
    uint8_t *sB = x ? sdO : sQ;    // B of the scores product (K-major)
    uint8_t *sB2 = x ? sQ : sdO;   // B of the accumulation (MN-major)
    const uint32_t col = x ? KV_COL_DP : KV_COL_S;
    const uint32_t col_a2 = x ? KV_COL_DS : KV_COL_P, col_acc = x ? KV_COL_DK : KV_COL_DV;
    auto issue_prod = [&](int st) {
      const int s = st % STAGES;
      const uint64_t bd = sdesc(smem_u32(sB + s * TILE_BYTES), 16, 1024);
#pragma unroll
      for (int kk = 0; kk < HD / 16; kk++)
        mma_bf16_e(tmem + col, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), ID_S,
                   kk > 0 ? 1u : 0u);
      mma_commit_e(s_full);
    };
    bool ok = warp_wait(kv_full, 0, abort_sh, gflag) && warp_wait(q_full, 0, abort_sh, gflag);
    if (ok) {
      fence_after();
      issue_prod(0);
    }
    for (int st = 0; st < nsteps && ok; st++) {
      const int s = st % STAGES;
      if (st + 1 < nsteps) {
        const int s1 = (st + 1) % STAGES;
        const uint32_t ph1 = ((st + 1) / STAGES) & 1;
        if (!warp_wait(q_full + 8 * s1, ph1, abort_sh, gflag) ||
            !warp_wait(s_free, st & 1, abort_sh, gflag)) {
          ok = false;
          break;
        }
        fence_after();
        issue_prod(st + 1);
      }
      if (!warp_wait(p_full, st & 1, abort_sh, gflag)) {
        ok = false;
        break;
      }
      fence_after();
      const uint64_t bm = sdesc(smem_u32(sB2 + s * TILE_BYTES), 8192, 1024);
#pragma unroll
      for (int kk = 0; kk < BQ / 16; kk++)
        mma_ts_e(tmem + col_acc, tmem + col_a2 + kk * 8, bm + (uint64_t)(kk * 128), ID_KV,
                 (st > 0 || kk > 0) ? 1u : 0u);
      mma_commit_e(q_empty + 8 * s);
      mma_commit_e(pv_done);
    }
    mma_commit_e(drain + 8 * x);
    if (lane == 0) drain_wait(drain + 8 * x, 0);
    __syncwarp();
  } else {
    // --------------------------------------------------------- elementwise
    const int quarter = warp & 3;
    const int cq = (warp - 2) >> 2;  // column group: queries [cq CW, cq CW + CW) of the block
    const int r = quarter * 32 + lane;
    const int kj = k0 + r;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float sl2 = scale * LOG2E;
    bool ok = true;
    for (int st = 0; st < nsteps && ok; st++) {
      const int s = st % STAGES;
      const int qb = kb + st % nq;
      if (!warp_wait(s_full, st & 1, abort_sh, gflag) ||
          !warp_wait(ld_full + 8 * s, (st / STAGES) & 1, abort_sh, gflag)) {
        ok = false;
        break;
      }
      fence_after();
      float sv[CW], dv[CW];
      tmem_ldn<CW>(tmem + lane_off + KV_COL_S + cq * CW, sv);
      tmem_ldn<CW>(tmem + lane_off + KV_COL_DP + cq * CW, dv);
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);
      const int qc0 = qb * BQ + cq * CW;
      const bool diag = (qb == kb);  // keys >= T occur only in this case, above the diagonal
      const float4 *L4 = reinterpret_cast<const float4 *>(sL + s * 128 + cq * CW);
      const float4 *D4 = reinterpret_cast<const float4 *>(sD + s * 128 + cq * CW);
      uint32_t wp[CW / 2], wd[CW / 2];
#pragma unroll
      for (int i = 0; i < CW; i += 4) {
        const float4 lq = L4[i / 4], dq = D4[i / 4];
        float p0 = ex2(fmaf(sv[i], sl2, -lq.x)), p1 = ex2(fmaf(sv[i + 1], sl2, -lq.y));
        float p2 = ex2(fmaf(sv[i + 2], sl2, -lq.z)), p3 = ex2(fmaf(sv[i + 3], sl2, -lq.w));
        if (diag) {
          if (kj > qc0 + i) p0 = 0.f;
          if (kj > qc0 + i + 1) p1 = 0.f;
          if (kj > qc0 + i + 2) p2 = 0.f;
          if (kj > qc0 + i + 3) p3 = 0.f;
        }
        wp[i / 2] = pack_bf16(p0, p1);
        wp[i / 2 + 1] = pack_bf16(p2, p3);
        wd[i / 2] = pack_bf16(p0 * (dv[i] - dq.x), p1 * (dv[i + 1] - dq.y));
        wd[i / 2 + 1] = pack_bf16(p2 * (dv[i + 2] - dq.z), p3 * (dv[i + 3] - dq.w));
      }
      // P^T and dS^T of the previous step are free once its products completed
      if (st > 0) {
        if (!warp_wait(pv_done, (st - 1) & 1, abort_sh, gflag)) {
          ok = false;
          break;
        }
        fence_after();
      }
#pragma unroll
      for (int c = 0; c < CW / 2; c += 16) {
        tmem_stn<(CW / 2 < 16 ? CW / 2 : 16)>(tmem + lane_off + KV_COL_P + cq * (CW / 2) + c, wp + c);
        tmem_stn<(CW / 2 < 16 ? CW / 2 : 16)>(tmem + lane_off + KV_COL_DS + cq * (CW / 2) + c, wd + c);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok) ok = warp_wait(pv_done, (nsteps - 1) & 1, abort_sh, gflag);
    if (ok) {
      fence_after();
      // column pairs (c, c + 32) of RoPE: this group takes c in [cq HW, cq HW + HW)
      float xx[HW], yy[HW];
      __nv_bfloat16 *dst = dqkv + ((int64_t)row_base + kj) * ld + d + g * HD + cq * HW;
      tmem_ldn<HW>(tmem + lane_off + KV_COL_DK + cq * HW, xx);
      tmem_ldn<HW>(tmem + lane_off + KV_COL_DK + 32 + cq * HW, yy);
      if (kj < T) {
        if (cos_t)
          rope_bwd_n<HW>(xx, yy, cos_t + (int64_t)kj * (HD / 2) + cq * HW,
                         sin_t + (int64_t)kj * (HD / 2) + cq * HW);
        store_n<HW>(dst, xx, scale);
        store_n<HW>(dst + 32, yy, scale);
      }
      tmem_ldn<HW>(tmem + lane_off + KV_COL_DV + cq * HW, xx);
      tmem_ldn<HW>(tmem + lane_off + KV_COL_DV + 32 + cq * HW, yy);
      if (kj < T) {
        store_n<HW>(dst + kvd, xx, 1.f);
        store_n<HW>(dst + kvd + 32, yy, 1.f);
      }
    }
  }
  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) tmem_free_512(tmem);
}

}  // namespace attn_tc_bwd

// Host side: tensor maps over qkv [B*T, qkvw] and dout [B*T, H*hd] (box 64 x
// 128); the dQ kernel runs first (it also writes D), then the dK/dV kernel.
bool attn_bwd_tc(const void *qkv, const void *o, const void *dout, const float *lse, float *Dbuf,
                 void *dqkv, int B, int T, int H, int Hkv, int hd, const float *cos_t,
                 const float *sin_t, int *flag, cudaStream_t s) {
  using namespace attn_tc_bwd;
  if (hd != HD || !flag || ((uintptr_t)o & 15) || ((uintptr_t)dqkv & 15) ||
      ((uintptr_t)cos_t & 15) || ((uintptr_t)sin_t & 15) || (!cos_t != !sin_t))
    return false;
  if (!smem_optin((const void *)k_attn_dq_tc, DQ_SMEM) ||
      !smem_optin((const void *)k_attn_dkv_tc, KV_SMEM))
    return false;
  const int64_t qkvw = (int64_t)(H + 2 * Hkv) * hd, dw = (int64_t)H * hd;
  CUtensorMap mq, md;
  if (!tc::tile_map_bf16(&mq, qkv, qkvw, (int64_t)B * T, qkvw, 128) ||
      !tc::tile_map_bf16(&md, dout, dw, (int64_t)B * T, dw, 128))
    return false;
  const int nb = (T + BQ - 1) / BQ;
  const float scale = 1.0f / sqrtf((float)hd);
  k_attn_dq_tc<<<dim3(H, B, nb), NTHREADS, DQ_SMEM, s>>>(
      mq, md, (const __nv_bfloat16 *)o, (const __nv_bfloat16 *)dout, lse, Dbuf,
      (__nv_bfloat16 *)dqkv, cos_t, sin_t, T, H, Hkv, scale, flag);
  k_attn_dkv_tc<<<dim3(Hkv, B, nb), NTHREADS, KV_SMEM, s>>>(mq, md, lse, Dbuf,
                                                            (__nv_bfloat16 *)dqkv, cos_t, sin_t,
                                                            T, H, Hkv, scale, flag);
  count_launch(2);
  return true;
}

}  // namespace llm
