// tcgen05 flash-attention backward for head sizes 64 and 32 (bf16 operands,
// fp32 scores and accumulators; a head-32 tile is the head-64 one with its
// upper 32 columns loaded as zeros, so every product and D below is the
// head-32 one, and only the head's own columns are stored).  With the forward's saved row log-sum-exp L and
// D_i = sum_e dO_ie O_ie, the causal softmax backward of strata's flash
// attention is, per (query i, key j) pair,
//     P_ij  = exp(scale * q_i.k_j - L_i)          (0 above the diagonal)
//     dS_ij = P_ij (dO_i.v_j - D_i)
//     dQ = scale * dS K,   dK = scale * dS^T Q,   dV = P^T dO,
// recomputed block by block so no T x T matrix reaches memory.  Two kernels,
// both with 128 x 128 blocks, one CTA per SM (512 TMEM columns), 19 warps:
//   warp 0      TMA producer (Q/dO or K/V once, the other pair through a
//               STAGES-deep ring);
//   warps 1, 18 MMA issuers A and B (whole converged warps, one elected lane),
//               each waiting only on the barriers of its own products; warp 1
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
//   The per-query L and D of each step travel with its Q/dO tiles (bulk
//   copies completing on the same barrier).
// dQ and dK leave through the backward of the rotate-half RoPE (when tables
// are given), then scale, bf16.  No atomics: every output element is written
// once by the CTA that owns its row.  The elementwise arithmetic runs on
// packed f32x2 pairs; NP_DQ (dQ) and NP_DKV (dK/dV) of every 16 pairs of
// exponentials take the polynomial 2^x on the FMA pipe (exp2_poly2), the rest
// the SFU (splits chosen by measurement: dQ fastest at 3, dK/dV at 0, whose
// ALU pipe is the busier).  Every wait is bounded
// (FLAG_TIMEOUT, then drain and free TMEM).
#include "common.cuh"
#include "gemm_tc.h"
#include "attn_tma.cuh"
#include "tcgen05.cuh"

namespace llm {
namespace attn_tc_bwd {

using namespace tc;
using namespace attn_maps;

// 2^x for pair i of a 16-pair chunk: NP of the 16 pairs (spread over the
// chunk) by the polynomial on the FMA pipe, the rest by the SFU.
template <int NP>
LLM_DEV float2 exp2_split(float2 x, int i) {
  return ((i & 15) * NP) % 16 < NP ? exp2_poly2(x) : make_float2(ex2(x.x), ex2(x.y));
}
constexpr int NP_DQ = 3;
constexpr int NP_DKV = 0;

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

// dQ kernel: TMEM columns; shared memory Q[2] | dO[2] | O | K[STAGES] | V[STAGES] |
// barriers | red[2] | -L
constexpr int DQ_COL_S = 0, DQ_COL_DP = 128, DQ_COL_DS = 256, DQ_COL_DQA = 320, DQ_COL_DQB = 384;
constexpr int BAR_BYTES = 512;  // 48 mbarrier slots, then the TMEM address and abort words
constexpr int DQ_SMEM =
    (5 + 2 * STAGES) * TILE_BYTES + 1024 + BAR_BYTES + 2 * NCQ * 128 * 4 + 128 * 4;
// dK/dV kernel: TMEM columns; shared memory K[2] | V[2] | Q[STAGES] | dO[STAGES] |
// L[STAGES] | D[STAGES] | barriers
constexpr int KV_COL_S = 0, KV_COL_DP = 128, KV_COL_P = 256, KV_COL_DS = 320, KV_COL_DV = 384,
              KV_COL_DK = 448;
constexpr int KV_SMEM = (4 + 2 * STAGES) * TILE_BYTES + 2 * STAGES * 128 * 4 + BAR_BYTES + 1024;

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

// N (8) values times mul as bf16 into 16-byte chunk c of a 128-byte row r of a
// tile in the 128-byte-swizzle layout of its tensor map (chunk c at c ^ (r & 7)).
template <int N>
LLM_DEV void stage_n(uint8_t *row, int c, int r, const float (&v)[N], float mul) {
  static_assert(N == 8, "one 16-byte chunk");
  *reinterpret_cast<uint4 *>(row + ((c ^ (r & 7)) << 4)) =
      make_uint4(pack_bf16(v[0] * mul, v[1] * mul), pack_bf16(v[2] * mul, v[3] * mul),
                 pack_bf16(v[4] * mul, v[5] * mul), pack_bf16(v[6] * mul, v[7] * mul));
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

// ------------------------------------------------------------------- dQ
// Persistent: gridDim.x CTAs (one per SM) walk the items (query block, head,
// batch), longest rows first, in the snake of sched_item.  Per item the
// producer loads Q and dO into slot it % 2, O (for D) and -L into single
// buffers, then streams the item's K_j, V_j through the ring.  The ring, the
// S/dP and dS barriers count key blocks over all of a CTA's items (gb), so
// the next item's tiles land and its first products run while this item's
// last blocks and epilogue are still in flight.
__global__ void __launch_bounds__(NTHREADS, 1)
    k_attn_dq_tc(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_do,
                 const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ CUtensorMap tm_st,
                 const float *__restrict__ lse,
                 float *__restrict__ Dv, __nv_bfloat16 *__restrict__ dqkv,
                 const float *__restrict__ cos_t, const float *__restrict__ sin_t, int B, int T,
                 int H, int Hkv, int hd, float scale, int bulk_l, int *gflag) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *sQ = smem, *sdO = smem + 2 * TILE_BYTES, *sO = smem + 4 * TILE_BYTES,
          *sK = smem + 5 * TILE_BYTES, *sV = sK + STAGES * TILE_BYTES;
  uint64_t *bars = (uint64_t *)(sV + STAGES * TILE_BYTES);
  uint32_t *tmem_sh = (uint32_t *)(bars + 48);
  volatile int *abort_sh = (volatile int *)(tmem_sh + 1);
  float *red = (float *)(bars + BAR_BYTES / 8);  // [2][NCQ][128] partial dot products
  float *sNL = red + 2 * NCQ * 128;              // [128] L of the item's rows (rows < T)
  const uint32_t b0 = smem_u32(bars);
  const uint32_t qd_full = b0, qd_empty = b0 + 16,  // [2]: Q/dO slot
                 o_full = b0 + 32, o_empty = b0 + 40, k_full = b0 + 48,
                 k_empty = k_full + 8 * STAGES, v_full = k_empty + 8 * STAGES,
                 v_empty = v_full + 8 * STAGES, s_full = v_empty + 8 * STAGES, s_free = s_full + 8,
                 ds_full = s_free + 8,    // [2]: key half a, b
                 dq_done = ds_full + 16,  // [2]
                 acc_free = dq_done + 16,
                 drain = acc_free + 8,    // [2]: one per MMA warp
                 qsync = drain + 16,      // [4]: per lane quarter, its rows of dQ staged
                 qred = qsync + 32;       // [4]: per lane quarter, its rows' D parts written
  static_assert(6 + 4 * STAGES + 18 <= 48, "barriers overlap the TMEM address word");
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int nqb = (T + BQ - 1) / BQ, n_items = nqb * H * B;
  const int G = gridDim.x, cta = blockIdx.x;
  // item -> (query block, head, batch): longest rows (last query blocks) first,
  // in bands of 4 query blocks taken pair by pair (band_item)
  auto decode = [&](int item, int &qb, int &h, int &b) {
    int z, pr;
    band_item(item, nqb, H * B, z, pr);
    qb = nqb - 1 - z;
    h = pr % H;
    b = pr / H;
  };

  if (threadIdx.x == 0) {
    *abort_sh = 0;
    for (int x = 0; x < 2; x++) {
      mbar_init(qd_full + 8 * x, 1);
      // both products' last MMAs on the slot, every elementwise thread's D,
      // and the bulk stores of dQ staged in the slot's Q tile (one per warp)
      mbar_init(qd_empty + 8 * x, 2 + 32 * EW_WARPS + EW_WARPS);
    }
    mbar_init(o_full, 1 + 32);  // the tile's expect-tx arrival and the 32 lanes writing -L
    mbar_init(o_empty, 32 * EW_WARPS);  // every elementwise thread read its O row and -L
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
    mbar_init(acc_free, EW_WARPS);  // the accumulators of the item were read out
    for (int q = 0; q < 4; q++) {
      mbar_init(qsync + 8 * q, 32 * NCQ);
      mbar_init(qred + 8 * q, 32 * NCQ);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc_512(tmem_sh);
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_sh;

  if (warp == 0) {
    // ---------------------------------------------- TMA producer (warp)
    int gb = 0, nqd = 0, no = 0;  // key blocks, Q/dO tiles and O tiles issued
    bool ok = true;
    for (int r = 0, it = 0; ok; r++, it++) {
      const int item = sched_item(r, G, cta);
      if (item >= n_items) break;
      int qb, h, b;
      decode(item, qb, h, b);
      const int q0 = qb * BQ, row_base = b * T, g = h / (H / Hkv), slot = it & 1;
      // Q, dO into the slot of item it - 2 once it was released
      if (!warp_wait(qd_empty + 8 * slot, ((it >> 1) & 1) ^ 1, abort_sh, gflag)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(qd_full + 8 * slot, 2 * TILE_BYTES);
        tma_load_3d(smem_u32(sQ + slot * TILE_BYTES), &tm_qkv, 0, h, row_base + q0,
                    qd_full + 8 * slot);
        tma_load_3d(smem_u32(sdO + slot * TILE_BYTES), &tm_do, 0, h, row_base + q0,
                    qd_full + 8 * slot);
      }
      nqd = it + 1;
      // O and L once the elementwise warps have formed D of item it - 1; L
      // by a bulk copy when its rows are 16-byte aligned (T % 4 == 0), else
      // by the lanes
      if (!warp_wait(o_empty, (it & 1) ^ 1, abort_sh, gflag)) break;
      const float *lrow = lse + ((int64_t)b * H + h) * T + q0;
      const int nvalid = min(BQ, T - q0);
      if (lane == 0) {
        mbar_arrive_expect_tx(o_full, TILE_BYTES + (bulk_l ? nvalid * 4 : 0));
        tma_load_3d(smem_u32(sO), &tm_o, 0, h, row_base + q0, o_full);
        if (bulk_l) bulk_load(smem_u32(sNL), lrow, nvalid * 4, o_full);
      }
      if (!bulk_l)
        for (int i = lane; i < nvalid; i += 32) sNL[i] = lrow[i];
      mbar_arrive(o_full);
      no = it + 1;
      for (int j = 0; j <= qb; j++) {
        const int s = gb % STAGES;
        const uint32_t ph = (gb / STAGES) & 1;
        if (!warp_wait(k_empty + 8 * s, ph ^ 1, abort_sh, gflag) ||
            !warp_wait(v_empty + 8 * s, ph ^ 1, abort_sh, gflag)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(k_full + 8 * s, TILE_BYTES);
          tma_load_3d(smem_u32(sK + s * TILE_BYTES), &tm_qkv, 0, H + g, row_base + j * BK,
                      k_full + 8 * s);
          mbar_arrive_expect_tx(v_full + 8 * s, TILE_BYTES);
          tma_load_3d(smem_u32(sV + s * TILE_BYTES), &tm_qkv, 0, H + Hkv + g,
                      row_base + j * BK, v_full + 8 * s);
        }
        gb++;
      }
    }
    // every copy this warp issued has landed before the CTA may exit
    if (lane == 0) {
      for (int i = max(0, nqd - 2); i < nqd; i++) drain_wait(qd_full + 8 * (i & 1), (i >> 1) & 1);
      if (no > 0) drain_wait(o_full, (no - 1) & 1);
      for (int i = max(0, gb - STAGES); i < gb; i++) {
        drain_wait(k_full + 8 * (i % STAGES), (i / STAGES) & 1);
        drain_wait(v_full + 8 * (i % STAGES), (i / STAGES) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == MMA_B_WARP) {
    // ------------------------------------- MMA issuers (whole warps)
    // A: S = Q K_j^T, dQ_a += dS_a K_j[0:64];  B: dP = dO V_j^T, dQ_b += dS_b K_j[64:128]
    const int x = warp == 1 ? 0 : 1;
    constexpr uint32_t ID_S = idesc_mn(128, BK, false, false);
    constexpr uint32_t ID_DQ = idesc_mn(128, HD, false, true);
    uint8_t *sA = x ? sdO : sQ;
    uint8_t *sB = x ? sV : sK;
    const uint32_t b_full = x ? v_full : k_full;
    const uint32_t col = x ? DQ_COL_DP : DQ_COL_S;
    auto issue_prod = [&](int slot, int s) {
      const uint64_t ad = sdesc(smem_u32(sA + slot * TILE_BYTES), 16, 1024);
      const uint64_t bd = sdesc(smem_u32(sB + s * TILE_BYTES), 16, 1024);
#pragma unroll
      for (int kk = 0; kk < HD / 16; kk++)
        mma_bf16_e(tmem + col, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), ID_S,
                   kk > 0 ? 1u : 0u);
      mma_commit_e(s_full);
      if (x) mma_commit_e(v_empty + 8 * s);  // V_j is not read again
    };
    bool ok = true;
    int gb = 0;
    int item = sched_item(0, G, cta);
    if (item < n_items) {  // products of the first block
      int qb, h, b;
      decode(item, qb, h, b);
      ok = warp_wait(qd_full, 0, abort_sh, gflag) && warp_wait(b_full, 0, abort_sh, gflag);
      if (ok) {
        fence_after();
        issue_prod(0, 0);
        if (qb == 0) mma_commit_e(qd_empty);  // the item's last products on slot 0
      }
    }
    for (int r = 0, it = 0; item < n_items && ok; r++, it++) {
      int qb, h, b;
      decode(item, qb, h, b);
      const int nj = qb + 1, slot = it & 1;
      const int next = sched_item(r + 1, G, cta);
      int qb_next = 0, hn, bn;
      if (next < n_items) decode(next, qb_next, hn, bn);
      for (int j = 0; j < nj && ok; j++, gb++) {
        const int s = gb % STAGES;
        const uint32_t ph = (gb / STAGES) & 1;
        // products of block gb + 1 (this item's next, or the next item's first)
        // once the elementwise warps have read S and dP of block gb
        const bool here = j + 1 < nj;
        if (here || next < n_items) {
          const int slot1 = here ? slot : slot ^ 1;
          const int s1 = (gb + 1) % STAGES;
          const uint32_t ph1 = ((gb + 1) / STAGES) & 1;
          if ((!here && !warp_wait(qd_full + 8 * slot1, ((it + 1) >> 1) & 1, abort_sh, gflag)) ||
              !warp_wait(b_full + 8 * s1, ph1, abort_sh, gflag) ||
              !warp_wait(s_free, gb & 1, abort_sh, gflag)) {
            ok = false;
            break;
          }
          fence_after();
          issue_prod(slot1, s1);
          // the last products that read this Q/dO slot
          if (here ? (j + 1 == nj - 1) : (qb_next == 0)) mma_commit_e(qd_empty + 8 * slot1);
        }
        // dQ_x += dS_x K_j[x half]; the accumulators of the previous item were read out
        if ((j == 0 && it > 0 && !warp_wait(acc_free, (it - 1) & 1, abort_sh, gflag)) ||
            !warp_wait(ds_full + 8 * x, gb & 1, abort_sh, gflag) ||
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
      item = next;
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
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float sl2 = scale * LOG2E;
    bool ok = true;
    int gb = 0, st_slot = -1;  // slot whose dQ store is still to be released
    for (int rr = 0, it = 0; ok; rr++, it++) {
      const int item = sched_item(rr, G, cta);
      if (item >= n_items) break;
      int qb, h, b;
      decode(item, qb, h, b);
      const int q0 = qb * BQ, nj = qb + 1, slot = it & 1;
      const int qi = q0 + r;
      const bool valid = qi < T;
      if (!warp_wait(o_full, it & 1, abort_sh, gflag) ||
          !warp_wait(qd_full + 8 * slot, (it >> 1) & 1, abort_sh, gflag)) {
        ok = false;
        break;
      }
      // D_i = dO_i . O_i over this thread's 64 / NCQ head columns, from the
      // tiles in shared memory (128-byte swizzle: 16-byte chunk c of row r at
      // position c ^ (r & 7))
      float dpart = 0.f;
      {
        const uint8_t *ro = sO + r * 128, *rdo = sdO + slot * TILE_BYTES + r * 128;
#pragma unroll
        for (int e = 0; e < HD / NCQ / 8; e++) {
          const int c = ((cq * (HD / NCQ / 8) + e) ^ (r & 7)) << 4;
          const uint4 a = *reinterpret_cast<const uint4 *>(ro + c);
          const uint4 cc = *reinterpret_cast<const uint4 *>(rdo + c);
          const __nv_bfloat162 *ha = reinterpret_cast<const __nv_bfloat162 *>(&a);
          const __nv_bfloat162 *hc = reinterpret_cast<const __nv_bfloat162 *>(&cc);
#pragma unroll
          for (int k = 0; k < 4; k++) {
            const float2 fa = __bfloat1622float2(ha[k]), fc = __bfloat1622float2(hc[k]);
            dpart += fa.x * fc.x + fa.y * fc.y;
          }
        }
      }
      // rows past T get -L = -inf, so every P of theirs is 0
      const float nl2 = valid ? -sNL[r] * LOG2E : -INFINITY;
      mbar_arrive(o_empty);              // this thread's O row and -L consumed
      mbar_arrive(qd_empty + 8 * slot);  // and its dO row
      float *rd = red + (it & 1) * NCQ * 128;
      rd[cq * 128 + r] = dpart;
      // the row's four column groups are the four warps of this lane quarter
      mbar_arrive(qred + 8 * quarter);
      if (!warp_wait(qred + 8 * quarter, it & 1, abort_sh, gflag)) {
        ok = false;
        break;
      }
      float Di = 0.f;
#pragma unroll
      for (int c = 0; c < NCQ; c++) Di += rd[c * 128 + r];
      // the previous item's dQ store has long read its tile: release the slot
      if (st_slot >= 0) {
        if (lane == 0) {
          bulk_wait_read();
          mbar_arrive(qd_empty + 8 * st_slot);
        }
        st_slot = -1;
      }
      if (cq == 0 && valid) Dv[((int64_t)b * H + h) * T + qi] = Di;
      const float2 nl = make_float2(nl2, nl2), nd = make_float2(-Di, -Di);
      for (int j = 0; j < nj && ok; j++, gb++) {
        if (!warp_wait(s_full, gb & 1, abort_sh, gflag)) {
          ok = false;
          break;
        }
        fence_after();
        float sv[CW], dv[CW];
        tmem_ld_pair<CW>(tmem + lane_off + DQ_COL_S + cq * CW, tmem + lane_off + DQ_COL_DP + cq * CW,
                         sv, dv);
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);  // the MMA warps may overwrite S and dP now
        const int k0 = j * BK + cq * CW;
        const bool diag = (j == qb);  // only the diagonal block masks (keys >= T lie above it)
        uint32_t w[CW / 2];
        if (diag) {  // the causal mask only on the diagonal block
#pragma unroll
          for (int i = 0; i < CW; i += 2) {
            float2 p = exp2_split<NP_DQ>(
                __ffma2_rn(make_float2(sv[i], sv[i + 1]), make_float2(sl2, sl2), nl), i / 2);
            if (k0 + i > qi) p.x = 0.f;
            if (k0 + i + 1 > qi) p.y = 0.f;
            const float2 ds = __fmul2_rn(p, __fadd2_rn(make_float2(dv[i], dv[i + 1]), nd));
            w[i / 2] = pack_bf16(ds.x, ds.y);
          }
        } else {
#pragma unroll
          for (int i = 0; i < CW; i += 2) {
            const float2 p = exp2_split<NP_DQ>(
                __ffma2_rn(make_float2(sv[i], sv[i + 1]), make_float2(sl2, sl2), nl), i / 2);
            const float2 ds = __fmul2_rn(p, __fadd2_rn(make_float2(dv[i], dv[i + 1]), nd));
            w[i / 2] = pack_bf16(ds.x, ds.y);
          }
        }
        // this half's dS of the previous block is free once its dQ product
        // completed (at an item's first block the epilogue already waited)
        if (j > 0) {
          if (!warp_wait(dq_done + 8 * x, (gb - 1) & 1, abort_sh, gflag)) {
            ok = false;
            break;
          }
          fence_after();
        }
#pragma unroll
        for (int c = 0; c < CW / 2; c += 16)
          tmem_stn<(CW / 2 < 16 ? CW / 2 : 16)>(tmem + lane_off + DQ_COL_DS + cq * (CW / 2) + c,
                                               w + c);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_full + 8 * x);
      }
      if (!ok) break;
      if (!warp_wait(dq_done, (gb - 1) & 1, abort_sh, gflag) ||
          !warp_wait(dq_done + 8, (gb - 1) & 1, abort_sh, gflag)) {
        ok = false;
        break;
      }
      fence_after();
      // column pairs (c, c + hd/2) of RoPE: this group takes c in [xc, xc + HW)
      // (head 32: groups 2 and 3 repeat 0 and 1 and stage nothing)
      const int half = hd / 2, xc = (hd == 64 ? cq : (cq & 1)) * HW;
      float xa[HW], ya[HW], xb[HW], yb[HW];
      {  // the four loads in flight together, one wait
        uint32_t ra[HW], rya[HW], rb[HW], ryb[HW];
        tmem_ld_raw<HW>(tmem + lane_off + DQ_COL_DQA + xc, ra);
        tmem_ld_raw<HW>(tmem + lane_off + DQ_COL_DQA + half + xc, rya);
        tmem_ld_raw<HW>(tmem + lane_off + DQ_COL_DQB + xc, rb);
        tmem_ld_raw<HW>(tmem + lane_off + DQ_COL_DQB + half + xc, ryb);
        tmem_wait_ld();
        tmem_after_wait(ra);
        tmem_after_wait(rya);
        tmem_after_wait(rb);
        tmem_after_wait(ryb);
#pragma unroll
        for (int i = 0; i < HW; i++) {
          xa[i] = __uint_as_float(ra[i]);
          ya[i] = __uint_as_float(rya[i]);
          xb[i] = __uint_as_float(rb[i]);
          yb[i] = __uint_as_float(ryb[i]);
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_free);  // the next item's dQ products may start
#pragma unroll
      for (int i = 0; i < HW; i++) {
        xa[i] += xb[i];
        ya[i] += yb[i];
      }
      if (valid && cos_t)
        rope_bwd_n<HW>(xa, ya, cos_t + (int64_t)qi * half + xc, sin_t + (int64_t)qi * half + xc);
      // dQ rows through the item's Q tile (its products are complete): the
      // 128-byte-swizzle image of the tile, then each warp stores 8 whole rows
      // of its lane quarter with one bulk tensor copy (rows past T clipped)
      uint8_t *srow = sQ + slot * TILE_BYTES + r * 128;
      if (hd == 64 || cq < 2) {
        stage_n<HW>(srow, xc / 8, r, xa, scale);
        stage_n<HW>(srow, (half + xc) / 8, r, ya, scale);
      }
      fence_proxy_async();
      mbar_arrive(qsync + 8 * quarter);
      if (!warp_wait(qsync + 8 * quarter, it & 1, abort_sh, gflag)) {
        ok = false;
        break;
      }
      if (lane == 0) {
        const int r0 = quarter * 32 + cq * 8;
        tma_store_4d(&tm_st, smem_u32(sQ + slot * TILE_BYTES + r0 * 128), 0, h, q0 + r0, b);
        bulk_commit();
      }
      st_slot = slot;  // released (below) once the store has read the tile
    }
    if (lane == 0) bulk_wait_all();
  }
  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) tmem_free_512(tmem);
}

// ---------------------------------------------------------------- dK, dV
// Persistent like the dQ kernel: items (key block, kv head, batch), first key
// blocks (the most query blocks) first; K and V of item it in slot it % 2,
// the (query head, query block) steps of all of a CTA's items through one
// ring (global step gs), so the next item's first products start while this
// item's last accumulations and epilogue run.
__global__ void __launch_bounds__(NTHREADS, 1)
    k_attn_dkv_tc(const __grid_constant__ CUtensorMap tm_qkv,
                  const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_st,
                  const float *__restrict__ lse,
                  const float *__restrict__ Dv, __nv_bfloat16 *__restrict__ dqkv,
                  const float *__restrict__ cos_t, const float *__restrict__ sin_t, int B, int T,
                  int H, int Hkv, int hd, float scale, int bulk_l, int *gflag) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *sK = smem, *sV = smem + 2 * TILE_BYTES, *sQ = smem + 4 * TILE_BYTES,
          *sdO = sQ + STAGES * TILE_BYTES;
  float *sL = (float *)(sdO + STAGES * TILE_BYTES);  // [STAGES][128] L (+inf past T)
  float *sD = sL + STAGES * 128;                      // [STAGES][128] D (0 past T)
  uint64_t *bars = (uint64_t *)(sD + STAGES * 128);
  uint32_t *tmem_sh = (uint32_t *)(bars + 48);
  volatile int *abort_sh = (volatile int *)(tmem_sh + 1);
  const uint32_t b0 = smem_u32(bars);
  const uint32_t kv_full = b0, kv_empty = b0 + 16,  // [2]: K/V slot
                 q_full = b0 + 32, q_empty = q_full + 8 * STAGES,
                 ld_full = q_empty + 8 * STAGES, s_full = ld_full + 8 * STAGES,
                 s_free = s_full + 8, p_full = s_free + 8, pv_done = p_full + 8,
                 drain = pv_done + 8,  // drain [2]: one per MMA warp
                 qsync = drain + 16;   // [4]: per lane quarter, its rows of dK, dV staged
  static_assert(4 + 3 * STAGES + 10 <= 48, "barriers overlap the TMEM address word");
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int nkb = (T + BK - 1) / BK, n_items = nkb * Hkv * B;
  const int G = gridDim.x, cta = blockIdx.x;
  const int grp = H / Hkv;
  // item -> (key block, kv head, batch), first key blocks first in bands of 4
  // taken pair by pair (band_item); steps = grp (nkb - kb)
  auto decode = [&](int item, int &kb, int &g, int &b) {
    int pr;
    band_item(item, nkb, Hkv * B, kb, pr);
    g = pr % Hkv;
    b = pr / Hkv;
  };

  if (threadIdx.x == 0) {
    *abort_sh = 0;
    for (int x = 0; x < 2; x++) {
      mbar_init(kv_full + 8 * x, 1);
      // both MMA warps' last products on the slot, and the bulk stores of dK
      // and dV staged in the slot (one per elementwise warp)
      mbar_init(kv_empty + 8 * x, 2 + EW_WARPS);
    }
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
    for (int q = 0; q < 4; q++) mbar_init(qsync + 8 * q, 32 * NCQ);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc_512(tmem_sh);
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_sh;

  if (warp == 0) {
    // ---------------------------------------------- TMA producer (warp)
    int gs = 0, nkv = 0;  // steps and K/V tiles issued
    bool ok = true;
    for (int r = 0, it = 0; ok; r++, it++) {
      const int item = sched_item(r, G, cta);
      if (item >= n_items) break;
      int kb, g, b;
      decode(item, kb, g, b);
      const int k0 = kb * BK, row_base = b * T, nq = nkb - kb, slot = it & 1;
      if (!warp_wait(kv_empty + 8 * slot, ((it >> 1) & 1) ^ 1, abort_sh, gflag)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(kv_full + 8 * slot, 2 * TILE_BYTES);
        tma_load_3d(smem_u32(sK + slot * TILE_BYTES), &tm_qkv, 0, H + g, row_base + k0,
                    kv_full + 8 * slot);
        tma_load_3d(smem_u32(sV + slot * TILE_BYTES), &tm_qkv, 0, H + Hkv + g, row_base + k0,
                    kv_full + 8 * slot);
      }
      nkv = it + 1;
      for (int st = 0; st < grp * nq; st++) {
        const int s = gs % STAGES;
        const uint32_t ph = (gs / STAGES) & 1;
        const int hq = g * grp + st / nq, qb = kb + st % nq;
        // the slot (tiles and L, D) of step gs - STAGES is free once its products completed
        if (!warp_wait(q_empty + 8 * s, ph ^ 1, abort_sh, gflag)) {
          ok = false;
          break;
        }
        // the step's L and D rows by bulk copies when 16-byte aligned (T % 4
        // == 0), else by the lanes; queries past T get L = +inf, so their P is
        // 0 (below 2^-125 where the polynomial exponential takes the pair), and D = 0
        const int64_t base = ((int64_t)b * H + hq) * T + qb * BQ;
        const int nvalid = min(BQ, T - qb * BQ);
        if (lane == 0) {
          mbar_arrive_expect_tx(q_full + 8 * s, 2 * TILE_BYTES + (bulk_l ? 8 * nvalid : 0));
          tma_load_3d(smem_u32(sQ + s * TILE_BYTES), &tm_qkv, 0, hq, row_base + qb * BQ,
                      q_full + 8 * s);
          tma_load_3d(smem_u32(sdO + s * TILE_BYTES), &tm_do, 0, hq, row_base + qb * BQ,
                      q_full + 8 * s);
          if (bulk_l) {
            bulk_load(smem_u32(sL + s * 128), lse + base, nvalid * 4, q_full + 8 * s);
            bulk_load(smem_u32(sD + s * 128), Dv + base, nvalid * 4, q_full + 8 * s);
          }
        }
#pragma unroll
        for (int i = lane; i < BQ; i += 32) {
          if (i >= nvalid) {
            sL[s * 128 + i] = INFINITY;
            sD[s * 128 + i] = 0.f;
          } else if (!bulk_l) {
            sL[s * 128 + i] = lse[base + i];
            sD[s * 128 + i] = Dv[base + i];
          }
        }
        mbar_arrive(ld_full + 8 * s);
        gs++;
      }
    }
    if (lane == 0) {
      for (int i = max(0, nkv - 2); i < nkv; i++) drain_wait(kv_full + 8 * (i & 1), (i >> 1) & 1);
      for (int i = max(0, gs - STAGES); i < gs; i++)
        drain_wait(q_full + 8 * (i % STAGES), (i / STAGES) & 1);
    }
    __syncwarp();
  } else if (warp == 1 || warp == MMA_B_WARP) {
    // ------------------------------------- MMA issuers (whole warps)
    // A: S^T = K Q^T, dV += P^T dO;  B: dP^T = V dO^T, dK += dS^T Q
    const int x = warp == 1 ? 0 : 1;
    constexpr uint32_t ID_S = idesc_mn(128, BQ, false, false);
    constexpr uint32_t ID_KV = idesc_mn(128, HD, false, true);
    uint8_t *sA = x ? sV : sK;     // A of the scores product, slot by item
    uint8_t *sB = x ? sdO : sQ;    // B of the scores product (K-major)
    uint8_t *sB2 = x ? sQ : sdO;   // B of the accumulation (MN-major)
    const uint32_t col = x ? KV_COL_DP : KV_COL_S;
    const uint32_t col_a2 = x ? KV_COL_DS : KV_COL_P, col_acc = x ? KV_COL_DK : KV_COL_DV;
    auto issue_prod = [&](int slot, int s) {
      const uint64_t ad = sdesc(smem_u32(sA + slot * TILE_BYTES), 16, 1024);
      const uint64_t bd = sdesc(smem_u32(sB + s * TILE_BYTES), 16, 1024);
#pragma unroll
      for (int kk = 0; kk < HD / 16; kk++)
        mma_bf16_e(tmem + col, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), ID_S,
                   kk > 0 ? 1u : 0u);
      mma_commit_e(s_full);
    };
    bool ok = true;
    int gs = 0;
    int item = sched_item(0, G, cta);
    if (item < n_items) {  // products of the first step
      int kb, g, b;
      decode(item, kb, g, b);
      ok = warp_wait(kv_full, 0, abort_sh, gflag) && warp_wait(q_full, 0, abort_sh, gflag);
      if (ok) {
        fence_after();
        issue_prod(0, 0);
        if (grp * (nkb - kb) == 1) mma_commit_e(kv_empty);  // the item's last products on slot 0
      }
    }
    for (int r = 0, it = 0; item < n_items && ok; r++, it++) {
      int kb, g, b;
      decode(item, kb, g, b);
      const int nsteps = grp * (nkb - kb), slot = it & 1;
      const int next = sched_item(r + 1, G, cta);
      int kb_next = nkb - 1, gn, bn;
      if (next < n_items) decode(next, kb_next, gn, bn);
      const int nsteps_next = grp * (nkb - kb_next);
      for (int st = 0; st < nsteps && ok; st++, gs++) {
        const int s = gs % STAGES;
        // products of step gs + 1 (this item's next, or the next item's first)
        // once the elementwise warps have read S^T and dP^T of step gs
        const bool here = st + 1 < nsteps;
        if (here || next < n_items) {
          const int slot1 = here ? slot : slot ^ 1;
          const int s1 = (gs + 1) % STAGES;
          const uint32_t ph1 = ((gs + 1) / STAGES) & 1;
          if ((!here && !warp_wait(kv_full + 8 * slot1, ((it + 1) >> 1) & 1, abort_sh, gflag)) ||
              !warp_wait(q_full + 8 * s1, ph1, abort_sh, gflag) ||
              !warp_wait(s_free, gs & 1, abort_sh, gflag)) {
            ok = false;
            break;
          }
          fence_after();
          issue_prod(slot1, s1);
          // the last products that read this K/V slot
          if (here ? (st + 1 == nsteps - 1) : (nsteps_next == 1)) mma_commit_e(kv_empty + 8 * slot1);
        }
        if (!warp_wait(p_full, gs & 1, abort_sh, gflag)) {
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
      item = next;
    }
    mma_commit_e(drain + 8 * x);
    if (lane == 0) drain_wait(drain + 8 * x, 0);
    __syncwarp();
  } else {
    // --------------------------------------------------------- elementwise
    const int quarter = warp & 3;
    const int cq = (warp - 2) >> 2;  // column group: queries [cq CW, cq CW + CW) of the block
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float sl2 = scale * LOG2E;
    bool ok = true;
    int gs = 0, st_slot = -1;  // slot whose dK/dV stores are still to be released
    for (int rr = 0, it = 0; ok; rr++, it++) {
      const int item = sched_item(rr, G, cta);
      if (item >= n_items) break;
      int kb, g, b;
      decode(item, kb, g, b);
      const int k0 = kb * BK, kj = k0 + r, nq = nkb - kb, slot = it & 1;
      const int nsteps = grp * nq;
      // the accumulators of the previous item were read out before this
      // warp's first P^T / dS^T arrival below (program order), so the
      // item's first accumulations (accumulate = 0) cannot overwrite them early
      for (int st = 0; st < nsteps && ok; st++, gs++) {
        const int s = gs % STAGES;
        const int qb = kb + st % nq;
        if (!warp_wait(s_full, gs & 1, abort_sh, gflag) ||
            !warp_wait(q_full + 8 * s, (gs / STAGES) & 1, abort_sh, gflag) ||
            !warp_wait(ld_full + 8 * s, (gs / STAGES) & 1, abort_sh, gflag)) {
          ok = false;
          break;
        }
        fence_after();
        const int qc0 = qb * BQ + cq * CW;
        const bool diag = (qb == kb);  // keys >= T occur only in this case, above the diagonal
        const float4 *L4 = reinterpret_cast<const float4 *>(sL + s * 128 + cq * CW);
        const float4 *D4 = reinterpret_cast<const float4 *>(sD + s * 128 + cq * CW);
        // two halves of the thread's CW queries, each read from TMEM, packed
        // and stored before the next (fewer live registers); S^T and dP^T are
        // released once the second half is read; P^T and dS^T of the previous
        // step are free once its products completed (at an item's first step
        // the epilogue already waited)
#pragma unroll
        for (int hf = 0; hf < 2; hf++) {
          constexpr int HC = CW / 2;
          float sv[HC], dv[HC];
          tmem_ld_pair<HC>(tmem + lane_off + KV_COL_S + cq * CW + hf * HC,
                           tmem + lane_off + KV_COL_DP + cq * CW + hf * HC, sv, dv);
          if (hf == 1) {
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_free);
          }
          uint32_t wp[HC / 2], wd[HC / 2];
#pragma unroll
          for (int i = 0; i < HC; i += 4) {
            const int c = hf * HC + i;  // query column within the thread's CW
            const float4 lq = L4[c / 4], dq = D4[c / 4];  // L and D of 4 queries
            const float2 nl01 = __fmul2_rn(make_float2(lq.x, lq.y), make_float2(-LOG2E, -LOG2E));
            const float2 nl23 = __fmul2_rn(make_float2(lq.z, lq.w), make_float2(-LOG2E, -LOG2E));
            const float2 x01 = __ffma2_rn(make_float2(sv[i], sv[i + 1]), make_float2(sl2, sl2),
                                          nl01);
            const float2 x23 = __ffma2_rn(make_float2(sv[i + 2], sv[i + 3]),
                                          make_float2(sl2, sl2), nl23);
            float2 p01 = exp2_split<NP_DKV>(x01, c / 2), p23 = exp2_split<NP_DKV>(x23, c / 2 + 1);
            if (diag) {
              if (kj > qc0 + c) p01.x = 0.f;
              if (kj > qc0 + c + 1) p01.y = 0.f;
              if (kj > qc0 + c + 2) p23.x = 0.f;
              if (kj > qc0 + c + 3) p23.y = 0.f;
            }
            wp[i / 2] = pack_bf16(p01.x, p01.y);
            wp[i / 2 + 1] = pack_bf16(p23.x, p23.y);
            const float2 d01 = __fmul2_rn(p01, __ffma2_rn(make_float2(dq.x, dq.y), make_float2(-1.f, -1.f),
                                                          make_float2(dv[i], dv[i + 1])));
            const float2 d23 = __fmul2_rn(p23, __ffma2_rn(make_float2(dq.z, dq.w), make_float2(-1.f, -1.f),
                                                          make_float2(dv[i + 2], dv[i + 3])));
            wd[i / 2] = pack_bf16(d01.x, d01.y);
            wd[i / 2 + 1] = pack_bf16(d23.x, d23.y);
          }
          if (hf == 0 && st > 0) {
            if (!warp_wait(pv_done, (gs - 1) & 1, abort_sh, gflag)) {
              ok = false;
              break;
            }
            fence_after();
          }
          tmem_stn<HC / 2>(tmem + lane_off + KV_COL_P + cq * (CW / 2) + hf * (HC / 2), wp);
          tmem_stn<HC / 2>(tmem + lane_off + KV_COL_DS + cq * (CW / 2) + hf * (HC / 2), wd);
        }
        if (!ok) break;
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        // the previous item's dK/dV stores have long read their tiles
        if (st_slot >= 0) {
          if (lane == 0) {
            bulk_wait_read();
            mbar_arrive(kv_empty + 8 * st_slot);
          }
          st_slot = -1;
        }
      }
      if (!ok) break;
      if (!warp_wait(pv_done, (gs - 1) & 1, abort_sh, gflag)) {
        ok = false;
        break;
      }
      fence_after();
      // column pairs (c, c + hd/2) of RoPE in dK: this group takes c in
      // [xc, xc + HW) (head 32: groups 2 and 3 repeat 0 and 1 and stage no dK);
      // dV: columns [cq HW, cq HW + HW) and 32 more (zero past head 32)
      const int half = hd / 2, xc = (hd == 64 ? cq : (cq & 1)) * HW;
      float xk[HW], yk[HW], xv[HW], yv[HW];
      {  // the four loads in flight together, one wait
        uint32_t rk[HW], ryk[HW], rv[HW], ryv[HW];
        tmem_ld_raw<HW>(tmem + lane_off + KV_COL_DK + xc, rk);
        tmem_ld_raw<HW>(tmem + lane_off + KV_COL_DK + half + xc, ryk);
        tmem_ld_raw<HW>(tmem + lane_off + KV_COL_DV + cq * HW, rv);
        tmem_ld_raw<HW>(tmem + lane_off + KV_COL_DV + 32 + cq * HW, ryv);
        tmem_wait_ld();
        tmem_after_wait(rk);
        tmem_after_wait(ryk);
        tmem_after_wait(rv);
        tmem_after_wait(ryv);
#pragma unroll
        for (int i = 0; i < HW; i++) {
          xk[i] = __uint_as_float(rk[i]);
          yk[i] = __uint_as_float(ryk[i]);
          xv[i] = __uint_as_float(rv[i]);
          yv[i] = __uint_as_float(ryv[i]);
        }
      }
      if (kj < T && cos_t)
        rope_bwd_n<HW>(xk, yk, cos_t + (int64_t)kj * half + xc, sin_t + (int64_t)kj * half + xc);
      // dK, dV rows through the item's K and V tiles (their products are
      // complete), then each warp stores 8 whole rows of its lane quarter of
      // both with bulk tensor copies (rows past T clipped)
      uint8_t *rk = sK + slot * TILE_BYTES + r * 128, *rv = sV + slot * TILE_BYTES + r * 128;
      if (hd == 64 || cq < 2) {
        stage_n<HW>(rk, xc / 8, r, xk, scale);
        stage_n<HW>(rk, (half + xc) / 8, r, yk, scale);
      }
      stage_n<HW>(rv, cq, r, xv, 1.f);
      stage_n<HW>(rv, 4 + cq, r, yv, 1.f);
      fence_proxy_async();
      mbar_arrive(qsync + 8 * quarter);
      if (!warp_wait(qsync + 8 * quarter, it & 1, abort_sh, gflag)) {
        ok = false;
        break;
      }
      if (lane == 0) {
        const int r0 = quarter * 32 + cq * 8;
        tma_store_4d(&tm_st, smem_u32(sK + slot * TILE_BYTES + r0 * 128), 0, H + g, k0 + r0, b);
        tma_store_4d(&tm_st, smem_u32(sV + slot * TILE_BYTES + r0 * 128), 0, H + Hkv + g, k0 + r0,
                     b);
        bulk_commit();
      }
      st_slot = slot;  // released after the next item's first step
    }
    if (lane == 0) bulk_wait_all();
  }
  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) tmem_free_512(tmem);
}

}  // namespace attn_tc_bwd


// Host side: head-indexed tensor maps (attn_tma.cuh) over qkv [B*T][H + 2 Hkv
// heads][hd], O and dout [B*T][H][hd] (box 64 x 1 x 128), and dqkv for the
// stores ([B][T][H + 2 Hkv][hd], box 64 x 1 x 8 x 1); the dQ kernel runs
// first (it also writes D), then the dK/dV kernel.
bool attn_bwd_tc(const void *qkv, const void *o, const void *dout, const float *lse, float *Dbuf,
                 void *dqkv, int B, int T, int H, int Hkv, int hd, const float *cos_t,
                 const float *sin_t, int *flag, cudaStream_t s) {
  using namespace attn_tc_bwd;
  if ((hd != 64 && hd != 32) || !flag || ((uintptr_t)o & 15) || ((uintptr_t)dqkv & 15) ||
      ((uintptr_t)cos_t & 15) || ((uintptr_t)sin_t & 15) || (!cos_t != !sin_t))
    return false;
  if (!smem_optin((const void *)k_attn_dq_tc, DQ_SMEM) ||
      !smem_optin((const void *)k_attn_dkv_tc, KV_SMEM))
    return false;
  const int64_t qkvw = (int64_t)(H + 2 * Hkv) * hd, dw = (int64_t)H * hd;
  CUtensorMap mq, md, mo, mst;
  if (!head_map_load(&mq, qkv, hd, H + 2 * Hkv, (int64_t)B * T, qkvw, 128) ||
      !head_map_load(&md, dout, hd, H, (int64_t)B * T, dw, 128) ||
      !head_map_load(&mo, o, hd, H, (int64_t)B * T, dw, 128) ||
      !head_map_store(&mst, dqkv, hd, H + 2 * Hkv, T, B, qkvw, 8))
    return false;
  const int nb = (T + BQ - 1) / BQ, sms = device_sms();
  const float scale = 1.0f / sqrtf((float)hd);
  // L and D rows of a (batch, head) start 16-byte aligned when T % 4 == 0
  const int bulk_l = (T % 4 == 0) && !((uintptr_t)lse & 15) && !((uintptr_t)Dbuf & 15);
  k_attn_dq_tc<<<min(nb * H * B, sms), NTHREADS, DQ_SMEM, s>>>(
      mq, md, mo, mst, lse, Dbuf, (__nv_bfloat16 *)dqkv, cos_t, sin_t, B, T, H, Hkv, hd, scale,
      bulk_l, flag);
  k_attn_dkv_tc<<<min(nb * Hkv * B, sms), NTHREADS, KV_SMEM, s>>>(
      mq, md, mst, lse, Dbuf, (__nv_bfloat16 *)dqkv, cos_t, sin_t, B, T, H, Hkv, hd, scale,
      bulk_l, flag);
  count_launch(2);
  return true;
}

}  // namespace llm
