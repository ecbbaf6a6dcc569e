// tcgen05 flash-attention forward for head sizes 64 and 32 (bf16 operands,
// fp32 softmax and accumulators): strata's online-softmax attention (no T x T
// scores in memory, only the row log-sum-exp saved) on the 5th-generation
// tensor cores.  A head-32 tile is loaded as the head-64 one with its upper
// 32 columns zero (the tensor maps of attn_tma.cuh), so the same products
// give the head-32 scores and an O whose upper half is zero and not stored.
//
// One CTA = 128 queries of one (batch, head); key blocks of 128, split into
// NQ key groups of KW = 128 / NQ keys.  Warps:
//   warp 0          TMA producer: the Q tile once, K and V tiles into
//                   STAGES-deep rings;
//   warp 1          TMEM allocation and MMA issuer A:
//                     S_j  = Q K_j^T     (M 128, N 128, K 64; both operands
//                                         K-major in shared memory) into TMEM
//                                         buffer j % 2
//                     O_g += P_g V_g     for key groups g < NQ/2 (M 128, N 64,
//                                         K KW; A = P_g from TMEM, B = the V
//                                         rows of group g, MN-major) -> TMEM O_g
//   last warp       MMA issuer B: O_g += P_g V_g for groups g >= NQ/2;
//   4 NQ warps      softmax, NQ per TMEM lane quarter: thread = one query row
//                   (TMEM lane) and one key group.
// S is double-buffered in TMEM and each group's P of a block is written back,
// packed bf16, over the first KW/2 of that group's own S columns once read:
// S_{j+1} is computed into the other buffer as soon as the P V products of
// block j - 1 (which read that buffer) have completed, so a softmax thread
// finishing block j finds S_{j+1} ready and never waits for the slowest
// thread to release its S; it waits for the P V products only before a rare
// rescale of its accumulator.  The key groups are NQ independent online
// softmaxes (split-K inside the CTA): each (row, group) thread keeps its own
// running maximum m_g, sum l_g and accumulator O_g; the groups meet once at
// the end, O = sum_g 2^(m_g-m) O_g / sum_g 2^(m_g-m) l_g with m = max_g m_g.
// The running maximum is lazy: the reference of a (row, group) moves only when
// a block's maximum exceeds it by more than 2^8, so P stays below 256 and O_g
// is rescaled only then.  The maximum is taken on the raw scores (the log2
// scale is positive) and only the diagonal block runs the causal mask, so an
// off-diagonal block costs half a three-input maximum, half a packed f32x2
// multiply-add and one exponential per score; NP_FWD of every 16 pairs of
// exponentials run as a polynomial on the FMA pipe (exp2_poly2), the rest on
// the SFU (16 results per clock and SM); the split was chosen by measurement
// (0 to 6 of 16 within 5% of each other, 3 the fastest).  MMAs are issued by whole converged warps (one elected lane).  Every wait is bounded (FLAG_TIMEOUT, then drain and free
// TMEM).
#include "common.cuh"
#include "gemm_tc.h"
#include "attn_tma.cuh"
#include "tcgen05.cuh"

namespace llm {
namespace attn_tc {

using namespace tc;
using namespace attn_maps;

// 2^x for pair i of a 16-pair chunk: NP of the 16 pairs (spread over the
// chunk) by the polynomial on the FMA pipe, the rest by the SFU.
template <int NP>
LLM_DEV float2 exp2_split(float2 x, int i) {
  return ((i & 15) * NP) % 16 < NP ? exp2_poly2(x) : make_float2(ex2(x.x), ex2(x.y));
}
constexpr int NP_FWD = 3;

constexpr int BQ = 128, BK = 128, HD = 64;
constexpr int TILE_BYTES = 128 * HD * 2;  // 16 KB: 128 rows x 64 bf16, 128-byte swizzle
constexpr int STAGES = 4;  // K and V rings: deep enough to cover the TMA latency under load
// Q slots: an item's O is staged in its own Q slot and released after the
// next item's first block, so the Q of item it + 1 goes into the slot of item
// it - 2; with two slots the next item's first S (and the MMA warp's P V of
// this item's last block, issued after it) would wait for that release and a
// Q load at every item boundary, which dominates items of one or two blocks
constexpr int QSLOTS = 3;
constexpr int NQ = 4;             // key groups of a block (independent softmaxes)
constexpr int KW = 128 / NQ;      // keys per group (softmax thread)
constexpr int SM_WARPS = 4 * NQ;  // softmax warps: 4 lane quarters x NQ groups
constexpr int MMA_B_WARP = 2 + SM_WARPS;
constexpr int NTHREADS = 32 * (MMA_B_WARP + 1);
constexpr int TMEM_COLS = 512;
// TMEM columns: two S buffers [0,128) and [128,256) (block j in buffer j % 2;
// group g's P of that block, packed bf16, over the first KW/2 of the group's
// own S columns once read), O_g at COL_O + 64 g
constexpr int COL_S = 0, COL_O = 256;
static_assert(COL_O + 64 * NQ <= TMEM_COLS, "TMEM columns");
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr float LAZY = 8.f;  // log2 units a row maximum may grow before O is rescaled
// shared memory: Q[2] | K[STAGES] | V[STAGES] | barriers | red[2]
constexpr int BAR_BYTES = 512;  // 48 mbarrier slots, then the TMEM address and abort words
constexpr int SMEM_BYTES =
    (QSLOTS + 2 * STAGES) * TILE_BYTES + BAR_BYTES + 2 * 2 * NQ * 128 * 4 + 1024;

// P = 2^(s sl2 - mr) for the KW scores of one (row, group), packed bf16 into
// w; returns their sum.  Pairs in packed f32x2 arithmetic; with FMA_EXP some
// pairs take the polynomial 2^x, the rest the SFU.
template <bool FMA_EXP>
LLM_DEV float exp_pack(const float (&sv)[KW], float sl2, float mr, uint32_t (&w)[KW / 2]) {
  float2 la = make_float2(0.f, 0.f), lb = make_float2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < KW; i += 2) {
    const float2 x = __ffma2_rn(make_float2(sv[i], sv[i + 1]), make_float2(sl2, sl2),
                                make_float2(-mr, -mr));
    const float2 p = FMA_EXP ? exp2_split<NP_FWD>(x, i / 2) : make_float2(ex2(x.x), ex2(x.y));
    if ((i >> 1) & 1) lb = __fadd2_rn(lb, p);
    else la = __fadd2_rn(la, p);
    w[i / 2] = pack_bf16(p.x, p.y);
  }
  return (la.x + lb.x) + (la.y + lb.y);
}

// Named barrier of the softmax warps (id 1) that ANDs a flag over them.
LLM_DEV bool softmax_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 1, %2, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(32 * SM_WARPS)
      : "memory");
  return r != 0;
}

// Named barrier of the softmax warps (id 1).
LLM_DEV void softmax_sync() { asm volatile("bar.sync 1, %0;" ::"n"(32 * SM_WARPS) : "memory"); }

__global__ void __launch_bounds__(NTHREADS, 1)
    k_attn_fwd_tc(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_o,
                  float *__restrict__ lse, int B, int T, int H, int Hkv, float scale, int *gflag) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *sQ = smem, *sK = smem + QSLOTS * TILE_BYTES, *sV = sK + STAGES * TILE_BYTES;
  uint64_t *bars = (uint64_t *)(sV + STAGES * TILE_BYTES);
  uint32_t *tmem_sh = (uint32_t *)(bars + 48);
  volatile int *abort_sh = (volatile int *)(tmem_sh + 1);
  float *red = (float *)(bars + BAR_BYTES / 8);  // [2][NQ][128]: m_g, then l_g per row
  const uint32_t b0 = smem_u32(bars);
  const uint32_t q_full = b0, q_empty = b0 + 8 * QSLOTS,  // [QSLOTS]: Q slot
                 k_full = b0 + 16 * QSLOTS, k_empty = k_full + 8 * STAGES,
                 v_full = k_empty + 8 * STAGES, v_empty = v_full + 8 * STAGES,
                 s_full = v_empty + 8 * STAGES,    // [2]: one per S buffer
                 buf_free = s_full + 16,           // [2]: the buffer's P V products done
                 // [2][NQ]: per S buffer and key group, so that a group's arrivals for
                 // blocks j and j + 1 (other buffer) can never alias one phase
                 p_full = buf_free + 16,
                 o_done = p_full + 16 * NQ,        // [NQ]
                 drain = o_done + 8 * NQ;          // [2]: one per MMA warp
  static_assert(2 * QSLOTS + 4 * STAGES + 4 + 3 * NQ + 2 <= 48,
                "barriers overlap the TMEM address word");
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
    for (int x = 0; x < QSLOTS; x++) {
      mbar_init(q_full + 8 * x, 1);
      // the item's last S product on the slot, then the bulk stores of O
      // staged in it (one per softmax warp)
      mbar_init(q_empty + 8 * x, 1 + SM_WARPS);
    }
    for (int s = 0; s < STAGES; s++) {
      mbar_init(k_full + 8 * s, 1);
      mbar_init(k_empty + 8 * s, 1);
      mbar_init(v_full + 8 * s, 1);
      mbar_init(v_empty + 8 * s, 2);  // both P V halves read V_j
    }
    for (int bb = 0; bb < 2; bb++) {
      mbar_init(s_full + 8 * bb, 1);
      mbar_init(buf_free + 8 * bb, 2);  // both MMA warps' P V products of the block
    }
    for (int g2 = 0; g2 < 2 * NQ; g2++) mbar_init(p_full + 8 * g2, 4);  // 4 lane-quarter warps
    for (int g2 = 0; g2 < NQ; g2++) mbar_init(o_done + 8 * g2, 1);
    mbar_init(drain, 1);
    mbar_init(drain + 8, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_sh)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_sh;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      int gb = 0, nq = 0;  // key blocks and Q tiles issued
      bool ok = true;
      for (int r = 0, it = 0; ok; r++, it++) {
        const int item = sched_item(r, G, cta);
        if (item >= n_items) break;
        int qb, h, b;
        decode(item, qb, h, b);
        const int row_base = b * T, g = h / (H / Hkv), slot = it % QSLOTS;
        // Q into the slot of item it - QSLOTS once its last S product and the
        // store of its O (staged in the slot) completed
        if (!mbar_wait(q_empty + 8 * slot, ((it / QSLOTS) & 1) ^ 1, abort_sh, gflag)) break;
        mbar_arrive_expect_tx(q_full + 8 * slot, TILE_BYTES);
        tma_load_3d(smem_u32(sQ + slot * TILE_BYTES), &tm_qkv, 0, h, row_base + qb * BQ,
                    q_full + 8 * slot);
        nq = it + 1;
        for (int j = 0; j <= qb; j++) {
          const int s = gb % STAGES;
          const uint32_t ph = (gb / STAGES) & 1;
          if (!mbar_wait(k_empty + 8 * s, ph ^ 1, abort_sh, gflag) ||
              !mbar_wait(v_empty + 8 * s, ph ^ 1, abort_sh, gflag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(k_full + 8 * s, TILE_BYTES);
          tma_load_3d(smem_u32(sK + s * TILE_BYTES), &tm_qkv, 0, H + g, row_base + j * BK,
                      k_full + 8 * s);
          mbar_arrive_expect_tx(v_full + 8 * s, TILE_BYTES);
          tma_load_3d(smem_u32(sV + s * TILE_BYTES), &tm_qkv, 0, H + Hkv + g,
                      row_base + j * BK, v_full + 8 * s);
          gb++;
        }
      }
      // every copy this thread issued has landed before the CTA may exit
      for (int i = max(0, nq - QSLOTS); i < nq; i++)
        drain_wait(q_full + 8 * (i % QSLOTS), (i / QSLOTS) & 1);
      for (int i = max(0, gb - STAGES); i < gb; i++) {
        drain_wait(k_full + 8 * (i % STAGES), (i / STAGES) & 1);
        drain_wait(v_full + 8 * (i % STAGES), (i / STAGES) & 1);
      }
    }
  } else if (warp == 1 || warp == MMA_B_WARP) {
    // ------------------------------------- MMA issuers (whole warps)
    const int x = warp == 1 ? 0 : 1;  // which key half's P V this warp issues
    constexpr uint32_t ID_S = idesc_mn(128, BK, false, false);
    constexpr uint32_t ID_O = idesc_mn(128, HD, false, true);
    auto issue_s = [&](int slot, int gbn) {  // S = Q K^T of global block gbn into buffer gbn % 2
      const int s = gbn % STAGES;
      const uint64_t qd = sdesc(smem_u32(sQ + slot * TILE_BYTES), 16, 1024);
      const uint64_t kd = sdesc(smem_u32(sK + s * TILE_BYTES), 16, 1024);
#pragma unroll
      for (int kk = 0; kk < HD / 16; kk++)
        mma_bf16_e(tmem + COL_S + 128 * (gbn & 1), qd + (uint64_t)(kk * 2),
                   kd + (uint64_t)(kk * 2), ID_S, kk > 0 ? 1u : 0u);
      mma_commit_e(s_full + 8 * (gbn & 1));
      mma_commit_e(k_empty + 8 * s);
    };
    bool ok = true;
    int gb = 0;
    int item = sched_item(0, G, cta);
    if (x == 0 && item < n_items) {  // scores of the first block
      int qb, h, b;
      decode(item, qb, h, b);
      ok = warp_wait(q_full, 0, abort_sh, gflag) && warp_wait(k_full, 0, abort_sh, gflag);
      if (ok) {
        fence_after();
        issue_s(0, 0);
        if (qb == 0) mma_commit_e(q_empty);  // the item's last S product on slot 0
      }
    }
    for (int r = 0, it = 0; item < n_items && ok; r++, it++) {
      int qb, h, b;
      decode(item, qb, h, b);
      const int nj = qb + 1, slot = it % QSLOTS;
      const int next = sched_item(r + 1, G, cta);
      int qb_next = 0, hn, bn;
      if (next < n_items) decode(next, qb_next, hn, bn);
      for (int j = 0; j < nj && ok; j++, gb++) {
        const int s = gb % STAGES;
        const uint32_t ph = (gb / STAGES) & 1;
        const bool here = j + 1 < nj;
        if (x == 0 && (here || next < n_items)) {
          // scores of block gb + 1 (this item's next, or the next item's
          // first) into the other buffer once its P V products (block gb - 1)
          // have completed
          const int slot1 = here ? slot : (it + 1) % QSLOTS;
          const int s1 = (gb + 1) % STAGES;
          const uint32_t ph1 = ((gb + 1) / STAGES) & 1;
          if ((!here && !warp_wait(q_full + 8 * slot1, ((it + 1) / QSLOTS) & 1, abort_sh, gflag)) ||
              !warp_wait(k_full + 8 * s1, ph1, abort_sh, gflag) ||
              (gb >= 1 && !warp_wait(buf_free + 8 * ((gb + 1) & 1), ((gb - 1) >> 1) & 1, abort_sh,
                                     gflag))) {
            ok = false;
            break;
          }
          fence_after();
          issue_s(slot1, gb + 1);
          if (here ? (j + 1 == nj - 1) : (qb_next == 0)) mma_commit_e(q_empty + 8 * slot1);
        }
        if (!warp_wait(v_full + 8 * s, ph, abort_sh, gflag)) {
          ok = false;
          break;
        }
        const uint64_t vd = sdesc(smem_u32(sV + s * TILE_BYTES), 8192, 1024);
        // O_g += P_g V[g KW : g KW + KW] for this warp's groups: KW / 16 K-steps
        // (at an item's first block the softmax warps arrive only after the
        // previous item's accumulators were read out)
#pragma unroll
        for (int gg = 0; gg < NQ / 2; gg++) {
          const int grp = x * (NQ / 2) + gg;
          if (!warp_wait(p_full + 8 * ((gb & 1) * NQ + grp), (gb >> 1) & 1, abort_sh, gflag)) {
            ok = false;
            break;
          }
          fence_after();
#pragma unroll
          for (int kk = 0; kk < KW / 16; kk++)
            mma_ts_e(tmem + COL_O + 64 * grp, tmem + COL_S + 128 * (gb & 1) + grp * KW + kk * 8,
                     vd + (uint64_t)((grp * (KW / 16) + kk) * 128), ID_O,
                     (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit_e(o_done + 8 * grp);
        }
        if (!ok) break;
        mma_commit_e(v_empty + 8 * s);
        mma_commit_e(buf_free + 8 * (gb & 1));
      }
      item = next;
    }
    mma_commit_e(drain + 8 * x);
    if (lane == 0) {
      unsigned long long t0 = gtimer();
      while (!mbar_try(drain + 8 * x, 0) && gtimer() - t0 < WAIT_NS) {
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3;
    const int grp = (warp - 2) >> 2;    // key group: keys [grp KW, grp KW + KW) of a block
    const int r = quarter * 32 + lane;  // row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t col_o = COL_O + 64 * grp;
    const float sl2 = scale * LOG2E;
    int gb = 0, st_slot = -1;  // Q slot whose O store is still to be released
    for (int rr = 0, it = 0;; rr++, it++) {
      const int item = sched_item(rr, G, cta);
      if (item >= n_items) break;
      int qb, h, b;
      decode(item, qb, h, b);
      const int q0 = qb * BQ, nj = qb + 1;
      const int qi = q0 + r;
      float m_ref = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = 0; j < nj && ok; j++, gb++) {
        const uint32_t col_s = COL_S + 128 * (gb & 1) + grp * KW;  // this group's S, then P
        if (!warp_wait(s_full + 8 * (gb & 1), (gb >> 1) & 1, abort_sh, gflag)) {
          ok = false;
          break;
        }
        fence_after();
        const int k0 = j * BK + grp * KW;
        const bool diag = (j * BK + BK > q0);  // only the diagonal block (or T) masks
        float sv[KW];
        tmem_ldn<KW>(tmem + lane_off + col_s, sv);
        // this group's block maximum on the raw scores (the log2 factor sl2 > 0
        // keeps the order), 4 independent chains; masked scores become -inf
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (diag) {  // the diagonal block (and keys past T): mask, then the maximum
#pragma unroll
          for (int i = 0; i < KW; i++) {
            if (k0 + i > qi || k0 + i >= T) sv[i] = -INFINITY;
            m4[i & 3] = fmaxf(m4[i & 3], sv[i]);
          }
        } else {  // three-input maxima, 4 independent chains
#pragma unroll
          for (int i = 0; i < KW; i += 2)
            m4[(i >> 1) & 3] = fmax3(m4[(i >> 1) & 3], sv[i], sv[i + 1]);
        }
        const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;
        // true on the first block with an unmasked key (m_ref = -inf until then)
        const bool need = mx > m_ref + LAZY;
        // O_g is rescaled only after the previous block's P V into it completed
        if (j > 0 && __any_sync(0xffffffffu, need)) {
          if (!warp_wait(o_done + 8 * grp, (gb - 1) & 1, abort_sh, gflag)) {
            ok = false;
            break;
          }
          fence_after();
          {
            const float corr = need ? ex2(m_ref - mx) : 1.f;  // 0 while m_ref = -inf
#pragma unroll
            for (int c = 0; c < 4; c++) {
              float v[16];
              uint32_t u[16];
              tmem_ld16(tmem + lane_off + col_o + c * 16, v);
#pragma unroll
              for (int i = 0; i < 16; i++) u[i] = __float_as_uint(v[i] * corr);
              tmem_st16(tmem + lane_off + col_o + c * 16, u);
            }
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
          }
        }
        if (need) {
          if (m_ref != -INFINITY) l *= ex2(m_ref - mx);
          m_ref = mx;
        }
        // P = 2^(s - m_ref), packed bf16 into this group's KW/2 TMEM columns; a
        // (row, group) with no unmasked key yet (m_ref = -inf) gets P = 0
        const float mr = m_ref == -INFINITY ? 0.f : m_ref;
        uint32_t w[KW / 2];
        // the diagonal block on the SFU alone (its masked scores give exact
        // zeros); elsewhere some pairs on the FMA pipe (exp2_split)
        l += diag ? exp_pack<false>(sv, sl2, mr, w) : exp_pack<true>(sv, sl2, mr, w);
#pragma unroll
        for (int c = 0; c < KW / 2; c += 16)
          tmem_stn<(KW / 2 < 16 ? KW / 2 : 16)>(tmem + lane_off + col_s + c, w + c);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + 8 * ((gb & 1) * NQ + grp));
        // the previous item's O store has long read its tile: release the slot
        if (st_slot >= 0) {
          if (lane == 0) {
            bulk_wait_read();
            mbar_arrive(q_empty + 8 * st_slot);
          }
          st_slot = -1;
        }
      }
      // the groups meet: shared reference m, combined sum and output; every
      // accumulator is complete once every o_done phase of the item's last
      // block is
#pragma unroll
      for (int g2 = 0; g2 < NQ; g2++)
        if (ok) ok = warp_wait(o_done + 8 * g2, (gb - 1) & 1, abort_sh, gflag);
      float *rd = red + (it & 1) * 2 * NQ * 128;
      rd[grp * 128 + r] = m_ref;
      rd[(NQ + grp) * 128 + r] = l;
      // barrier of the softmax warps that also tells whether every one
      // finished (each warp reaches it once per item, also after a failed
      // wait, so all of them leave together)
      if (!softmax_all(ok)) break;
      fence_after();
      float m = -INFINITY;
#pragma unroll
      for (int g2 = 0; g2 < NQ; g2++) m = fmaxf(m, rd[g2 * 128 + r]);
      float f[NQ], lt = 0.f;
#pragma unroll
      for (int g2 = 0; g2 < NQ; g2++) {
        const float mg = rd[g2 * 128 + r];
        f[g2] = mg == -INFINITY ? 0.f : ex2(mg - m);
        lt += rd[(NQ + g2) * 128 + r] * f[g2];
      }
      const float inv = 1.f / lt;
      // this thread's 64 / NQ output columns: [grp 64/NQ, grp 64/NQ + 64/NQ)
      constexpr int OW = 64 / NQ;
      float acc[OW];
#pragma unroll
      for (int i = 0; i < OW; i++) acc[i] = 0.f;
      // two groups' loads in flight per wait, added in group order
#pragma unroll
      for (int g2 = 0; g2 < NQ; g2 += 2) {
        uint32_t va[OW], vb[OW];
        tmem_ld_raw<OW>(tmem + lane_off + COL_O + 64 * g2 + grp * OW, va);
        tmem_ld_raw<OW>(tmem + lane_off + COL_O + 64 * (g2 + 1) + grp * OW, vb);
        tmem_wait_ld();
        tmem_after_wait(va);
        tmem_after_wait(vb);
        const float ca = f[g2] * inv, cb = f[g2 + 1] * inv;
#pragma unroll
        for (int i = 0; i < OW; i++) acc[i] += __uint_as_float(va[i]) * ca;
#pragma unroll
        for (int i = 0; i < OW; i++) acc[i] += __uint_as_float(vb[i]) * cb;
      }
      // O rows through the item's Q tile (its last S product is complete):
      // this thread's two 16-byte chunks of row r in the tile's
      // 128-byte-swizzle image
      uint8_t *srow = sQ + (it % QSLOTS) * TILE_BYTES + r * 128;
#pragma unroll
      for (int c = 0; c < OW / 8; c++) {
        const int ch = grp * (OW / 8) + c;
        *reinterpret_cast<uint4 *>(srow + ((ch ^ (r & 7)) << 4)) =
            make_uint4(pack_bf16(acc[8 * c], acc[8 * c + 1]), pack_bf16(acc[8 * c + 2], acc[8 * c + 3]),
                       pack_bf16(acc[8 * c + 4], acc[8 * c + 5]),
                       pack_bf16(acc[8 * c + 6], acc[8 * c + 7]));
      }
      fence_proxy_async();
      // every softmax warp has read every accumulator (before any of them
      // releases the next item's first P, whose P V overwrites O_g) and staged
      // its part of O
      fence_before();
      softmax_sync();
      if (lane == 0) {  // 8 whole rows of this warp's lane quarter (rows past T clipped)
        const int r0 = quarter * 32 + grp * 8;
        tma_store_4d(&tm_o, smem_u32(sQ + (it % QSLOTS) * TILE_BYTES + r0 * 128), 0, h, q0 + r0, b);
        bulk_commit();
      }
      st_slot = it % QSLOTS;  // released after the next item's first block
      if (grp == 0 && qi < T) lse[((int64_t)b * H + h) * T + qi] = (m + __log2f(lt)) * LN2;
    }
    if (lane == 0) bulk_wait_all();
  }
  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

}  // namespace attn_tc

bool attn_tc_covers(DType dt, int hd, int T) {
  return dt == DT_BF16 && (hd == 64 || hd == 32) && T >= 1;
}

// Host side: one tensor map over qkv [B*T rows][H + 2 Hkv heads][hd] serves
// the Q, K and V tiles (box 64 x 1 head x 128 rows, 128-byte swizzle); O
// leaves through a [B][T][H][hd] map (box 64 x 1 x 8 rows x 1).
bool attn_fwd_tc(const void *qkv, void *o, float *lse, int B, int T, int H, int Hkv, int hd,
                 int *flag, cudaStream_t s) {
  using namespace attn_tc;
  if ((hd != 64 && hd != 32) || !flag) return false;
  if (!smem_optin((const void *)k_attn_fwd_tc, SMEM_BYTES)) return false;
  const int64_t qkvw = (int64_t)(H + 2 * Hkv) * hd;
  CUtensorMap map, mo;
  if (!head_map_load(&map, qkv, hd, H + 2 * Hkv, (int64_t)B * T, qkvw, 128) ||
      !head_map_store(&mo, o, hd, H, T, B, (int64_t)H * hd, 8))
    return false;
  const int items = ((T + BQ - 1) / BQ) * H * B;
  k_attn_fwd_tc<<<min(items, device_sms()), NTHREADS, SMEM_BYTES, s>>>(
      map, mo, lse, B, T, H, Hkv, 1.0f / sqrtf((float)hd), flag);
  count_launch();
  return true;
}

}  // namespace llm
