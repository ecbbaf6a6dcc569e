// tcgen05 GEMM for sm_100a: C[M,N] = A[M,K] . B[N,K]^T, bf16 operands, fp32
// accumulation in tensor memory (TMEM).
//
// Persistent kernel, one CTA per SM, 10 warps:
//   warp 0      TMA producer: A and B tiles into a STAGES-deep shared-memory
//               ring (128-byte swizzle), completion counted on mbarriers;
//   warp 1      allocates 512 TMEM columns; issues tcgen05.mma (M=128, N=256,
//               K=16) and commits each stage back to the ring;
// (warps 0 and 1 run as whole converged warps; one elected lane issues each
// copy, MMA and commit)
//   warps 2..9  epilogue, two warps per TMEM lane quarter, each taking half
//               of the tile's columns: tcgen05.ld of the accumulator (one
//               TMEM lane = one output row per thread), the fused epilogue,
//               and bulk tensor stores of a swizzled shared staging square
//               (a residual comes in through bulk tensor loads of the same
//               square).
// Two accumulators of 256 columns alternate so the epilogue of one tile
// overlaps the main loop of the next.  Products with M and N of at least 512
// run on CTA pairs instead (k_gemm_tc2 below: 256 x 256 tiles on two SMs,
// tcgen05.mma.cta_group::2), the rest on single CTAs.  Operands may be K-major or MN-major
// (both supported by the UMMA descriptors), which covers the forward
// (x W), data-gradient (dy W^T) and weight-gradient (x^T dy) orientations
// without transposed copies.  Every mbarrier wait is bounded; on time-out the
// kernel records FLAG_TIMEOUT, drains its own copies and MMAs, frees TMEM and
// returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>
#include <unordered_map>

#include "common.cuh"
#include "gemm_tc.h"
#include "tcgen05.cuh"

namespace llm {

namespace tc {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int STG_BUFS = 1;  // staging squares per epilogue warp (bulk stores in flight)
constexpr int A_BYTES = BM * BK * 2;            // 16 KB
constexpr int B_BYTES = BN * BK * 2;            // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 48 KB
constexpr int EPI_WARPS = 8;
constexpr int STAGING_BYTES = EPI_WARPS * STG_BUFS * 32 * 32 * 4;  // 32x32 float squares
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + STAGING_BYTES + 256 /*barriers*/;
constexpr int TMEM_COLS = 512;
constexpr int NTHREADS = 64 + 32 * EPI_WARPS;

struct Args {
  int M, N, K;
  int tiles_m, tiles_n, splits, kchunk, total;
  int nfast;  // tile order of a split: n tiles fastest (1) or m tiles fastest (0)
  int out, epi;
  void *C;
  int64_t ldc;
  const float *R;
  int64_t ldr;
  const float *cos_t, *sin_t;
  int T, hd, rot_cols;
  int *flag;
};

// Tile `tile` of a split -> (m tile, n tile).  With few n tiles (a product of
// N <= 2048 over a long A, e.g. a data gradient dY W with K = vocabulary or
// hidden width) n runs fastest, so the CTAs at work together take every n tile
// of the same A rows and read each A panel from HBM once, sharing it in L2 (m
// fastest re-read every A panel once per n tile: 3.4-3.8x the algorithmic
// bytes); otherwise m runs fastest and the A operand stays in L2 across n.
LLM_DEV void tile_mn(const Args &a, int tile, int &mt, int &nt) {
  if (a.nfast) {
    mt = tile / a.tiles_n;
    nt = tile - mt * a.tiles_n;
  } else {
    nt = tile / a.tiles_m;
    mt = tile - nt * a.tiles_m;
  }
}

// ------------------------------------------------------------ epilogue stores
// A warp's 32 x 32 fp32 chunk (lane i holds row i in v) in the per-warp
// staging square: 16-byte group g of row r sits at position g ^ (r & 7), the
// 128-byte-swizzle image of a 32-row x 128-byte box, so the row-wise 16-byte
// writes spread over all banks and the square is what a bulk tensor copy of
// that box reads or writes.
LLM_DEV float4 *sq(float *stg, int r, int g) {
  return reinterpret_cast<float4 *>(stg + r * 32 + 4 * (g ^ (r & 7)));
}
LLM_DEV void stage32(float *stg, const float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int g = 0; g < 8; g++) *sq(stg, lane, g) = make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
  __syncwarp();
}
// Bulk tensor stores.  The staging square is laid out as the 128-byte-swizzle
// image of a 32-row x 128-byte box (16-byte group g of row r at g ^ (r & 7)),
// i.e. exactly what the tensor map of C expects; the copy engine clips rows
// and columns outside C.  One store group per warp is in flight at a time:
// stg_acquire waits until the previous store has read the square.
LLM_DEV void stg_acquire() {
  if ((threadIdx.x & 31) == 0)
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(STG_BUFS - 1) : "memory");
  __syncwarp();
}
LLM_DEV void bulk_store(const float *stg, const CUtensorMap *tm, int x, int y, int z, bool three_d) {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncwarp();
  if ((threadIdx.x & 31) == 0) {
    if (three_d)
      asm volatile(
          "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
              (uint64_t)tm),
          "r"(x), "r"(y), "r"(z), "r"(smem_u32(stg))
          : "memory");
    else
      asm volatile(
          "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
              (uint64_t)tm),
          "r"(x), "r"(y), "r"(smem_u32(stg))
          : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  }
}
// 64 bf16 columns of the warp's 32 rows (lo = columns 0..31, hi = 32..63):
// 8 groups of 8 values per row, swizzled like the float square.
LLM_DEV void stage64_bf16(float *stg, const float (&lo)[32], const float (&hi)[32]) {
  const int lane = threadIdx.x & 31;
  uint4 *row = reinterpret_cast<uint4 *>(stg + lane * 32);
#pragma unroll
  for (int j = 0; j < 4; j++) {
    row[j ^ (lane & 7)] = make_uint4(pack_bf16(lo[8 * j], lo[8 * j + 1]), pack_bf16(lo[8 * j + 2], lo[8 * j + 3]),
                                     pack_bf16(lo[8 * j + 4], lo[8 * j + 5]), pack_bf16(lo[8 * j + 6], lo[8 * j + 7]));
    row[(4 + j) ^ (lane & 7)] = make_uint4(pack_bf16(hi[8 * j], hi[8 * j + 1]), pack_bf16(hi[8 * j + 2], hi[8 * j + 3]),
                                           pack_bf16(hi[8 * j + 4], hi[8 * j + 5]), pack_bf16(hi[8 * j + 6], hi[8 * j + 7]));
  }
}
LLM_DEV void rope32(float (&v)[32], const float *cos_row, const float *sin_row) {
  // both halves of a 32-wide head in one chunk: (v[j], v[j+16]) rotate by angle j
  const float4 *ct = reinterpret_cast<const float4 *>(cos_row);
  const float4 *st = reinterpret_cast<const float4 *>(sin_row);
#pragma unroll
  for (int j4 = 0; j4 < 4; j4++) {
    float4 c4 = ct[j4], s4 = st[j4];
    const float cc[4] = {c4.x, c4.y, c4.z, c4.w}, ss[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
    for (int k = 0; k < 4; k++) {
      int j = 4 * j4 + k;
      float x = v[j], y = v[j + 16];
      v[j] = x * cc[k] - y * ss[k];
      v[j + 16] = y * cc[k] + x * ss[k];
    }
  }
}

// One output tile's epilogue for a warp: rows [row0, row0+32) of the tile
// (TMEM lanes of this warp's quarter, lane i = row row0 + i) and the warp's
// half of the columns, [n0 + c_lo, n0 + c_lo + BN/2).  Every lane executes
// every tcgen05.ld (warp-uniform control); rows past M and columns past N are
// clipped only at the stores.
LLM_DEV void epilogue_tile(const Args &a, const CUtensorMap *tmC, const CUtensorMap *tmR,
                           const CUtensorMap *tmU,
                           uint32_t rbar, uint32_t &rph, volatile int *abort_sh, uint32_t tm,
                           int row0, int n0, int c_lo, int split, bool zero, float *stg_base,
                           int &sb) {
  float *stg = stg_base;
  const int lane = threadIdx.x & 31;
  const int m = row0 + lane;
  const int rows = max(0, min(32, a.M - row0));
  const int N = a.N;
  float v[32];
  {
    if (rows == 0) return;  // the warp's 32 rows lie past M: nothing to store
    if (a.out == OUT_ACT) {
      // bf16, 64 columns per store: plain, or RoPE on q/k head columns
      const int t = m % a.T, half = a.hd / 2;
      for (int c0 = c_lo; c0 < c_lo + BN / 2; c0 += 64) {
        const int n = n0 + c0;
        if (n >= N) break;
        float lo[32], hi[32];
        if (zero) {
          for (int i = 0; i < 32; i++) lo[i] = hi[i] = 0.f;
        } else {
          tmem_ld32(tm + c0, lo);
          tmem_ld32(tm + c0 + 32, hi);
        }
        if (a.epi == TC_EPI_ROPE && n < a.rot_cols) {
          const float *cr = a.cos_t + (int64_t)t * half, *sr = a.sin_t + (int64_t)t * half;
          if (a.hd == 64) {
            const float4 *ct = reinterpret_cast<const float4 *>(cr);
            const float4 *st = reinterpret_cast<const float4 *>(sr);
#pragma unroll
            for (int j4 = 0; j4 < 8; j4++) {
              float4 c4 = ct[j4], s4 = st[j4];
              const float cc[4] = {c4.x, c4.y, c4.z, c4.w}, ss[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
              for (int k = 0; k < 4; k++) {
                int j = 4 * j4 + k;
                float x = lo[j], y = hi[j];
                lo[j] = x * cc[k] - y * ss[k];
                hi[j] = y * cc[k] + x * ss[k];
              }
            }
          } else {  // hd == 32: each 32-column chunk is one head
            rope32(lo, cr, sr);
            if (n + 32 < a.rot_cols) rope32(hi, cr, sr);
          }
        }
        stg = stg_base + sb * 32 * 32;
        sb = sb + 1 == STG_BUFS ? 0 : sb + 1;
        stg_acquire();
        stage64_bf16(stg, lo, hi);
        bulk_store(stg, tmC, n, row0, 0, false);
      }
      if (a.epi == TC_EPI_SWIGLU && n0 + c_lo < N) {
        // the warp's 128 columns are one interleaved block, a for 64 hidden
        // units then b for the same units: u = silu(a) b from the
        // accumulator rounded as the stored [a|b] is, 32 units at a time,
        // into the u tile at hidden column (n0 + c_lo) / 2
        float u0[32], u1[32];
        {
          float av[32], bv[32];
          if (zero) {
            for (int i = 0; i < 32; i++) av[i] = bv[i] = 0.f;
          } else {
            tmem_ld32(tm + c_lo, av);
            tmem_ld32(tm + c_lo + 64, bv);
          }
#pragma unroll
          for (int i = 0; i < 32; i++) u0[i] = swiglu_unit_bf16(av[i], bv[i]);
        }
        {
          float av[32], bv[32];
          if (zero) {
            for (int i = 0; i < 32; i++) av[i] = bv[i] = 0.f;
          } else {
            tmem_ld32(tm + c_lo + 32, av);
            tmem_ld32(tm + c_lo + 96, bv);
          }
#pragma unroll
          for (int i = 0; i < 32; i++) u1[i] = swiglu_unit_bf16(av[i], bv[i]);
        }
        stg = stg_base + sb * 32 * 32;
        sb = sb + 1 == STG_BUFS ? 0 : sb + 1;
        stg_acquire();
        stage64_bf16(stg, u0, u1);
        bulk_store(stg, tmU, (n0 + c_lo) / 2, row0, 0, false);
      }
    } else {
      // fp32 (plain, residual add, or split-K partial into slab `split`), 32
      // columns per store; the residual chunk R[rows, n : n + 32] is brought
      // into the staging square by a bulk tensor load (zero past M and N)
      // while the accumulator is read from TMEM, then added in place
      const bool part = a.out == OUT_PARTIAL, add = a.out == OUT_ADD_F32;
      for (int c0 = c_lo; c0 < c_lo + BN / 2; c0 += 32) {
        const int n = n0 + c0;
        if (n >= N) break;
        stg = stg_base + sb * 32 * 32;
        sb = sb + 1 == STG_BUFS ? 0 : sb + 1;
        stg_acquire();
        if (add) {
          mbar_arrive_expect_tx_e(rbar, 32 * 32 * 4);
          tma_load_2d_e(smem_u32(stg), tmR, n, row0, rbar);
        }
        if (zero) { for (int i = 0; i < 32; i++) v[i] = 0.f; }
        else tmem_ld32(tm + c0, v);
        if (add) {
          const uint32_t ph = rph;
          rph ^= 1u;
          if (!warp_wait(rbar, ph, abort_sh, a.flag)) {
            // time-out: the load must land before the square is reused or freed
            if ((threadIdx.x & 31) == 0) {
              const unsigned long long t0 = gtimer();
              while (!mbar_try(rbar, ph) && gtimer() - t0 < WAIT_NS) {
              }
            }
            __syncwarp();
            return;
          }
#pragma unroll
          for (int g = 0; g < 8; g++) {
            const float4 r4 = *sq(stg, lane, g);
            v[4 * g] += r4.x; v[4 * g + 1] += r4.y; v[4 * g + 2] += r4.z; v[4 * g + 3] += r4.w;
          }
          __syncwarp();
        }
        stage32(stg, v);
        bulk_store(stg, tmC, n, row0, split, part);
      }
    }
  }
}

template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmR,
              const __grid_constant__ CUtensorMap tmU, const Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t *bars = (uint64_t *)(smem + STAGES * STAGE_BYTES + STAGING_BYTES);
  // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2], drain, rbar[EPI_WARPS]
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_sh;
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const uint32_t full0 = smem_u32(bars), empty0 = full0 + 8 * STAGES;
  const uint32_t tfull0 = empty0 + 8 * STAGES, tempty0 = tfull0 + 16, drain = tempty0 + 16;
  const uint32_t rbar0 = drain + 8;  // residual-load barrier of each epilogue warp
  static_assert(8 * (2 * STAGES + 5 + EPI_WARPS) <= 256, "barrier space");

  if (threadIdx.x == 0) {
    abort_sh = 0;
    for (int s = 0; s < STAGES; s++) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, EPI_WARPS);
    }
    mbar_init(drain, 1);
    for (int w = 0; w < EPI_WARPS; w++) mbar_init(rbar0 + 8 * w, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tmem_base_sh)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = tmem_base_sh;
  const int tiles_mn = a.tiles_m * a.tiles_n;
  const int kblocks_total = (a.K + BK - 1) / BK;

  auto kblocks_of = [&](int split, int &kb0) {
    int kb_per = a.kchunk / BK;
    kb0 = split * kb_per;
    int kb1 = min(kblocks_total, kb0 + kb_per);
    return max(0, kb1 - kb0);
  };

  if (warp == 0) {
    // -------------------------------------------------- TMA producer
    // whole warp (warp-uniform control flow); one elected lane issues
    int s = 0;
    uint32_t ph = 0;
    uint32_t issued_parity[STAGES];
    bool issued[STAGES];
    for (int i = 0; i < STAGES; i++) issued[i] = false;
    bool ok = true;
    for (int w = blockIdx.x; w < a.total && ok; w += gridDim.x) {
      int split = w / tiles_mn, tile = w % tiles_mn, mt, nt;
      tile_mn(a, tile, mt, nt);
      int m0 = mt * BM, n0 = nt * BN;
      int kb0, nkb = kblocks_of(split, kb0);
      for (int kb = 0; kb < nkb; kb++) {
        if (!warp_wait(empty0 + 8 * s, ph ^ 1, &abort_sh, a.flag)) { ok = false; break; }
        uint32_t fb = full0 + 8 * s;
        mbar_arrive_expect_tx_e(fb, STAGE_BYTES);
        uint32_t sa = smem_u32(smem + s * STAGE_BYTES), sb = sa + A_BYTES;
        int k0 = (kb0 + kb) * BK;
        if (A_MN) {
          tma_load_2d_e(sa, &tmA, m0, k0, fb);
          tma_load_2d_e(sa + 8192, &tmA, m0 + 64, k0, fb);
        } else {
          tma_load_2d_e(sa, &tmA, k0, m0, fb);
        }
        if (B_MN) {
#pragma unroll
          for (int j = 0; j < 4; j++) tma_load_2d_e(sb + 8192 * j, &tmB, n0 + 64 * j, k0, fb);
        } else {
          tma_load_2d_e(sb, &tmB, k0, n0, fb);
        }
        issued[s] = true;
        issued_parity[s] = ph;
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
    }
    // Our copies must have landed before the CTA exits (normally they were
    // consumed already; after an abort they may still be in flight).
    if (lane == 0)
      for (int i = 0; i < STAGES; i++)
        if (issued[i]) {
          unsigned long long t0 = gtimer();
          while (!mbar_try(full0 + 8 * i, issued_parity[i]) && gtimer() - t0 < WAIT_NS) {
          }
        }
    __syncwarp();
  } else if (warp == 1) {
    // -------------------------------------------------- MMA issuer
    // The whole warp runs the loop (warp-uniform control flow); one elected
    // lane issues each MMA and commit.
    constexpr uint32_t ID = idesc_mn(BM, BN, A_MN, B_MN);
    int s = 0;
    uint32_t ph = 0;
    int acc = 0;
    uint32_t aph = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < a.total && ok; w += gridDim.x) {
      int split = w / tiles_mn;
      int kb0, nkb = kblocks_of(split, kb0);
      if (nkb == 0) continue;  // epilogue writes zeros without waiting
      if (!warp_wait(tempty0 + 8 * acc, aph ^ 1, &abort_sh, a.flag)) break;
      fence_after();
      uint32_t td = tmem + acc * BN;
      for (int kb = 0; kb < nkb; kb++) {
        if (!warp_wait(full0 + 8 * s, ph, &abort_sh, a.flag)) { ok = false; break; }
        fence_after();
        uint32_t sa = smem_u32(smem + s * STAGE_BYTES), sb = sa + A_BYTES;
        uint64_t ad = A_MN ? sdesc(sa, 8192, 1024) : sdesc(sa, 16, 1024);
        uint64_t bd = B_MN ? sdesc(sb, 8192, 1024) : sdesc(sb, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < BK / 16; kk++) {
          // advance 16 K elements: 32 bytes inside a K-major swizzle row, or
          // 16 rows (2048 bytes) of an MN-major tile; >>4 for the descriptor
          uint64_t da = (uint64_t)(A_MN ? kk * 128 : kk * 2);
          uint64_t db = (uint64_t)(B_MN ? kk * 128 : kk * 2);
          mma_bf16_e(td, ad + da, bd + db, ID, (kb > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit_e(empty0 + 8 * s);  // frees the stage when these MMAs finish
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
      if (!ok) break;
      mma_commit_e(tfull0 + 8 * acc);  // accumulator ready for the epilogue
      if (++acc == 2) { acc = 0; aph ^= 1; }
    }
    // drain: every MMA this warp issued has completed
    mma_commit_e(drain);
    if (lane == 0) {
      unsigned long long t0 = gtimer();
      while (!mbar_try(drain, 0) && gtimer() - t0 < WAIT_NS) {
      }
    }
    __syncwarp();
  } else {
    // -------------------------------------------------- epilogue warps
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const int ew = warp - 2;       // epilogue warp 0..7
    const int c_lo = (ew / 4) * (BN / 2);
    float *stg = reinterpret_cast<float *>(smem + STAGES * STAGE_BYTES) + ew * STG_BUFS * 32 * 32;
    int sb = 0;  // next staging square of this warp
    uint32_t rph = 0;  // phase of this warp's residual-load barrier
    const uint32_t rbar = rbar0 + 8 * ew;
    int acc = 0;
    uint32_t aph = 0;
    for (int w = blockIdx.x; w < a.total; w += gridDim.x) {
      int split = w / tiles_mn, tile = w % tiles_mn, mt, nt;
      tile_mn(a, tile, mt, nt);
      int m0 = mt * BM, n0 = nt * BN;
      int kb0, nkb = kblocks_of(split, kb0);
      const int row0 = m0 + quarter * 32;
      if (nkb == 0) {
        epilogue_tile(a, &tmC, &tmR, &tmU, rbar, rph, &abort_sh, 0, row0, n0, c_lo, split, true, stg,
                      sb);
        continue;
      }
      if (!warp_wait(tfull0 + 8 * acc, aph, &abort_sh, a.flag)) break;
      fence_after();
      uint32_t tm = tmem + acc * BN + ((uint32_t)(quarter * 32) << 16);
      epilogue_tile(a, &tmC, &tmR, &tmU, rbar, rph, &abort_sh, tm, row0, n0, c_lo, split, false, stg,
                    sb);
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
      if (++acc == 2) { acc = 0; aph ^= 1; }
    }
    // this warp's bulk stores have completed before the CTA may exit
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    __syncwarp();
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

// ------------------------------------------------- CTA-pair (cta_group::2)
// A cluster of two CTAs on two SMs computes one 256 x 256 tile: CTA r loads
// rows [m0 + 128 r, m0 + 128 r + 128) of A and columns [n0 + 128 r, ...) of
// B (32 KiB per stage, no multicast), and the leader (r = 0) issues
// tcgen05.mma.cta_group::2 (M 256, N 256, K 16), which reads A's halves and
// B's halves from both CTAs' shared memory at the same offsets and leaves rows
// 128 r .. 128 r + 127 of the tile in CTA r's TMEM.  Per output element each
// SM moves a third fewer operand bytes than the single-CTA 128 x 256 tile.
//   full[s] (leader): both CTAs' copies of stage s complete on it (the
//     cta_group::2 form of the tensor copy takes the leader's barrier), armed
//     once by the leader for both CTAs' bytes;
//   empty[s], tfull[b]: the leader's commits arrive on both CTAs' barriers
//     (commit multicast);
//   tempty[b] (leader): both CTAs' epilogue warps arrive (the peer's remotely).
// (A first form let each CTA's copies complete on its own barrier and had the
// peer relay the completion to the leader: measured at half the rate of the
// single-CTA kernel, the relay hop serialising every stage.)  The leader's
// drain waits on its full barriers, which count both CTAs' bytes, and the
// final cluster barrier keeps the peer resident until then.  Both CTAs walk
// the same work items; every wait is bounded.
constexpr int STAGES2 = 6;
constexpr int HALF_BYTES = 128 * BK * 2;          // 16 KB: 128 rows x 64 K
constexpr int STAGE2_BYTES = 2 * HALF_BYTES;      // this CTA's A rows and B columns
constexpr int SMEM2_BYTES = STAGES2 * STAGE2_BYTES + 1024 + STAGING_BYTES + 512;

LLM_DEV uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Shared-memory address of the same object in CTA `rank` of the cluster.
LLM_DEV uint32_t cluster_addr(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
// TMA load into this CTA's shared memory whose bytes complete on the barrier
// at cluster address `bar` (the leader's), cta_group::2 form.
LLM_DEV void tma_load_2d_pair_e(uint32_t dst, const CUtensorMap *map, int c0, int c1, uint32_t bar) {
  asm volatile(
      "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
      " @e cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];\n}\n" ::"r"(dst),
      "l"((uint64_t)map), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
LLM_DEV void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
LLM_DEV void mbar_arrive_remote(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}
LLM_DEV void mma_pair_e(uint32_t tmem_d, uint64_t ad, uint64_t bd, uint32_t id, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p, e;\n setp.ne.b32 p, %4, 0;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(ad), "l"(bd), "r"(id), "r"(acc)
      : "memory");
}
// Arrive (when the leader's prior MMAs complete) on the barrier at offset
// `bar` in both CTAs of the pair.
LLM_DEV void commit_pair_both_e(uint32_t bar) {
  asm volatile(
      "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;\n}\n" ::"r"(bar),
      "h"((unsigned short)3)
      : "memory");
}

// Arrive on this CTA's barrier when the leader's prior pair MMAs complete.
LLM_DEV void commit_pair_e(uint32_t bar) {
  asm volatile(
      "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n" ::"r"(
          bar)
      : "memory");
}

template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_gemm_tc2(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmR,
               const __grid_constant__ CUtensorMap tmU, const Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t *bars = (uint64_t *)(smem + STAGES2 * STAGE2_BYTES + STAGING_BYTES);
  // bars: full[S2], empty[S2], tfull[2], tempty[2], drain, rbar[EPI_WARPS]
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_sh;
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const uint32_t full0 = smem_u32(bars), empty0 = full0 + 8 * STAGES2;
  const uint32_t tfull0 = empty0 + 8 * STAGES2, tempty0 = tfull0 + 16, drain = tempty0 + 16;
  const uint32_t rbar0 = drain + 8;
  static_assert(8 * (2 * STAGES2 + 5 + EPI_WARPS) <= 512, "barrier space");

  if (threadIdx.x == 0) {
    abort_sh = 0;
    for (int s = 0; s < STAGES2; s++) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, 2 * EPI_WARPS);
    }
    mbar_init(drain, 1);
    for (int w = 0; w < EPI_WARPS; w++) mbar_init(rbar0 + 8 * w, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tmem_base_sh)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any remote arrival
  fence_after();
  const uint32_t tmem = tmem_base_sh;
  const int tiles_mn = a.tiles_m * a.tiles_n;  // tiles of 256 x 256
  const int kblocks_total = (a.K + BK - 1) / BK;
  const int cid = blockIdx.x / 2, ncl = gridDim.x / 2;
  auto kblocks_of = [&](int split, int &kb0) {
    int kb_per = a.kchunk / BK;
    kb0 = split * kb_per;
    int kb1 = min(kblocks_total, kb0 + kb_per);
    return max(0, kb1 - kb0);
  };

  if (warp == 0) {
    // ------------------------------------ TMA producer (each CTA, its halves)
    int s = 0;
    uint32_t ph = 0;
    uint32_t issued_parity[STAGES2];
    bool issued[STAGES2];
    for (int i = 0; i < STAGES2; i++) issued[i] = false;
    bool ok = true;
    const uint32_t lead_full0 = cluster_addr(full0, 0);
    for (int w = cid; w < a.total && ok; w += ncl) {
      const int split = w / tiles_mn, tile = w % tiles_mn;
      int mt, nt;
      tile_mn(a, tile, mt, nt);
      const int m0 = mt * 256 + 128 * (int)rank;
      const int n0 = nt * 256 + 128 * (int)rank;
      int kb0, nkb = kblocks_of(split, kb0);
      for (int kb = 0; kb < nkb; kb++) {
        if (!warp_wait(empty0 + 8 * s, ph ^ 1, &abort_sh, a.flag)) { ok = false; break; }
        // both CTAs' bytes complete on the leader's full[s], armed once for both
        const uint32_t fb = lead_full0 + 8 * s;
        if (leader) mbar_arrive_expect_tx_e(full0 + 8 * s, 2 * STAGE2_BYTES);
        const uint32_t sa = smem_u32(smem + s * STAGE2_BYTES), sb = sa + HALF_BYTES;
        const int k0 = (kb0 + kb) * BK;
        if (A_MN) {
          tma_load_2d_pair_e(sa, &tmA, m0, k0, fb);
          tma_load_2d_pair_e(sa + 8192, &tmA, m0 + 64, k0, fb);
        } else {
          tma_load_2d_pair_e(sa, &tmA, k0, m0, fb);
        }
        if (B_MN) {
          tma_load_2d_pair_e(sb, &tmB, n0, k0, fb);
          tma_load_2d_pair_e(sb + 8192, &tmB, n0 + 64, k0, fb);
        } else {
          tma_load_2d_pair_e(sb, &tmB, k0, n0, fb);
        }
        issued[s] = true;
        issued_parity[s] = ph;
        if (++s == STAGES2) { s = 0; ph ^= 1; }
      }
    }
    // both CTAs' copies complete on the leader's full barriers: the leader
    // waits for them before the pair may exit (normally they were consumed
    // already); the final cluster barrier holds the peer until then
    if (lane == 0 && leader)
      for (int i = 0; i < STAGES2; i++)
        if (issued[i]) {
          const unsigned long long t0 = gtimer();
          while (!mbar_try(full0 + 8 * i, issued_parity[i]) && gtimer() - t0 < WAIT_NS) {
          }
        }
    __syncwarp();
  } else if (warp == 1 && !leader) {
    // the peer's warp 1 only shares the TMEM allocation
  } else if (warp == 1) {
    // ------------------------------------ MMA issuer (leader)
    constexpr uint32_t ID = idesc_mn(256, BN, A_MN, B_MN);
    int s = 0;
    uint32_t ph = 0;
    int acc = 0;
    uint32_t aph = 0;
    bool ok = true;
    for (int w = cid; w < a.total && ok; w += ncl) {
      const int split = w / tiles_mn;
      int kb0, nkb = kblocks_of(split, kb0);
      if (nkb == 0) continue;  // the epilogues write zeros without waiting
      if (!warp_wait(tempty0 + 8 * acc, aph ^ 1, &abort_sh, a.flag)) break;
      fence_after();
      const uint32_t td = tmem + acc * BN;
      for (int kb = 0; kb < nkb; kb++) {
        if (!warp_wait(full0 + 8 * s, ph, &abort_sh, a.flag)) { ok = false; break; }
        fence_after();
        const uint32_t sa = smem_u32(smem + s * STAGE2_BYTES), sb = sa + HALF_BYTES;
        const uint64_t ad = A_MN ? sdesc(sa, 8192, 1024) : sdesc(sa, 16, 1024);
        const uint64_t bd = B_MN ? sdesc(sb, 8192, 1024) : sdesc(sb, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < BK / 16; kk++) {
          const uint64_t da = (uint64_t)(A_MN ? kk * 128 : kk * 2);
          const uint64_t db = (uint64_t)(B_MN ? kk * 128 : kk * 2);
          mma_pair_e(td, ad + da, bd + db, ID, (kb > 0 || kk > 0) ? 1u : 0u);
        }
        commit_pair_both_e(empty0 + 8 * s);  // frees the stage in both CTAs
        if (++s == STAGES2) { s = 0; ph ^= 1; }
      }
      if (!ok) break;
      commit_pair_both_e(tfull0 + 8 * acc);  // accumulator ready in both CTAs
      if (++acc == 2) { acc = 0; aph ^= 1; }
    }
    commit_pair_e(drain);
    if (lane == 0) {
      const unsigned long long t0 = gtimer();
      while (!mbar_try(drain, 0) && gtimer() - t0 < WAIT_NS) {
      }
    }
    __syncwarp();
  } else if (warp >= 2) {
    // ------------------------------------ epilogue warps (each CTA, its rows)
    const int quarter = warp & 3;
    const int ew = warp - 2;
    const int c_lo = (ew / 4) * (BN / 2);
    float *stg = reinterpret_cast<float *>(smem + STAGES2 * STAGE2_BYTES) + ew * STG_BUFS * 32 * 32;
    int sb = 0;
    uint32_t rph = 0;
    const uint32_t rbar = rbar0 + 8 * ew;
    const uint32_t lead_tempty0 = cluster_addr(tempty0, 0);
    int acc = 0;
    uint32_t aph = 0;
    for (int w = cid; w < a.total; w += ncl) {
      const int split = w / tiles_mn, tile = w % tiles_mn;
      int mt, nt;
      tile_mn(a, tile, mt, nt);
      const int m0 = mt * 256 + 128 * (int)rank;
      const int n0 = nt * 256;
      int kb0, nkb = kblocks_of(split, kb0);
      const int row0 = m0 + quarter * 32;
      if (nkb == 0) {
        epilogue_tile(a, &tmC, &tmR, &tmU, rbar, rph, &abort_sh, 0, row0, n0, c_lo, split, true, stg,
                      sb);
        continue;
      }
      if (!warp_wait(tfull0 + 8 * acc, aph, &abort_sh, a.flag)) break;
      fence_after();
      const uint32_t tm = tmem + acc * BN + ((uint32_t)(quarter * 32) << 16);
      epilogue_tile(a, &tmC, &tmR, &tmU, rbar, rph, &abort_sh, tm, row0, n0, c_lo, split, false, stg,
                    sb);
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead_tempty0 + 8 * acc);
      if (++acc == 2) { acc = 0; aph ^= 1; }
    }
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    __syncwarp();
  }
  fence_before();
  __syncthreads();
  cluster_sync_all();  // no arrival may target a CTA that has left
  fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

}  // namespace tc

// ------------------------------------------------------------------ host side
struct TcPlan {
  PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  int num_sms = 148;
  const float *cos_t, *sin_t;
  int T, hd;
  int64_t rot_cols, hp;
  int *flag = nullptr;  // device flag word for time-outs (set by the owner)
  bool pairs = true;  // CTA-pair kernel for large shapes
  std::mutex mu;
  struct Key {
    const void *p;
    uint64_t d0, d1, s1, d2;
    uint32_t b0, b1, esz;
    bool operator==(const Key &o) const {
      return p == o.p && d0 == o.d0 && d1 == o.d1 && s1 == o.s1 && d2 == o.d2 && b0 == o.b0 &&
             b1 == o.b1 && esz == o.esz;
    }
  };
  struct KeyHash {
    size_t operator()(const Key &k) const {
      return std::hash<const void *>()(k.p) ^ (k.d0 * 1315423911u) ^ (k.d1 * 2654435761u) ^
             (k.s1 << 7) ^ ((uint64_t)k.b0 << 20) ^ ((uint64_t)k.b1 << 40) ^ (k.d2 << 13) ^
             ((uint64_t)k.esz << 52);
    }
  };
  std::unordered_map<Key, CUtensorMap, KeyHash> maps;

  // 2-D bf16 tensor map: inner dim d0 (contiguous), outer d1 with row
  // stride s1 elements; box b0 x b1; 128-byte swizzle; zero fill outside.
  bool map(const void *p, uint64_t d0, uint64_t d1, uint64_t s1, uint32_t b0, uint32_t b1,
           CUtensorMap *out) {
    Key k{p, d0, d1, s1, 1, b0, b1, 2};
    std::lock_guard<std::mutex> g(mu);
    auto it = maps.find(k);
    if (it != maps.end()) { *out = it->second; return true; }
    cuuint64_t dims[2] = {d0, d1};
    cuuint64_t strides[1] = {s1 * 2};
    cuuint32_t box[2] = {b0, b1};
    cuuint32_t es[2] = {1, 1};
    CUresult r = encode(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(p), dims,
                        strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    maps.emplace(k, *out);
    return true;
  }
  // Output map of C: bf16 (esz 2, box 64 x 32) or fp32 (esz 4, box 32 x 32)
  // over [d1 rows][d0 cols] with row stride s1 elements.  three_d adds a
  // third dimension of d2 slabs of d1 rows (split-K partial sums; always
  // three-dimensional, also for d2 = 1, because the kernel's partial-sum
  // store is), so the edge of one slab never spills into the next.
  // 128-byte swizzle (one box row = 128 bytes).
  bool map_out(const void *p, uint64_t d0, uint64_t d1, uint64_t s1, uint64_t d2, bool three_d,
               uint32_t esz, CUtensorMap *out) {
    const uint32_t b0 = esz == 2 ? 64 : 32;
    Key k{p, d0, d1, s1, three_d ? d2 + 1 : 0, b0, 32, esz};
    std::lock_guard<std::mutex> g(mu);
    auto it = maps.find(k);
    if (it != maps.end()) { *out = it->second; return true; }
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {s1 * esz, s1 * esz * d1};
    cuuint32_t box[3] = {b0, 32, 1};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = encode(out, esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                        three_d ? 3 : 2, const_cast<void *>(p), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    maps.emplace(k, *out);
    return true;
  }
};

TcPlan *tc_plan_create(DType dt, const float *cos_t, const float *sin_t, int T, int hd,
                       int64_t rot_cols, int64_t hp) {
  if (dt != DT_BF16) return nullptr;
  int dev = 0, major = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (major != 10) return nullptr;
  TcPlan *p = new TcPlan();
  cudaDriverEntryPointQueryResult q;
  void *fn = nullptr;
  if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                       &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn) {
    delete p;
    return nullptr;
  }
  p->encode = (PFN_cuTensorMapEncodeTiled_v12000)fn;
  cudaDeviceGetAttribute(&p->num_sms, cudaDevAttrMultiProcessorCount, dev);
  p->cos_t = cos_t; p->sin_t = sin_t; p->T = T; p->hd = hd; p->rot_cols = rot_cols; p->hp = hp;
  // the plan's device is current here: opt every variant in on it
  if (!smem_optin((const void *)tc::k_gemm_tc2<false, false>, tc::SMEM2_BYTES) ||
      !smem_optin((const void *)tc::k_gemm_tc2<false, true>, tc::SMEM2_BYTES) ||
      !smem_optin((const void *)tc::k_gemm_tc2<true, false>, tc::SMEM2_BYTES) ||
      !smem_optin((const void *)tc::k_gemm_tc2<true, true>, tc::SMEM2_BYTES) ||
      !smem_optin((const void *)tc::k_gemm_tc<false, false>, tc::SMEM_BYTES) ||
      !smem_optin((const void *)tc::k_gemm_tc<false, true>, tc::SMEM_BYTES) ||
      !smem_optin((const void *)tc::k_gemm_tc<true, false>, tc::SMEM_BYTES) ||
      !smem_optin((const void *)tc::k_gemm_tc<true, true>, tc::SMEM_BYTES)) {
    delete p;
    return nullptr;
  }
  return p;
}

// CTA pairs (256 x 256 tiles) once both sides span at least two tiles of
// the pair kernel: smaller problems keep the 128 x 256 tiles' parallelism.
bool tc_gemm_pairs(const TcPlan *p, int64_t M, int64_t N) {
  return p && p->pairs && M >= 512 && N >= 512;
}

void tc_plan_set_flag(TcPlan *p, int *flag) {
  if (p) p->flag = flag;
}

void tc_plan_destroy(TcPlan *p) { delete p; }

static bool al16(const void *p) { return ((uintptr_t)p & 15) == 0; }

bool tc_gemm(TcPlan *p, const GemmOperands &g, GemmOut out, void *C, int64_t ldc, const float *R,
             int64_t ldr, int splits, int epi, cudaStream_t s, void *U, int64_t ldu) {
  using namespace tc;
  if (!p || g.in != DT_BF16 || !p->flag) return false;
  if (g.M < 1 || g.N < 1 || g.K < 1) return false;
  if (!al16(g.A) || !al16(g.B) || !al16(C) || (g.lda * 2) % 16 || (g.ldb * 2) % 16) return false;
  if (out == OUT_ACT ? (ldc % 8) : (ldc % 4)) return false;
  if (out == OUT_ADD_F32 && (!R || !al16(R) || ldr % 4)) return false;
  if (epi == TC_EPI_ROPE && !(p->hd == 32 || p->hd == 64)) return false;
  if (epi != TC_EPI_NONE && epi != TC_EPI_ROPE && epi != TC_EPI_SWIGLU) return false;
  // SwiGLU: N = 2 hp columns in interleaved blocks of 128 (a then b), u is
  // [M][hp] bf16 with a 16-byte aligned row stride
  if (epi == TC_EPI_SWIGLU && (!U || !al16(U) || ldu % 8 || g.N % 128 || ldu < g.N / 2))
    return false;
  if (epi != TC_EPI_NONE && out != OUT_ACT) return false;
  // tensor maps: A as [rows][K] (K-major) or [K][M] (MN-major); same for B
  CUtensorMap ta, tb;
  bool ok = g.a_kmajor ? p->map(g.A, g.K, g.M, g.lda, 64, BM, &ta)
                       : p->map(g.A, g.M, g.K, g.lda, 64, 64, &ta);
  ok = ok && (g.b_kmajor ? p->map(g.B, g.K, g.N, g.ldb, 64, BN, &tb)
                         : p->map(g.B, g.N, g.K, g.ldb, 64, 64, &tb));
  if (!ok) return false;
  if (out != OUT_PARTIAL) splits = 1;
  // C leaves through bulk tensor stores; a residual R comes in through bulk
  // tensor loads of the same 32 x 32 fp32 boxes
  CUtensorMap tcm, trm;
  memset(&tcm, 0, sizeof(tcm));
  memset(&trm, 0, sizeof(trm));
  if (!p->map_out(C, g.N, g.M, ldc, max(1, splits), out == OUT_PARTIAL, out == OUT_ACT ? 2 : 4,
                  &tcm))
    return false;
  if (out == OUT_ADD_F32 && !p->map_out(R, g.N, g.M, ldr, 1, false, 4, &trm)) return false;
  CUtensorMap tum;
  memset(&tum, 0, sizeof(tum));
  if (epi == TC_EPI_SWIGLU && !p->map_out(U, g.N / 2, g.M, ldu, 1, false, 2, &tum)) return false;
  Args a{};
  a.M = g.M; a.N = g.N; a.K = g.K;
  a.tiles_m = (g.M + BM - 1) / BM;
  a.tiles_n = (g.N + BN - 1) / BN;
  a.splits = max(1, splits);
  int kc = (g.K + a.splits - 1) / a.splits;
  a.kchunk = ((kc + BK - 1) / BK) * BK;
  a.total = a.tiles_m * a.tiles_n * a.splits;
  a.nfast = a.tiles_n <= 8;
  a.out = out; a.epi = epi; a.C = C; a.ldc = ldc; a.R = R; a.ldr = ldr;
  a.cos_t = p->cos_t; a.sin_t = p->sin_t; a.T = p->T; a.hd = p->hd; a.rot_cols = (int)p->rot_cols;
  a.flag = p->flag;
  bool amn = !g.a_kmajor, bmn = !g.b_kmajor;
  if (tc_gemm_pairs(p, g.M, g.N)) {
    // CTA pairs: B boxes of 128 rows (K-major), tiles of 256 x 256
    if (g.b_kmajor && !p->map(g.B, g.K, g.N, g.ldb, 64, 128, &tb)) return false;
    a.tiles_m = (g.M + 255) / 256;
    a.tiles_n = (g.N + BN - 1) / BN;
    a.total = a.tiles_m * a.tiles_n * a.splits;
    a.nfast = a.tiles_n <= 8;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * (unsigned)min(a.total, p->num_sms / 2), 1, 1);
    cfg.blockDim = dim3(NTHREADS, 1, 1);
    cfg.dynamicSmemBytes = SMEM2_BYTES;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (!amn && !bmn) e = cudaLaunchKernelEx(&cfg, k_gemm_tc2<false, false>, ta, tb, tcm, trm, tum, a);
    else if (!amn && bmn) e = cudaLaunchKernelEx(&cfg, k_gemm_tc2<false, true>, ta, tb, tcm, trm, tum, a);
    else if (amn && !bmn) e = cudaLaunchKernelEx(&cfg, k_gemm_tc2<true, false>, ta, tb, tcm, trm, tum, a);
    else e = cudaLaunchKernelEx(&cfg, k_gemm_tc2<true, true>, ta, tb, tcm, trm, tum, a);
    count_launch();
    return e == cudaSuccess;
  }
  int grid = min(a.total, p->num_sms);
  if (!amn && !bmn) k_gemm_tc<false, false><<<grid, NTHREADS, SMEM_BYTES, s>>>(ta, tb, tcm, trm, tum, a);
  else if (!amn && bmn) k_gemm_tc<false, true><<<grid, NTHREADS, SMEM_BYTES, s>>>(ta, tb, tcm, trm, tum, a);
  else if (amn && !bmn) k_gemm_tc<true, false><<<grid, NTHREADS, SMEM_BYTES, s>>>(ta, tb, tcm, trm, tum, a);
  else k_gemm_tc<true, true><<<grid, NTHREADS, SMEM_BYTES, s>>>(ta, tb, tcm, trm, tum, a);
  count_launch();
  return true;
}

void attention_fwd(TcPlan *p, const void *qkv, void *o, float *lse, DType dt, int B, int T, int H,
                   int Hkv, int hd, cudaStream_t s) {
  if (p && p->flag && attn_tc_covers(dt, hd, T) &&
      attn_fwd_tc(qkv, o, lse, B, T, H, Hkv, hd, p->flag, s))
    return;
  if (attn_mma_covers(dt, hd)) attn_fwd_mma(qkv, o, lse, B, T, H, Hkv, hd, s);
  else attn_fwd_simt(qkv, o, lse, dt, B, T, H, Hkv, hd, s);
}
void attention_bwd(TcPlan *p, const void *qkv, const void *o, const void *dout, const float *lse,
                   float *Dbuf, void *dqkv, DType dt, int B, int T, int H, int Hkv, int hd,
                   const float *cos_t, const float *sin_t, cudaStream_t s) {
  if (p && p->flag && attn_tc_covers(dt, hd, T) &&
      attn_bwd_tc(qkv, o, dout, lse, Dbuf, dqkv, B, T, H, Hkv, hd, cos_t, sin_t, p->flag, s))
    return;
  if (attn_mma_covers(dt, hd)) {
    attn_bwd_mma(qkv, o, dout, lse, Dbuf, dqkv, B, T, H, Hkv, hd, cos_t, sin_t, s);
    return;
  }
  attn_bwd_simt(qkv, o, dout, lse, Dbuf, dqkv, dt, B, T, H, Hkv, hd, s);
  if (cos_t)
    rope_apply(dqkv, dt, cos_t, sin_t, (int64_t)B * T, T, (H + Hkv) * hd,
               (int64_t)(H + 2 * Hkv) * hd, hd, -1, s);
}

}  // namespace llm
