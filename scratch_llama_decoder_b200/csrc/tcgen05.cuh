// Inline-PTX helpers for sm_100a: mbarriers with bounded waits, TMA tile
// loads, tcgen05 MMA / commit / TMEM loads and stores, and the shared-memory
// matrix descriptors of the tensor cores.  Shared by the GEMM and attention
// kernels.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace llm {
namespace tc {

constexpr unsigned long long WAIT_NS = 2000000000ull;  // 2 s bound on any wait

LLM_DEV uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
LLM_DEV unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
LLM_DEV void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
LLM_DEV bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait on the phase of `parity`; false (and FLAG_TIMEOUT) on time-out
// or when another role of this CTA already gave up.
LLM_DEV bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag, int *gflag) {
  if (mbar_try(bar, parity)) return true;
  unsigned long long t0 = gtimer();
  for (uint32_t it = 1;; it++) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 255) == 0) {
      if (*abort_flag) return false;
      if (gtimer() - t0 > WAIT_NS) {
        *abort_flag = 1;
        atomicOr(gflag, FLAG_TIMEOUT);
        return false;
      }
    }
  }
}
// Bounded wait used only on the way out (the copies / MMAs of this thread).
LLM_DEV void drain_wait(uint32_t bar, uint32_t parity) {
  const unsigned long long t0 = gtimer();
  while (!mbar_try(bar, parity) && gtimer() - t0 < WAIT_NS) {
  }
}
LLM_DEV void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
LLM_DEV void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
LLM_DEV void tma_load_2d(uint32_t dst, const CUtensorMap *map, int c0, int c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"((uint64_t)map), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
LLM_DEV void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
LLM_DEV void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor (UMMA): start address, leading/stride byte
// offsets (16-byte units), descriptor version 1, 128-byte swizzle (mode 2).
LLM_DEV uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}
LLM_DEV void mma_bf16(uint32_t tmem_d, uint64_t ad, uint64_t bd, uint32_t id, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(ad), "l"(bd), "r"(id), "r"(acc)
      : "memory");
}
LLM_DEV void mma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}
LLM_DEV void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; i++) v[i] = __uint_as_float(r[i]);
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B,
// per-operand major-ness, N>>3 and M>>4.
__host__ __device__ constexpr uint32_t idesc_mn(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
         ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
LLM_DEV uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}
LLM_DEV void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]),
      "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]),
      "f"(v[15]), "f"(v[16]), "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]),
      "f"(v[22]), "f"(v[23]), "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]),
      "f"(v[29]), "f"(v[30]), "f"(v[31])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// 2^x by the SFU's single ex2.approx instruction (flushes denormals; relative
// error of a few ulp) -- the softmax exponent.
LLM_DEV float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 2^x for a pair on the FMA pipe instead of the SFU, so that a softmax loop
// can split its exponentials between the two units.  Range reduction in the
// style of Cody and Waite (Software Manual for the Elementary Functions,
// 1980): x = k + f with k = round(x) taken by adding 1.5 * 2^23 (the rounded
// sum holds k in its low mantissa bits), f in [-1/2, 1/2]; 2^f by the degree-3
// polynomial that minimises the maximum relative error on that interval
// (Remez exchange, fitted by exp2_poly_fit.py beside this file: 7.5e-5, well
// under half a bf16 ulp); 2^k applied by adding k to the exponent field.
// Domain x <= 126 (the softmax loops pass x <= 8); x is clamped below at
// -126, where the result is a tiny positive number (under 2^-125) rather
// than 0.
constexpr float EXP2_C0 = 0.9999280571937561f, EXP2_C1 = 0.6932609677314758f,
                EXP2_C2 = 0.2426111251115799f, EXP2_C3 = 0.0551716685295105f;
LLM_DEV float2 exp2_poly2(float2 x) {
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 t = __fadd2_rn(x, make_float2(12582912.f, 12582912.f));
  const float2 k = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));
  const float2 f = __ffma2_rn(k, make_float2(-1.f, -1.f), x);
  float2 p = __ffma2_rn(make_float2(EXP2_C3, EXP2_C3), f, make_float2(EXP2_C2, EXP2_C2));
  p = __ffma2_rn(p, f, make_float2(EXP2_C1, EXP2_C1));
  p = __ffma2_rn(p, f, make_float2(EXP2_C0, EXP2_C0));
  // t's bit pattern is that of 1.5 * 2^23 plus k: shifted left by 23 bits,
  // only k << 23 remains (mod 2^32), the exponent-field increment
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}
// Whether pair `i` (of the 16 pairs of a 32-score chunk) of a softmax loop
// takes the polynomial: 5 of 16, spread over the chunk, which balanced the
// SFU against the FMA pipe and the issue slots best in a measured sweep.
LLM_DEV constexpr bool exp2_on_fma(int i) { return ((i & 15) * 5) % 16 < 5; }
// 2^x for a pair: the polynomial or the SFU, by the pair's index.
LLM_DEV float2 exp2_pair(float2 x, int i) {
  return exp2_on_fma(i) ? exp2_poly2(x) : make_float2(ex2(x.x), ex2(x.y));
}
// Work item of a persistent kernel in scheduling round r: the G CTAs take
// the items (ordered heaviest first) in a snake, CTA c taking item r G + c in
// even rounds and r G + G - 1 - c in odd ones, which evens out the summed
// weights of a CTA's items when the weights fall in steps.
LLM_DEV int sched_item(int r, int G, int c) { return r * G + ((r & 1) ? G - 1 - c : c); }
// Work item -> (weight class z, pair p) for nz classes (z = 0 heaviest) of np
// pairs: classes in bands of 4, pair-major inside a band, so that the CTAs
// that work at one time on a pair's classes stream the same tiles and share
// them in L2, while the weights still fall band by band for the snake.
LLM_DEV void band_item(int item, int nz, int np, int &z, int &p) {
  constexpr int BW = 4;
  const int band = item / (BW * np);
  const int rem = item - band * BW * np;
  const int nbb = min(BW, nz - band * BW);
  p = rem / nbb;
  z = band * BW + rem - p * nbb;
}
// max(a, b, c) in one instruction.
LLM_DEV float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// tcgen05.mma with the A operand in TMEM (bf16 pairs packed in 32-bit
// columns: K 16 = 8 columns) and B in shared memory.
LLM_DEV void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bd, uint32_t id, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bd), "r"(id), "r"(acc)
      : "memory");
}
LLM_DEV void tmem_st16(uint32_t taddr, const uint32_t (&w)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16};" ::"r"(taddr),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]),
      "r"(w[8]), "r"(w[9]), "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]),
      "r"(w[15])
      : "memory");
}

// Two 32-column TMEM loads in flight, one wait.
LLM_DEV void tmem_ld64(uint32_t taddr, float (&v)[64]) {
  uint32_t r[64];
#define LD32(OFF)                                                                                \
  asm volatile(                                                                                  \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"  \
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"        \
      : "=r"(r[OFF + 0]), "=r"(r[OFF + 1]), "=r"(r[OFF + 2]), "=r"(r[OFF + 3]),                \
        "=r"(r[OFF + 4]), "=r"(r[OFF + 5]), "=r"(r[OFF + 6]), "=r"(r[OFF + 7]),                \
        "=r"(r[OFF + 8]), "=r"(r[OFF + 9]), "=r"(r[OFF + 10]), "=r"(r[OFF + 11]),              \
        "=r"(r[OFF + 12]), "=r"(r[OFF + 13]), "=r"(r[OFF + 14]), "=r"(r[OFF + 15]),            \
        "=r"(r[OFF + 16]), "=r"(r[OFF + 17]), "=r"(r[OFF + 18]), "=r"(r[OFF + 19]),            \
        "=r"(r[OFF + 20]), "=r"(r[OFF + 21]), "=r"(r[OFF + 22]), "=r"(r[OFF + 23]),            \
        "=r"(r[OFF + 24]), "=r"(r[OFF + 25]), "=r"(r[OFF + 26]), "=r"(r[OFF + 27]),            \
        "=r"(r[OFF + 28]), "=r"(r[OFF + 29]), "=r"(r[OFF + 30]), "=r"(r[OFF + 31])             \
      : "r"(taddr + OFF))
  LD32(0);
  LD32(32);
#undef LD32
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 64; i++) v[i] = __uint_as_float(r[i]);
}
LLM_DEV void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; i++) v[i] = __uint_as_float(r[i]);
}
// Issue from a converged warp: every lane executes the call with warp-uniform
// operands, and the lane that elect.sync picks (the same lane each time for a
// full warp) issues the instruction.  Back-to-back tcgen05.mma issued this way
// measured ~127 cycles each (M 128, any N up to 256), against 160-190 from a
// lone lane inside a divergent branch.
LLM_DEV void mma_bf16_e(uint32_t tmem_d, uint64_t ad, uint64_t bd, uint32_t id, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p, e;\n setp.ne.b32 p, %4, 0;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(ad), "l"(bd), "r"(id), "r"(acc)
      : "memory");
}
LLM_DEV void mma_ts_e(uint32_t d_tmem, uint32_t a_tmem, uint64_t bd, uint32_t id, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p, e;\n setp.ne.b32 p, %4, 0;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bd), "r"(id), "r"(acc)
      : "memory");
}
LLM_DEV void mma_commit_e(uint32_t bar) {
  asm volatile(
      "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n" ::"r"(
          bar)
      : "memory");
}
LLM_DEV void tma_load_2d_e(uint32_t dst, const CUtensorMap *map, int c0, int c1, uint32_t bar) {
  asm volatile(
      "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
      " @e cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];\n}\n" ::"r"(dst),
      "l"((uint64_t)map), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
LLM_DEV void mbar_arrive_expect_tx_e(uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
      " @e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n}\n" ::"r"(bar),
      "r"(bytes)
      : "memory");
}
// Warp-wide bounded wait: every lane polls (the warp stays converged, each
// lane acquires the phase itself); lane 0 alone checks the time and abort
// flag every 256 polls and the warp leaves together.  A lone polling lane with
// a broadcast afterwards measured 1.4-1.8x slower in the MMA-issuing warps.
LLM_DEV bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort_sh, int *gflag) {
  if (__all_sync(0xffffffffu, mbar_try(bar, parity))) return true;
  const unsigned long long t0 = gtimer();
  for (uint32_t it = 1;; it++) {
    if (__all_sync(0xffffffffu, mbar_try(bar, parity))) return true;
    if ((it & 255) == 0) {
      int stop = 0;
      if ((threadIdx.x & 31) == 0) {
        if (*abort_sh) {
          stop = 1;
        } else if (gtimer() - t0 > WAIT_NS) {
          stop = 1;
          *abort_sh = 1;
          atomicOr(gflag, FLAG_TIMEOUT);
        }
      }
      if (__shfl_sync(0xffffffffu, stop, 0)) return false;
    }
  }
}
// N consecutive TMEM columns of this thread's lane (N = 8, 16, 32 or 64),
// one wait for all of them.
template <int N>
LLM_DEV void tmem_ldn(uint32_t taddr, float (&v)[N]) {
  if constexpr (N == 64) {
    tmem_ld64(taddr, v);
  } else if constexpr (N == 32) {
    tmem_ld32(taddr, v);
  } else if constexpr (N == 16) {
    tmem_ld16(taddr, v);
  } else {
    static_assert(N == 8, "tmem_ldn: 8, 16, 32 or 64 columns");
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 8; i++) v[i] = __uint_as_float(r[i]);
  }
}
// N packed words (N = 8 or 16) into consecutive TMEM columns, no wait.
template <int N>
LLM_DEV void tmem_stn(uint32_t taddr, const uint32_t *w) {
  if constexpr (N == 16) {
    tmem_st16(taddr, *reinterpret_cast<const uint32_t (*)[16]>(w));
  } else {
    static_assert(N == 8, "tmem_stn: 8 or 16 columns");
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(
                     taddr),
                 "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]),
                 "r"(w[7])
                 : "memory");
  }
}
LLM_DEV void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Host: tensor map over a row-major bf16 matrix [rows, cols] (row stride ld
// elements) with a box of 64 columns x box_rows rows and 128-byte swizzle;
// rows past the end read as zero.  False when the driver entry point is
// missing or the encoder rejects the arguments (base or stride not 16-byte
// aligned).
inline bool tile_map_bf16(CUtensorMap *map, const void *base, int64_t cols, int64_t rows,
                          int64_t ld, int box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = [] {
    cudaDriverEntryPointQueryResult q;
    void *fn = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
    return (PFN_cuTensorMapEncodeTiled_v12000)fn;
  }();
  if (!encode || ((uintptr_t)base & 15) || (ld * 2) % 16) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor map over a [batches, rows, cols] bf16 array (row stride ld
// elements, batch stride rows * ld) with a box of 64 columns x box_rows rows
// x 1 batch and 128-byte swizzle: a bulk store through it clips at the end of
// each batch's rows, not only at the end of the array.
inline bool tile_map_bf16_3d(CUtensorMap *map, const void *base, int64_t cols, int64_t rows,
                             int64_t batches, int64_t ld, int box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = [] {
    cudaDriverEntryPointQueryResult q;
    void *fn = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
    return (PFN_cuTensorMapEncodeTiled_v12000)fn;
  }();
  if (!encode || ((uintptr_t)base & 15) || (ld * 2) % 16) return false;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)batches};
  cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)(ld * rows * 2)};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Bulk tensor store of a box from shared memory (3-D map), its commit, and
// the wait until every committed store of this thread has read its source.
LLM_DEV void tma_store_3d(const CUtensorMap *map, uint32_t src, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
          (uint64_t)map),
      "r"(x), "r"(y), "r"(z), "r"(src)
      : "memory");
}
// Bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned)
// from global to shared memory, completing on `bar`'s transaction count.
LLM_DEV void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
LLM_DEV void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
LLM_DEV void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
LLM_DEV void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
LLM_DEV void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

}  // namespace tc
}  // namespace llm
