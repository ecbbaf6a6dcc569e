// Float32 GEMM on the 5th-generation tensor cores in split precision
// (3xTF32): each operand x is split into hi = x rounded to tf32 (10-bit
// mantissa) and lo = x - hi (exact in float32), and
//     A.B^T ~ Ahi.Bhi^T + Ahi.Blo^T + Alo.Bhi^T
// with float32 accumulation in TMEM (the dropped Alo.Blo^T term and the tf32
// rounding of lo leave a relative error of about 2^-21 per product, against
// 2^-11 for a single tf32 product).  Used by the float32 configurations,
// whose parity gates (1e-4 logits, 1e-3 gradients) a single tf32 pass cannot
// meet.
//
// A split pass (k_tf32_split) writes hi and lo of each operand K-major,
// [rows][Kp] with Kp = K rounded up to 32 (zeros past K), transposing the
// MN-major operands through shared memory.  The GEMM kernel: persistent, one
// CTA per SM over the 128 x 128 output tiles (and K splits), warp 0 the TMA
// producer (Ahi, Alo,
// Bhi, Blo tiles of 128 rows x 32 floats, 128-byte swizzle, a 3-deep ring),
// warp 1 allocates TMEM and issues per K step of 8 the three products
// (tcgen05.mma kind::tf32, M 128, N 128, K 8), warps 2-5 read the
// accumulator rows from TMEM and write them out (float32, plus a residual,
// or a split's partial slab).  The accumulation runs in chunks of 16 K blocks
// in two TMEM buffers, each finished chunk added into float32 registers by the
// epilogue warps, which bounds the tensor core's own accumulation chains (and,
// over a CTA's items, lets one tile's stores overlap the next tile's
// products).  Every wait is bounded (2 s, FLAG_TIMEOUT).
#include "common.cuh"
#include "tcgen05.cuh"

namespace llm {
namespace tf32g {

using namespace tc;

constexpr int BM = 128, BN = 128, BKF = 32;           // tile; K block in floats (128 bytes)
constexpr int TILE = 128 * BKF * 4;                   // 16 KB
constexpr int STAGES = 3;
constexpr int STAGE_BYTES = 4 * TILE;                 // Ahi, Alo, Bhi, Blo
constexpr int SMEM = STAGES * STAGE_BYTES + 1024 + 256;
constexpr int NTHREADS = 6 * 32;
// The tensor core's float32 accumulation drops low bits on every addition,
// so no TMEM accumulation runs longer than CH K blocks (K = 512): chunk c
// accumulates in TMEM buffer c % 2 and the epilogue warps add each finished
// chunk into float32 registers (round to nearest) while the next chunk runs.
constexpr int CH = 16;
constexpr int TMEM_COLS = 256;
// kind::tf32 instruction descriptor: f32 accumulator (bits 4-5 = 1), A and B
// tf32 (bits 7-9 and 10-12 = 2), both K-major, N >> 3 at bit 17, M >> 4 at 24.
constexpr uint32_t IDESC = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(BN >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);

// Issued from a converged warp; the lane elect.sync picks issues it.
LLM_DEV void mma_tf32_e(uint32_t d_tmem, uint64_t ad, uint64_t bd, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p, e;\n setp.ne.b32 p, %4, 0;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(ad), "l"(bd), "r"(IDESC), "r"(acc)
      : "memory");
}

// x rounded to the nearest tf32 (ties away from zero); finite x.
LLM_DEV float tf32_round(float x) {
  return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}

// hi, lo of X's element (r, k) at [r * Kp + k]; X element (r, k) is
// X[r * ld + k] (K-major) or X[k * ld + r]; zeros for k >= K (and r >= rows
// is not written).  Block 32 x 8 threads over a 32 x 32 tile.
template <bool KMAJOR>
__global__ void __launch_bounds__(256) k_tf32_split(const float *__restrict__ X, int64_t ld,
                                                    int rows, int K, int Kp,
                                                    float *__restrict__ hi,
                                                    float *__restrict__ lo) {
  __shared__ float t[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int k0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  if (KMAJOR) {
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const int r = r0 + ty + 8 * i, k = k0 + tx;
      if (r < rows) {
        const float x = k < K ? X[(int64_t)r * ld + k] : 0.f;
        const float h = tf32_round(x);
        hi[(int64_t)r * Kp + k] = h;
        lo[(int64_t)r * Kp + k] = x - h;
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const int k = k0 + ty + 8 * i, r = r0 + tx;
      t[ty + 8 * i][tx] = (k < K && r < rows) ? X[(int64_t)k * ld + r] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const int r = r0 + ty + 8 * i, k = k0 + tx;
      if (r < rows) {
        const float x = t[tx][ty + 8 * i];
        const float h = tf32_round(x);
        hi[(int64_t)r * Kp + k] = h;
        lo[(int64_t)r * Kp + k] = x - h;
      }
    }
  }
}

// The K-major split as a grid-stride pass, one thread per 4 consecutive
// elements of a row (Kp a multiple of 32, so a row is whole float4 groups):
// 16-byte loads when X is 16-byte aligned with ld a multiple of 4, and 16-byte
// stores of hi and lo (the tiled kernel above moved 4 KiB per 256-thread
// block, which left it launch-bound).
__global__ void __launch_bounds__(256) k_tf32_split_rows(const float *__restrict__ X, int64_t ld,
                                                         int rows, int K, int Kp, bool vec,
                                                         float *__restrict__ hi,
                                                         float *__restrict__ lo) {
  const uint32_t q = (uint32_t)Kp / 4, n = (uint32_t)rows * q;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const uint32_t r = i / q;
    const int k = 4 * (int)(i - r * q);
    const float *xr = X + (int64_t)r * ld;
    float x[4];
    if (vec && k + 4 <= K) {
      const float4 v = *reinterpret_cast<const float4 *>(xr + k);
      x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; e++) x[e] = k + e < K ? xr[k + e] : 0.f;
    }
    float h[4], l[4];
#pragma unroll
    for (int e = 0; e < 4; e++) {
      h[e] = tf32_round(x[e]);
      l[e] = x[e] - h[e];
    }
    *reinterpret_cast<float4 *>(hi + (int64_t)r * Kp + k) = make_float4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<float4 *>(lo + (int64_t)r * Kp + k) = make_float4(l[0], l[1], l[2], l[3]);
  }
}

struct Args {
  int M, N, Kp, kchunk;  // kchunk: K floats per split (a multiple of 32)
  int tiles_n, tiles, splits;  // work items: tiles x splits, tile = (row block, column block)
  int out;               // GemmOut
  float *C;
  int64_t ldc;
  const float *R;
  int64_t ldr;
  bool vec;              // 16-byte stores (C, R and their strides aligned)
  int *flag;
};

// Persistent: gridDim.x CTAs take the work items (tile, split) round-robin.
// The ring stages and the TMEM chunk buffers are counted over all of a CTA's
// items, so an item's stores overlap the next item's products.
__global__ void __launch_bounds__(NTHREADS, 1)
    k_gemm_tf32(const __grid_constant__ CUtensorMap tAh, const __grid_constant__ CUtensorMap tAl,
                const __grid_constant__ CUtensorMap tBh, const __grid_constant__ CUtensorMap tBl,
                const Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t *bars = (uint64_t *)(smem + STAGES * STAGE_BYTES);
  __shared__ uint32_t tmem_sh;
  __shared__ volatile int abort_sh;
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const uint32_t full0 = smem_u32(bars), empty0 = full0 + 8 * STAGES,
                 tfull = empty0 + 8 * STAGES,  // [2]: chunk of the buffer accumulated
                 tempty = tfull + 16,          // [2]: chunk of the buffer read out
                 drain = tempty + 16;
  const int items = a.tiles * a.splits;
  // item -> output tile origin and the split's K blocks
  auto item_of = [&](int w, int &m0, int &n0, int &kf0, int &nkb) {
    const int tile = w % a.tiles, split = w / a.tiles;
    m0 = (tile / a.tiles_n) * BM;
    n0 = (tile % a.tiles_n) * BN;
    kf0 = split * a.kchunk;
    const int kf1 = min(a.Kp, kf0 + a.kchunk);
    nkb = max(0, (kf1 - kf0) / BKF);
  };

  if (threadIdx.x == 0) {
    abort_sh = 0;
    for (int s = 0; s < STAGES; s++) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(tfull + 8 * b, 1);
      mbar_init(tempty + 8 * b, 4);  // the four epilogue warps
    }
    mbar_init(drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tmem_sh)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = tmem_sh;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    int gk = 0;  // K blocks issued over all items
    bool ok = true;
    for (int w = blockIdx.x; w < items && ok; w += gridDim.x) {
      int m0, n0, kf0, nkb;
      item_of(w, m0, n0, kf0, nkb);
      for (int kb = 0; kb < nkb; kb++) {
        const int s = gk % STAGES;
        const uint32_t ph = (gk / STAGES) & 1;
        if (!warp_wait(empty0 + 8 * s, ph ^ 1, &abort_sh, a.flag)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          const uint32_t bar = full0 + 8 * s;
          uint8_t *st = smem + s * STAGE_BYTES;
          const int kx = kf0 + kb * BKF;
          mbar_arrive_expect_tx(bar, STAGE_BYTES);
          tma_load_2d(smem_u32(st), &tAh, kx, m0, bar);
          tma_load_2d(smem_u32(st + TILE), &tAl, kx, m0, bar);
          tma_load_2d(smem_u32(st + 2 * TILE), &tBh, kx, n0, bar);
          tma_load_2d(smem_u32(st + 3 * TILE), &tBl, kx, n0, bar);
        }
        gk++;
      }
    }
    if (lane == 0)
      for (int i = max(0, gk - STAGES); i < gk; i++)
        drain_wait(full0 + 8 * (i % STAGES), (i / STAGES) & 1);
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------- MMA issuer (whole warp, elected)
    bool ok = true;
    int gk = 0, gc = 0;  // K blocks and TMEM chunks over all items
    for (int w = blockIdx.x; w < items && ok; w += gridDim.x) {
      int m0, n0, kf0, nkb;
      item_of(w, m0, n0, kf0, nkb);
      for (int kb = 0; kb < nkb && ok; kb++, gk++) {
        const int s = gk % STAGES;
        const uint32_t ph = (gk / STAGES) & 1;
        if (kb % CH == 0) {
          // a buffer is reused once the epilogue has read its previous chunk
          if (gc >= 2 && !warp_wait(tempty + 8 * (gc & 1), ((gc >> 1) - 1) & 1, &abort_sh,
                                    a.flag)) {
            ok = false;
            break;
          }
        }
        if (!warp_wait(full0 + 8 * s, ph, &abort_sh, a.flag)) {
          ok = false;
          break;
        }
        fence_after();
        uint8_t *st = smem + s * STAGE_BYTES;
        const uint64_t ah = sdesc(smem_u32(st), 16, 1024), al = sdesc(smem_u32(st + TILE), 16, 1024);
        const uint64_t bh = sdesc(smem_u32(st + 2 * TILE), 16, 1024),
                       bl = sdesc(smem_u32(st + 3 * TILE), 16, 1024);
        const uint32_t acc = tmem + 128 * (gc & 1);
#pragma unroll
        for (int kk = 0; kk < BKF / 8; kk++) {  // K steps of 8 floats = 32 bytes
          const uint64_t o = (uint64_t)(kk * 2);
          mma_tf32_e(acc, ah + o, bh + o, (kb % CH > 0 || kk > 0) ? 1u : 0u);
          mma_tf32_e(acc, ah + o, bl + o, 1u);
          mma_tf32_e(acc, al + o, bh + o, 1u);
        }
        mma_commit_e(empty0 + 8 * s);
        if (kb % CH == CH - 1 || kb == nkb - 1) {
          mma_commit_e(tfull + 8 * (gc & 1));
          gc++;
        }
      }
    }
    mma_commit_e(drain);
    if (lane == 0) drain_wait(drain, 0);
    __syncwarp();
  } else {
    // --------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes 32 quarter .. 32 quarter + 31
    const uint32_t row_t = tmem + ((uint32_t)(quarter * 32) << 16);
    bool ok = true;
    int gc = 0;
    for (int w = blockIdx.x; w < items && ok; w += gridDim.x) {
      int m0, n0, kf0, nkb;
      item_of(w, m0, n0, kf0, nkb);
      const int m = m0 + quarter * 32 + lane, split = w / a.tiles;
      float acc[BN];
#pragma unroll
      for (int i = 0; i < BN; i++) acc[i] = 0.f;
      const int nch = (nkb + CH - 1) / CH;
      for (int ci = 0; ci < nch; ci++, gc++) {
        const int buf = gc & 1;
        if (!warp_wait(tfull + 8 * buf, (gc >> 1) & 1, &abort_sh, a.flag)) {
          ok = false;
          break;
        }
        fence_after();
#pragma unroll
        for (int c0 = 0; c0 < BN; c0 += 32) {
          float v[32];
          tmem_ldn<32>(row_t + 128 * buf + c0, v);
#pragma unroll
          for (int i = 0; i < 32; i++) acc[c0 + i] += v[i];
        }
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty + 8 * buf);
      }
      if (!ok || m >= a.M) continue;
      float *crow = a.C + (a.out == OUT_PARTIAL ? (int64_t)split * a.M * a.ldc : 0) +
                    (int64_t)m * a.ldc;
      const float *rrow = a.R ? a.R + (int64_t)m * a.ldr : nullptr;
      if (a.vec && n0 + BN <= a.N) {
#pragma unroll
        for (int i = 0; i < BN; i += 4) {
          float4 v = make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]);
          if (a.out == OUT_ADD_F32) {
            const float4 q = *reinterpret_cast<const float4 *>(rrow + n0 + i);
            v.x += q.x; v.y += q.y; v.z += q.z; v.w += q.w;
          }
          *reinterpret_cast<float4 *>(crow + n0 + i) = v;
        }
      } else {
#pragma unroll
        for (int i = 0; i < BN; i++)
          if (n0 + i < a.N) crow[n0 + i] = a.out == OUT_ADD_F32 ? rrow[n0 + i] + acc[i] : acc[i];
      }
    }
  }
  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(TMEM_COLS)
                 : "memory");
}

// Tensor map over a [rows][Kp] float32 array, box 32 floats x 128 rows,
// 128-byte swizzle.
static bool tile_map_f32(CUtensorMap *map, const float *base, int64_t Kp, int64_t rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = [] {
    cudaDriverEntryPointQueryResult q;
    void *fn = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
    return (PFN_cuTensorMapEncodeTiled_v12000)fn;
  }();
  if (!encode || ((uintptr_t)base & 15) || (Kp * 4) % 16) return false;
  cuuint64_t dims[2] = {(cuuint64_t)Kp, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)Kp * 4};
  cuuint32_t box[2] = {BKF, 128};
  cuuint32_t es[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(base), dims, strides,
                box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

static void split(const float *X, int64_t ld, bool kmajor, int rows, int K, int Kp, float *hi,
                  float *lo, cudaStream_t s) {
  dim3 grid((unsigned)(Kp / 32), (unsigned)((rows + 31) / 32));
  if (kmajor && (int64_t)rows * (Kp / 4) < (int64_t(1) << 31)) {
    const bool vec = ((uintptr_t)X & 15) == 0 && ld % 4 == 0;
    const int64_t groups = (int64_t)rows * (Kp / 4);
    const unsigned g1 = (unsigned)std::min<int64_t>((groups + 255) / 256, 148 * 16);
    k_tf32_split_rows<<<g1, 256, 0, s>>>(X, ld, rows, K, Kp, vec, hi, lo);
  } else if (kmajor) {
    k_tf32_split<true><<<grid, 256, 0, s>>>(X, ld, rows, K, Kp, hi, lo);
  } else {
    k_tf32_split<false><<<grid, 256, 0, s>>>(X, ld, rows, K, Kp, hi, lo);
  }
  count_launch();
}

}  // namespace tf32g

int64_t gemm_tf32_scratch_floats(int64_t M, int64_t N, int64_t K) {
  const int64_t Kp = (K + 31) / 32 * 32;
  return 2 * (M + N) * Kp;
}

bool gemm_tf32(const GemmOperands &g, GemmOut out, void *C, int64_t ldc, const float *R,
               int64_t ldr, int splits, float *scratch, int64_t scratch_floats, int *flag,
               cudaStream_t s) {
  using namespace tf32g;
  if (g.in != DT_F32 || !scratch || !flag || g.M < 1 || g.N < 1 || g.K < 1) return false;
  if (gemm_tf32_scratch_floats(g.M, g.N, g.K) > scratch_floats) return false;
  if (((uintptr_t)scratch & 15) != 0) return false;
  if (!smem_optin((const void *)k_gemm_tf32, SMEM)) return false;
  const int Kp = (g.K + 31) / 32 * 32;
  float *ah = scratch, *al = ah + (int64_t)g.M * Kp, *bh = al + (int64_t)g.M * Kp,
        *bl = bh + (int64_t)g.N * Kp;
  CUtensorMap tAh, tAl, tBh, tBl;
  if (!tile_map_f32(&tAh, ah, Kp, g.M) || !tile_map_f32(&tAl, al, Kp, g.M) ||
      !tile_map_f32(&tBh, bh, Kp, g.N) || !tile_map_f32(&tBl, bl, Kp, g.N))
    return false;
  split((const float *)g.A, g.lda, g.a_kmajor, g.M, g.K, Kp, ah, al, s);
  split((const float *)g.B, g.ldb, g.b_kmajor, g.N, g.K, Kp, bh, bl, s);
  Args a{};
  a.M = g.M; a.N = g.N; a.Kp = Kp;
  if (out != OUT_PARTIAL) splits = 1;
  splits = std::max(1, splits);
  int kc = (Kp + splits - 1) / splits;
  a.kchunk = (kc + BKF - 1) / BKF * BKF;
  a.out = out; a.C = (float *)C; a.ldc = ldc; a.R = R; a.ldr = ldr; a.flag = flag;
  a.vec = ((uintptr_t)C & 15) == 0 && ldc % 4 == 0 &&
          (out != OUT_ADD_F32 || (((uintptr_t)R & 15) == 0 && ldr % 4 == 0));
  a.tiles_n = (g.N + BN - 1) / BN;
  a.tiles = a.tiles_n * ((g.M + BM - 1) / BM);
  a.splits = splits;
  const int grid = std::min(a.tiles * splits, device_sms());
  k_gemm_tf32<<<grid, NTHREADS, SMEM, s>>>(tAh, tAl, tBh, tBl, a);
  count_launch();
  return true;
}

}  // namespace llm
