// Memory-bound kernels of the training step: weight casts, embedding gather and
// scatter-add, RMSNorm forward/backward, RoPE, SwiGLU, cross-entropy, loss
// reduction, AdamW and initialisation.  Each cites the passage it computes.
#include <algorithm>
#include <map>
#include <mutex>
#include <utility>

#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace llm {

thread_local int g_launches = 0;

bool smem_optin(const void *func, int bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  static std::mutex mu;
  static std::map<std::pair<int, const void *>, int> done;  // largest size set per (device, kernel)
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(dev, func);
  auto it = done.find(key);
  if (it != done.end() && it->second >= bytes) return true;
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return false;
  done[key] = bytes;
  return true;
}

int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  static std::mutex mu;
  static std::map<int, int> sms;
  std::lock_guard<std::mutex> lock(mu);
  auto it = sms.find(dev);
  if (it != sms.end()) return it->second;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
    n = 1;
  sms[dev] = n;
  return n;
}

static inline unsigned cdiv(int64_t a, int64_t b) { return (unsigned)((a + b - 1) / b); }

// ------------------------------------------------------------------ RoPE table
// Hephaistos, Architecture at a glance (Positions): rotary embedding of q and
// k.  theta_j = base^(-2j/hd); angle = (t / scale) * theta_j for position t
// (scale 1; strata, RoPE row: position interpolation folds extended positions
// into the trained range with scale > 1).  The table is built in double
// precision, then rounded to float.
__global__ void k_rope_table(float *cos_t, float *sin_t, int T, int half, int hd, double base,
                             double scale) {
  int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= (int64_t)T * half) return;
  int t = (int)(i / half), j = (int)(i % half);
  double ang = ((double)t / scale) * pow(base, -2.0 * j / hd);
  cos_t[i] = (float)cos(ang);
  sin_t[i] = (float)sin(ang);
}
void rope_table(float *cos_t, float *sin_t, int T, int hd, float base, cudaStream_t s,
                double scale) {
  int64_t n = (int64_t)T * (hd / 2);
  k_rope_table<<<cdiv(n, 256), 256, 0, s>>>(cos_t, sin_t, T, hd / 2, hd, (double)base, scale);
  count_launch();
}

// ------------------------------------------------------------- weight casts
// dst[r, c] (rows_p x cols_p, zero padding) from src [rows x cols]; mode 1
// interleaves W1 | W3 in blocks of SWIGLU_BLOCK columns.  One block per row
// (grid-stride), 4 columns per thread: the 4 source columns of an aligned
// group are contiguous in both modes (SWIGLU_BLOCK and h are multiples of 4),
// so they move as one 16-byte load when vec is set.
// 4 consecutive values, one vector store when the address allows it
LLM_DEV void put4(__nv_bfloat16 *d, const float (&v)[4]) {
  if (((uintptr_t)d & 7) == 0) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
    *reinterpret_cast<uint2 *>(d) =
        make_uint2(*reinterpret_cast<uint32_t *>(&a), *reinterpret_cast<uint32_t *>(&b));
  } else {
    for (int k = 0; k < 4; k++) d[k] = __float2bfloat16_rn(v[k]);
  }
}
LLM_DEV void put4(float *d, const float (&v)[4]) {
  if (((uintptr_t)d & 15) == 0) *reinterpret_cast<float4 *>(d) = make_float4(v[0], v[1], v[2], v[3]);
  else for (int k = 0; k < 4; k++) d[k] = v[k];
}
LLM_DEV int64_t cast_src_col(int64_t c, int mode, int64_t h) {
  if (mode == 0) return c;
  int64_t blk = c / (2 * SWIGLU_BLOCK), w = c % (2 * SWIGLU_BLOCK);
  int64_t j = blk * SWIGLU_BLOCK + (w % SWIGLU_BLOCK);
  return j < h ? (w < SWIGLU_BLOCK ? j : h + j) : -1;
}
template <typename A>
__global__ void k_cast_weight(const float *__restrict__ src, A *__restrict__ dst, int64_t rows,
                              int64_t cols, int64_t rows_p, int64_t cols_p, int mode, int64_t h,
                              int64_t hp, int64_t sbs, int64_t dbs, bool vec) {
  src += blockIdx.y * sbs;
  dst += blockIdx.y * dbs;
  const int64_t ncols = mode == 0 ? cols : 2 * h;  // valid source columns
  for (int64_t r = blockIdx.x; r < rows_p; r += gridDim.x) {
    const float *sr = src + r * cols;
    A *dr = dst + r * cols_p;
    for (int64_t c = 4 * (int64_t)threadIdx.x; c < cols_p; c += 4 * (int64_t)blockDim.x) {
      float v[4] = {0.f, 0.f, 0.f, 0.f};
      if (r < rows) {
        const int64_t sc = cast_src_col(c, mode, h);
        if (vec && sc >= 0 && sc + 4 <= ncols && (mode == 0 ? c + 4 <= cols : true)) {
          const float4 q = *reinterpret_cast<const float4 *>(sr + sc);
          v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
        } else {
          for (int k = 0; k < 4; k++) {
            const int64_t cc = c + k;
            const int64_t sk = cast_src_col(cc, mode, h);
            if (sk >= 0 && (mode != 0 || cc < cols)) v[k] = sr[sk];
          }
        }
      }
      if (c + 4 <= cols_p) put4(dr + c, v);
      else for (int k = 0; c + k < cols_p; k++) dr[c + k] = from_f<A>(v[k]);
    }
  }
}
void cast_weight(const float *src, void *dst, DType dt, int64_t rows, int64_t cols,
                 int64_t rows_p, int64_t cols_p, int mode, int64_t h, int64_t hp, int batch,
                 int64_t sbs, int64_t dbs, cudaStream_t s) {
  // 16-byte source groups need aligned rows (and for mode 1 a 4-aligned h)
  const bool vec = ((uintptr_t)src & 15) == 0 && cols % 4 == 0 && sbs % 4 == 0 &&
                   (mode == 0 || h % 4 == 0) && cols_p % 4 == 0 && dbs % 4 == 0;
  dim3 grid((unsigned)std::min<int64_t>(rows_p, 148 * 8), batch);
  if (dt == DT_BF16)
    k_cast_weight<<<grid, 256, 0, s>>>(src, (__nv_bfloat16 *)dst, rows, cols, rows_p, cols_p, mode,
                                       h, hp, sbs, dbs, vec);
  else
    k_cast_weight<<<grid, 256, 0, s>>>(src, (float *)dst, rows, cols, rows_p, cols_p, mode, h, hp,
                                       sbs, dbs, vec);
  count_launch();
}

// ------------------------------------------------------------ embedding fwd
// Hephaistos, Architecture at a glance: token embedding, no positional table.
// x[i,:] = wte[tok_i,:].  Out-of-range ids set FLAG_TOKEN and read row 0.
__global__ void k_embed_fwd(const float *__restrict__ wte, const int32_t *__restrict__ tok,
                            float *__restrict__ x, int64_t N, int d, int V, int *flag) {
  int64_t row = blockIdx.x;
  int t = tok[row];
  if (t < 0 || t >= V) {
    if (threadIdx.x == 0) atomicOr(flag, FLAG_TOKEN);
    t = 0;
  }
  const float *src = wte + (int64_t)t * d;
  float *dst = x + row * d;
  if ((d & 3) == 0) {
    for (int j = threadIdx.x; j < d / 4; j += blockDim.x)
      reinterpret_cast<float4 *>(dst)[j] = reinterpret_cast<const float4 *>(src)[j];
  } else {
    for (int j = threadIdx.x; j < d; j += blockDim.x) dst[j] = src[j];
  }
}
void embed_fwd(const float *wte, const int32_t *tok, float *x, int64_t N, int d, int V, int *flag,
               cudaStream_t s) {
  k_embed_fwd<<<(unsigned)N, min(256, max(32, d / 4)), 0, s>>>(wte, tok, x, N, d, V, flag);
  count_launch();
}

// Four values to 4 consecutive elements: one 8-byte store for bf16, one
// 16-byte store for float (dst aligned to the element group).
LLM_DEV void store4(__nv_bfloat16 *dst, float4 o) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(o.x, o.y), hi = __floats2bfloat162_rn(o.z, o.w);
  uint2 q;
  q.x = *reinterpret_cast<uint32_t *>(&lo);
  q.y = *reinterpret_cast<uint32_t *>(&hi);
  *reinterpret_cast<uint2 *>(dst) = q;
}
LLM_DEV void store4(float *dst, float4 o) { *reinterpret_cast<float4 *>(dst) = o; }

// -------------------------------------------------------------- RMSNorm fwd
// Hephaistos, Architecture at a glance (Normalization); MicroGPT in Rust,
// RMSNorm: r = (mean_j x_j^2 + eps)^-1/2, y = g * x * r; r is cached.
// One warp per row.
template <typename A>
__global__ void k_rmsnorm_fwd(const float *__restrict__ x, const float *__restrict__ g,
                              A *__restrict__ y, float *__restrict__ rstd, int64_t N, int d,
                              float eps) {
  int64_t row = blockIdx.x * (int64_t)(blockDim.x / 32) + threadIdx.x / 32;
  int lane = threadIdx.x & 31;
  if (row >= N) return;
  const float *xr = x + row * d;
  float ss = 0.f;
  if ((d & 127) == 0) {
    for (int j = lane * 4; j < d; j += 128) {
      float4 v = *reinterpret_cast<const float4 *>(xr + j);
      ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
  } else {
    for (int j = lane; j < d; j += 32) ss += xr[j] * xr[j];
  }
  ss = warp_sum(ss);
  float r = 1.0f / sqrtf(ss / (float)d + eps);
  if (lane == 0) rstd[row] = r;
  A *yr = y + row * d;
  for (int j = lane; j < d; j += 32) yr[j] = from_f<A>(g[j] * xr[j] * r);
}
// d = 128 * VPL: one warp per row, each lane holding VPL float4 of the row
// (one read), the normalised row written with 8-byte (bf16) or 16-byte stores.
template <typename A, int VPL>
__global__ void __launch_bounds__(256) k_rmsnorm_fwd_v(const float *__restrict__ x,
                                                       const float *__restrict__ g,
                                                       A *__restrict__ y, float *__restrict__ rstd,
                                                       int64_t N, float eps) {
  constexpr int d = 128 * VPL;
  const int64_t row = blockIdx.x * (int64_t)(blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= N) return;
  const float4 *xr = reinterpret_cast<const float4 *>(x + row * d);
  float4 v[VPL];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < VPL; k++) {
    v[k] = xr[lane + 32 * k];
    ss += v[k].x * v[k].x + v[k].y * v[k].y + v[k].z * v[k].z + v[k].w * v[k].w;
  }
  ss = warp_sum(ss);
  const float r = 1.0f / sqrtf(ss / (float)d + eps);
  if (lane == 0) rstd[row] = r;
#pragma unroll
  for (int k = 0; k < VPL; k++) {
    const float4 gv = reinterpret_cast<const float4 *>(g)[lane + 32 * k];
    float4 o;
    o.x = gv.x * v[k].x * r; o.y = gv.y * v[k].y * r; o.z = gv.z * v[k].z * r; o.w = gv.w * v[k].w * r;
    store4(y + row * d + 4 * (lane + 32 * k), o);
  }
}
void rmsnorm_fwd(const float *x, const float *g, void *y, DType dt, float *rstd, int64_t N, int d,
                 float eps, cudaStream_t s) {
  unsigned grid = cdiv(N, 8);
  if ((d == 128 || d == 256 || d == 512 || d == 1024) && ((uintptr_t)x & 15) == 0 &&
      ((uintptr_t)g & 15) == 0 && ((uintptr_t)y & 15) == 0) {
#define RF(VPL)                                                                                  \
  do {                                                                                           \
    if (dt == DT_BF16)                                                                           \
      k_rmsnorm_fwd_v<__nv_bfloat16, VPL><<<grid, 256, 0, s>>>(x, g, (__nv_bfloat16 *)y, rstd, N, \
                                                                eps);                            \
    else                                                                                         \
      k_rmsnorm_fwd_v<float, VPL><<<grid, 256, 0, s>>>(x, g, (float *)y, rstd, N, eps);         \
  } while (0)
    if (d == 128) RF(1);
    else if (d == 256) RF(2);
    else if (d == 512) RF(4);
    else RF(8);
#undef RF
    count_launch();
    return;
  }
  if (dt == DT_BF16)
    k_rmsnorm_fwd<<<grid, 256, 0, s>>>(x, g, (__nv_bfloat16 *)y, rstd, N, d, eps);
  else
    k_rmsnorm_fwd<<<grid, 256, 0, s>>>(x, g, (float *)y, rstd, N, d, eps);
  count_launch();
}

// -------------------------------------------------------------- RMSNorm bwd
// Backward of y = g x r:  dx = r g dy - x r^3 (1/d) sum_j g_j dy_j x_j, plus
// the residual gradient dres; dg = sum over rows of dy x r, reduced in a fixed
// order: each block writes the partial sum of its rows, and reduce_partials
// adds the blocks in index order.  The N rows are split evenly over
// RMS_BLOCKS blocks (at least 16 rows each): two whole waves of the d = 1024
// kernel, whose 188 registers a thread leave room for one block per SM (64
// rows a block made 1.73 waves), and one wave at smaller d.
constexpr int RMS_BLOCKS = 2 * 148;
int rmsnorm_bwd_blocks(int64_t N) {
  return (int)std::max<int64_t>(1, std::min<int64_t>(cdiv(N, 16), RMS_BLOCKS));
}

template <typename A>
__global__ void k_rmsnorm_bwd(const float *__restrict__ x, const float *__restrict__ rstd,
                              const float *__restrict__ g, const float *__restrict__ dy,
                              const float *dres, float *dx,  // may alias (read then write)
                              A *__restrict__ dx_act, float *__restrict__ part, int64_t N, int d) {
  extern __shared__ float sacc[];  // [nwarps][d]
  int warp = threadIdx.x / 32, lane = threadIdx.x & 31, nw = blockDim.x / 32;
  float *acc = sacc + (int64_t)warp * d;
  for (int j = lane; j < d; j += 32) acc[j] = 0.f;
  const int64_t r1 = (blockIdx.x + 1) * N / gridDim.x;
  for (int64_t row = blockIdx.x * N / gridDim.x + warp; row < r1; row += nw) {
    const float *xr = x + row * d, *dyr = dy + row * d;
    float r = rstd[row];
    float dot = 0.f;
    for (int j = lane; j < d; j += 32) dot += g[j] * dyr[j] * xr[j];
    dot = warp_sum(dot);
    float c = r * r * r * dot / (float)d;
    for (int j = lane; j < d; j += 32) {
      float v = r * g[j] * dyr[j] - xr[j] * c;
      if (dres) v += dres[row * d + j];
      dx[row * d + j] = v;
      if (dx_act) dx_act[row * d + j] = from_f<A>(v);
      acc[j] += dyr[j] * xr[j] * r;
    }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    float s = 0.f;
    for (int w = 0; w < nw; w++) s += sacc[(int64_t)w * d + j];
    part[(int64_t)blockIdx.x * d + j] = s;
  }
}

// Vectorised form for d = 128 * VPL: each lane owns VPL float4 columns of a
// row, keeps its gain-gradient partial sums in registers, and the block adds
// its 8 warps' partials in warp order.
template <typename A, int VPL>
__global__ void __launch_bounds__(256) k_rmsnorm_bwd_v(const float *__restrict__ x,
                                                       const float *__restrict__ rstd,
                                                       const float *__restrict__ g,
                                                       const float *__restrict__ dy,
                                                       const float *dres, float *dx,
                                                       A *__restrict__ dx_act,
                                                       float *__restrict__ part, int64_t N) {
  constexpr int d = 128 * VPL;
  __shared__ float4 sred[8][32 * VPL];
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  float4 gv[VPL], acc[VPL];
#pragma unroll
  for (int k = 0; k < VPL; k++) {
    gv[k] = reinterpret_cast<const float4 *>(g)[lane + 32 * k];
    acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const int64_t r1 = (blockIdx.x + 1) * N / gridDim.x;
  for (int64_t row = blockIdx.x * N / gridDim.x + warp; row < r1; row += 8) {
    const float4 *xr = reinterpret_cast<const float4 *>(x + row * d);
    const float4 *dyr = reinterpret_cast<const float4 *>(dy + row * d);
    float4 xv[VPL], dv[VPL], rv[VPL];
    float dot = 0.f;
#pragma unroll
    for (int k = 0; k < VPL; k++) {
      xv[k] = xr[lane + 32 * k];
      dv[k] = dyr[lane + 32 * k];
      rv[k] = dres ? reinterpret_cast<const float4 *>(dres + row * d)[lane + 32 * k]
                   : make_float4(0.f, 0.f, 0.f, 0.f);
      dot += gv[k].x * dv[k].x * xv[k].x + gv[k].y * dv[k].y * xv[k].y +
             gv[k].z * dv[k].z * xv[k].z + gv[k].w * dv[k].w * xv[k].w;
    }
    dot = warp_sum(dot);
    const float r = rstd[row];
    const float c = r * r * r * dot / (float)d;
#pragma unroll
    for (int k = 0; k < VPL; k++) {
      float4 o;
      o.x = r * gv[k].x * dv[k].x - xv[k].x * c;
      o.y = r * gv[k].y * dv[k].y - xv[k].y * c;
      o.z = r * gv[k].z * dv[k].z - xv[k].z * c;
      o.w = r * gv[k].w * dv[k].w - xv[k].w * c;
      o.x += rv[k].x; o.y += rv[k].y; o.z += rv[k].z; o.w += rv[k].w;
      reinterpret_cast<float4 *>(dx + row * d)[lane + 32 * k] = o;
      if (dx_act) store4(dx_act + row * d + 4 * (lane + 32 * k), o);
      acc[k].x += dv[k].x * xv[k].x * r;
      acc[k].y += dv[k].y * xv[k].y * r;
      acc[k].z += dv[k].z * xv[k].z * r;
      acc[k].w += dv[k].w * xv[k].w * r;
    }
  }
#pragma unroll
  for (int k = 0; k < VPL; k++) sred[warp][lane + 32 * k] = acc[k];
  __syncthreads();
  for (int j = threadIdx.x; j < 32 * VPL; j += 256) {
    float4 t = sred[0][j];
    for (int w = 1; w < 8; w++) {
      float4 q = sred[w][j];
      t.x += q.x; t.y += q.y; t.z += q.z; t.w += q.w;
    }
    reinterpret_cast<float4 *>(part + (int64_t)blockIdx.x * d)[j] = t;
  }
}

int rmsnorm_bwd(const float *x, const float *rstd, const float *g, const float *dy,
                const float *dres, float *dx, void *dx_act, DType dt, float *part, int64_t N, int d,
                cudaStream_t s) {
  int nblk = rmsnorm_bwd_blocks(N);
  if (d == 128 || d == 256 || d == 512 || d == 1024) {
#define RB(VPL)                                                                                \
  do {                                                                                         \
    if (dt == DT_BF16)                                                                         \
      k_rmsnorm_bwd_v<__nv_bfloat16, VPL><<<nblk, 256, 0, s>>>(x, rstd, g, dy, dres, dx,       \
                                                                (__nv_bfloat16 *)dx_act, part, N); \
    else                                                                                       \
      k_rmsnorm_bwd_v<float, VPL><<<nblk, 256, 0, s>>>(x, rstd, g, dy, dres, dx, (float *)dx_act, \
                                                        part, N);                              \
  } while (0)
    if (d == 128) RB(1);
    else if (d == 256) RB(2);
    else if (d == 512) RB(4);
    else RB(8);
#undef RB
    count_launch();
    return nblk;
  }
  // generic width: 8 warps' gain-gradient rows in shared memory (128 KiB at
  // the largest accepted width, 4096), so opt in above the 48 KiB default
  const int smem = (int)(sizeof(float) * 8 * d);
  if (dt == DT_BF16) {
    smem_optin((const void *)k_rmsnorm_bwd<__nv_bfloat16>, smem);  // a refusal fails the launch
    k_rmsnorm_bwd<<<nblk, 256, smem, s>>>(x, rstd, g, dy, dres, dx, (__nv_bfloat16 *)dx_act, part,
                                          N, d);
  } else {
    smem_optin((const void *)k_rmsnorm_bwd<float>, smem);
    k_rmsnorm_bwd<<<nblk, 256, smem, s>>>(x, rstd, g, dy, dres, dx, (float *)dx_act, part, N, d);
  }
  count_launch();
  return nblk;
}

// out[j] = sum over b of part[b][j]: RP_GROUPS groups of threads add
// interleaved rows (b = grp, grp + RP_GROUPS, ...; four loads in flight, added
// in row order), then the group sums are added in group order (a fixed order,
// so the result does not depend on scheduling).  One block per 32 columns.
constexpr int RP_GROUPS = 32;
__global__ void __launch_bounds__(32 * RP_GROUPS)
    k_reduce_partials(const float *__restrict__ part, int nblk, int d, float *__restrict__ out) {
  __shared__ float sh[RP_GROUPS][33];
  const int c = threadIdx.x & 31, grp = threadIdx.x >> 5;
  const int j = blockIdx.x * 32 + c;
  float s = 0.f;
  if (j < d) {
    int b = grp;
    for (; b + 3 * RP_GROUPS < nblk; b += 4 * RP_GROUPS) {
      const float v0 = part[(int64_t)b * d + j], v1 = part[(int64_t)(b + RP_GROUPS) * d + j],
                  v2 = part[(int64_t)(b + 2 * RP_GROUPS) * d + j],
                  v3 = part[(int64_t)(b + 3 * RP_GROUPS) * d + j];
      s += v0;
      s += v1;
      s += v2;
      s += v3;
    }
    for (; b < nblk; b += RP_GROUPS) s += part[(int64_t)b * d + j];
  }
  sh[grp][c] = s;
  __syncthreads();
  if (grp == 0 && j < d) {
    float t = sh[0][c];
    for (int k = 1; k < RP_GROUPS; k++) t += sh[k][c];
    out[j] = t;
  }
}
void reduce_partials(const float *part, int nblk, int d, float *out, cudaStream_t s) {
  k_reduce_partials<<<cdiv(d, 32), 32 * RP_GROUPS, 0, s>>>(part, nblk, d, out);
  count_launch();
}

// --------------------------------------------------------------------- RoPE
// Rotate-half rotation of the q and k columns (the first ncols_rot columns of
// each row, heads of hd) by +angle (sign 1, forward) or -angle (sign -1, the
// backward of the forward rotation).  Position = row % T.
template <typename A>
__global__ void k_rope_apply(A *__restrict__ qkv, const float *__restrict__ cos_t,
                             const float *__restrict__ sin_t, int64_t N, int T, int ncols_rot,
                             int64_t ld, int hd, float sign) {
  int half = hd / 2;
  int64_t pairs_per_row = ncols_rot / 2;
  int64_t n = N * pairs_per_row;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    int64_t row = i / pairs_per_row;
    int p = (int)(i % pairs_per_row);
    int head = p / half, j = p % half;
    int t = (int)(row % T);
    float c = cos_t[(int64_t)t * half + j], sn = sign * sin_t[(int64_t)t * half + j];
    A *u = qkv + row * ld + (int64_t)head * hd;
    float a = to_f(u[j]), b = to_f(u[j + half]);
    u[j] = from_f<A>(a * c - b * sn);
    u[j + half] = from_f<A>(b * c + a * sn);
  }
}
void rope_apply(void *qkv, DType dt, const float *cos_t, const float *sin_t, int64_t N, int T,
                int ncols_rot, int64_t ld, int hd, int sign, cudaStream_t s) {
  int64_t n = N * (ncols_rot / 2);
  unsigned grid = min(cdiv(n, 256), 148u * 16);
  if (dt == DT_BF16)
    k_rope_apply<<<grid, 256, 0, s>>>((__nv_bfloat16 *)qkv, cos_t, sin_t, N, T, ncols_rot, ld, hd,
                                      (float)sign);
  else
    k_rope_apply<<<grid, 256, 0, s>>>((float *)qkv, cos_t, sin_t, N, T, ncols_rot, ld, hd,
                                      (float)sign);
  count_launch();
}

// ------------------------------------------------------------------- SwiGLU
// Hephaistos, Architecture at a glance (Feed-forward): u = silu(a) * b.
// ab is [N, 2hp] in interleaved blocks (a columns then b columns per block).
template <typename A>
__global__ void k_swiglu_fwd(const A *__restrict__ ab, A *__restrict__ u, int64_t N, int64_t hp) {
  int64_t n = N * hp;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    int64_t row = i / hp, j = i % hp;
    const A *r = ab + row * 2 * hp;
    int64_t ca = w1_col(j);
    float a = to_f(r[ca]), b = to_f(r[ca + SWIGLU_BLOCK]);
    u[i] = from_f<A>(a * sigmoidf_(a) * b);
  }
}
// da = du * b * silu'(a), db = du * silu(a), silu'(a) = s (1 + a (1 - s)).
template <typename A>
__global__ void k_swiglu_bwd(const A *__restrict__ ab, const A *__restrict__ du,
                             A *__restrict__ dab, int64_t N, int64_t hp) {
  int64_t n = N * hp;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    int64_t row = i / hp, j = i % hp;
    const A *r = ab + row * 2 * hp;
    int64_t ca = w1_col(j);
    float a = to_f(r[ca]), b = to_f(r[ca + SWIGLU_BLOCK]), g = to_f(du[i]);
    float sg = sigmoidf_(a);
    dab[row * 2 * hp + ca] = from_f<A>(g * b * sg * (1.f + a * (1.f - sg)));
    dab[row * 2 * hp + ca + SWIGLU_BLOCK] = from_f<A>(g * a * sg);
  }
}
// bf16, 8 hidden units per thread with 16-byte accesses (8 | 64, so the 8
// units share one interleave block: a and b are 8 contiguous elements each).
LLM_DEV void unpack8(uint4 q, float (&f)[8]) {
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&q);
#pragma unroll
  for (int k = 0; k < 4; k++) {
    float2 t = __bfloat1622float2(h[k]);
    f[2 * k] = t.x;
    f[2 * k + 1] = t.y;
  }
}
LLM_DEV uint4 pack8(const float (&f)[8]) {
  uint4 q;
  uint32_t *w = reinterpret_cast<uint32_t *>(&q);
#pragma unroll
  for (int k = 0; k < 4; k++) {
    __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * k], f[2 * k + 1]);
    w[k] = *reinterpret_cast<uint32_t *>(&h);
  }
  return q;
}
// Grid-stride over (row, 8-unit group) items with 32-bit index arithmetic
// (the launcher keeps N * hp / 8 below 2^31).
__global__ void k_swiglu_fwd_v8(const __nv_bfloat16 *__restrict__ ab, __nv_bfloat16 *__restrict__ u,
                                int64_t N, int64_t hp) {
  const uint32_t per_row = (uint32_t)(hp / 8), n = (uint32_t)(N * (hp / 8));
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const uint32_t row = i / per_row, j = (i - row * per_row) * 8;
    const __nv_bfloat16 *r = ab + (int64_t)row * 2 * hp + w1_col(j);
    float a[8], b[8], o[8];
    unpack8(*reinterpret_cast<const uint4 *>(r), a);
    unpack8(*reinterpret_cast<const uint4 *>(r + SWIGLU_BLOCK), b);
#pragma unroll
    for (int k = 0; k < 8; k++) o[k] = swiglu_unit(a[k], b[k]);
    *reinterpret_cast<uint4 *>(u + (int64_t)row * hp + j) = pack8(o);
  }
}
__global__ void k_swiglu_bwd_v8(const __nv_bfloat16 *__restrict__ ab, const __nv_bfloat16 *__restrict__ du,
                                __nv_bfloat16 *__restrict__ dab, int64_t N, int64_t hp) {
  const uint32_t per_row = (uint32_t)(hp / 8), n = (uint32_t)(N * (hp / 8));
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const uint32_t row = i / per_row, j = (i - row * per_row) * 8;
    const int64_t ca = (int64_t)row * 2 * hp + w1_col(j);
    float a[8], b[8], g[8], da[8], db[8];
    unpack8(*reinterpret_cast<const uint4 *>(ab + ca), a);
    unpack8(*reinterpret_cast<const uint4 *>(ab + ca + SWIGLU_BLOCK), b);
    unpack8(*reinterpret_cast<const uint4 *>(du + (int64_t)row * hp + j), g);
#pragma unroll
    for (int k = 0; k < 8; k++) swiglu_bwd_unit(a[k], b[k], g[k], da[k], db[k]);
    *reinterpret_cast<uint4 *>(dab + ca) = pack8(da);
    *reinterpret_cast<uint4 *>(dab + ca + SWIGLU_BLOCK) = pack8(db);
  }
}

void swiglu_fwd(const void *ab, void *u, DType dt, int64_t N, int64_t hp, cudaStream_t s) {
  if (dt == DT_BF16 && hp % 8 == 0 && ((uintptr_t)ab & 15) == 0 && ((uintptr_t)u & 15) == 0 &&
      N * (hp / 8) < ((int64_t)1 << 31)) {
    k_swiglu_fwd_v8<<<min(cdiv(N * hp / 8, 256), 148u * 16), 256, 0, s>>>(
        (const __nv_bfloat16 *)ab, (__nv_bfloat16 *)u, N, hp);
    count_launch();
    return;
  }
  unsigned grid = min(cdiv(N * hp, 256), 148u * 16);
  if (dt == DT_BF16)
    k_swiglu_fwd<<<grid, 256, 0, s>>>((const __nv_bfloat16 *)ab, (__nv_bfloat16 *)u, N, hp);
  else
    k_swiglu_fwd<<<grid, 256, 0, s>>>((const float *)ab, (float *)u, N, hp);
  count_launch();
}
void swiglu_bwd(const void *ab, const void *du, void *dab, DType dt, int64_t N, int64_t hp,
                cudaStream_t s) {
  if (dt == DT_BF16 && hp % 8 == 0 && ((uintptr_t)ab & 15) == 0 && ((uintptr_t)du & 15) == 0 &&
      ((uintptr_t)dab & 15) == 0 && N * (hp / 8) < ((int64_t)1 << 31)) {
    k_swiglu_bwd_v8<<<min(cdiv(N * hp / 8, 256), 148u * 16), 256, 0, s>>>(
        (const __nv_bfloat16 *)ab, (const __nv_bfloat16 *)du, (__nv_bfloat16 *)dab, N, hp);
    count_launch();
    return;
  }
  unsigned grid = min(cdiv(N * hp, 256), 148u * 16);
  if (dt == DT_BF16)
    k_swiglu_bwd<<<grid, 256, 0, s>>>((const __nv_bfloat16 *)ab, (const __nv_bfloat16 *)du,
                                      (__nv_bfloat16 *)dab, N, hp);
  else
    k_swiglu_bwd<<<grid, 256, 0, s>>>((const float *)ab, (const float *)du, (float *)dab, N, hp);
  count_launch();
}

// ------------------------------------------------------------ cross-entropy
// Fused softmax cross-entropy forward and backward over the vocabulary
// (Hephaistos, "What you'll see": softmax+CE; randyGPT: over all positions).
// Per row: lse = log sum_v exp(z_v); loss_i = lse - z_{y_i};
// dz_v = (exp(z_v - lse) - [v = y_i]) * inv_n written over z in place.
// Probabilities are never stored.  Columns >= V (padding) become 0.
template <typename A, int NT>
__global__ void __launch_bounds__(NT) k_cross_entropy(A *__restrict__ z, const int32_t *__restrict__ tgt,
                                                      float *__restrict__ rowloss, int V,
                                                      int64_t ldz, float inv_n, int *flag) {
  __shared__ float sm[NT / 32], ss[NT / 32];
  int64_t row = blockIdx.x;
  A *zr = z + row * ldz;
  float m = -INFINITY, s = 0.f;
  auto acc = [&](float x) {
    if (x > m) { s = s * expf(m - x) + 1.f; m = x; }
    else s += expf(x - m);
  };
  constexpr int VW = 16 / sizeof(A);  // elements per 16-byte vector
  const bool vec = (ldz % VW) == 0 && (((uintptr_t)z) & 15) == 0;
  const int Vv = vec ? V / VW : 0;    // whole vectors inside [0, V)
  for (int i = threadIdx.x; i < Vv; i += NT) {
    uint4 q = reinterpret_cast<const uint4 *>(zr)[i];
    const A *e = reinterpret_cast<const A *>(&q);
#pragma unroll
    for (int k = 0; k < VW; k++) acc(to_f(e[k]));
  }
  for (int v = Vv * VW + threadIdx.x; v < V; v += NT) acc(to_f(zr[v]));
  // merge (m, s) across the block
  int lane = threadIdx.x & 31, w = threadIdx.x / 32;
  for (int o = 16; o > 0; o >>= 1) {
    float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
    float mm = fmaxf(m, m2);
    s = (mm == -INFINITY) ? 0.f : s * expf(m - mm) + s2 * expf(m2 - mm);
    m = mm;
  }
  if (lane == 0) { sm[w] = m; ss[w] = s; }
  __syncthreads();
  float M = -INFINITY;
  for (int i = 0; i < NT / 32; i++) M = fmaxf(M, sm[i]);
  float S = 0.f;
  for (int i = 0; i < NT / 32; i++) S += (sm[i] == -INFINITY) ? 0.f : ss[i] * expf(sm[i] - M);
  float lse = M + logf(S);
  int y = tgt[row];
  if (y < 0 || y >= V) {
    if (threadIdx.x == 0) atomicOr(flag, FLAG_TOKEN);
    y = 0;
  }
  float zy = to_f(zr[y]);
  __syncthreads();  // every thread has read z[y] before it is overwritten
  if (threadIdx.x == 0) rowloss[row] = lse - zy;
  const int Lv = vec ? (int)(ldz / VW) : 0;
  for (int i = threadIdx.x; i < Lv; i += NT) {
    uint4 q = reinterpret_cast<const uint4 *>(zr)[i];
    A *e = reinterpret_cast<A *>(&q);
#pragma unroll
    for (int k = 0; k < VW; k++) {
      int v = i * VW + k;
      float g = 0.f;
      if (v < V) g = (expf(to_f(e[k]) - lse) - (v == y ? 1.f : 0.f)) * inv_n;
      e[k] = from_f<A>(g);
    }
    reinterpret_cast<uint4 *>(zr)[i] = q;
  }
  for (int64_t v = (int64_t)Lv * VW + threadIdx.x; v < ldz; v += NT) {
    float g = 0.f;
    if (v < V) g = (expf(to_f(zr[v]) - lse) - (v == y ? 1.f : 0.f)) * inv_n;
    zr[v] = from_f<A>(g);
  }
}
// bf16 rows held in registers: each thread keeps R 16-byte vectors (8
// logits each, vector i = threadIdx.x + NT * k) from one read of the row and
// writes the gradient back over them once.  One exponential per logit: each
// thread takes its own maximum m_t and sum s_t = sum 2^((z - m_t) log2 e) over
// its logits, keeping the terms e = 2^((z - m_t) log2 e) (rounded to bf16, in
// the registers that held the logits); one block reduction of the (m_t, s_t)
// pairs in a fixed tree order gives the row's maximum M and sum S (the sum
// from the float32 terms), and the gradient is e * 2^((m_t - M) log2 e) / S
// minus 1 at the target, times 1/N.  Storing e rounds it once more than
// computing it afresh would (relative 2^-9, the bf16 output's own rounding).
// Exponentials by the single-instruction ex2 (relative error of a few ulp).
// Columns >= V inside the row (padding) get gradient 0.
LLM_DEV float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// (m, s) pairs with s relative to 2^(m log2 e): the pair of the union.
LLM_DEV void ms_combine(float &m, float &s, float m2, float s2) {
  constexpr float L2E = 1.4426950408889634f;
  const float mm = fmaxf(m, m2);
  if (mm == -INFINITY) return;  // both empty
  s = (m == -INFINITY ? 0.f : s * ex2_fast((m - mm) * L2E)) +
      (m2 == -INFINITY ? 0.f : s2 * ex2_fast((m2 - mm) * L2E));
  m = mm;
}
template <int NT, int R>
__global__ void __launch_bounds__(NT) k_cross_entropy_reg(__nv_bfloat16 *__restrict__ z,
                                                          const int32_t *__restrict__ tgt,
                                                          float *__restrict__ rowloss, int V,
                                                          int64_t ldz, float inv_n, int *flag) {
  constexpr float L2E = 1.4426950408889634f;
  __shared__ float red_m[NT / 32], red_s[NT / 32];
  __shared__ float bc_m, bc_s;
  const int64_t row = blockIdx.x;
  __nv_bfloat16 *zr = z + row * ldz;
  const int nvec = (int)(ldz / 8);
  const int lane = threadIdx.x & 31, w = threadIdx.x / 32;
  uint4 q[R];
#pragma unroll
  for (int k = 0; k < R; k++) {
    const int i = threadIdx.x + NT * k;
    q[k] = i < nvec ? reinterpret_cast<const uint4 *>(zr)[i] : make_uint4(0, 0, 0, 0);
  }
  int y = tgt[row];
  if (y < 0 || y >= V) {
    if (threadIdx.x == 0) atomicOr(flag, FLAG_TOKEN);
    y = 0;
  }
  const float zy = __bfloat162float(zr[y]);
  // this thread's maximum
  float mt = -INFINITY;
#pragma unroll
  for (int k = 0; k < R; k++) {
    const int v0 = 8 * (threadIdx.x + NT * k);
    const __nv_bfloat162 *e = reinterpret_cast<const __nv_bfloat162 *>(&q[k]);
#pragma unroll
    for (int t = 0; t < 4; t++) {
      const float2 f = __bfloat1622float2(e[t]);
      if (v0 + 2 * t < V) mt = fmaxf(mt, f.x);
      if (v0 + 2 * t + 1 < V) mt = fmaxf(mt, f.y);
    }
  }
  // terms relative to mt, kept as bf16 in place of the logits; their sum
  const float mt2 = mt == -INFINITY ? 0.f : mt * L2E;
  float st = 0.f;
#pragma unroll
  for (int k = 0; k < R; k++) {
    const int v0 = 8 * (threadIdx.x + NT * k);
    __nv_bfloat162 *e = reinterpret_cast<__nv_bfloat162 *>(&q[k]);
#pragma unroll
    for (int t = 0; t < 4; t++) {
      const float2 f = __bfloat1622float2(e[t]);
      const float ea = v0 + 2 * t < V ? ex2_fast(fmaf(f.x, L2E, -mt2)) : 0.f;
      const float eb = v0 + 2 * t + 1 < V ? ex2_fast(fmaf(f.y, L2E, -mt2)) : 0.f;
      st += ea + eb;
      e[t] = __floats2bfloat162_rn(ea, eb);
    }
  }
  // the row's (M, S): warp tree, then the warps in order by thread 0
  float m = mt, sm = st;
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, sm, o);
    ms_combine(m, sm, m2, s2);
  }
  if (lane == 0) {
    red_m[w] = m;
    red_s[w] = sm;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float M = red_m[0], S = red_s[0];
    for (int i = 1; i < NT / 32; i++) ms_combine(M, S, red_m[i], red_s[i]);
    bc_m = M;
    bc_s = S;
  }
  __syncthreads();
  const float M = bc_m, S = bc_s;
  const float lse = M + logf(S);
  if (threadIdx.x == 0) rowloss[row] = lse - zy;
  // every thread read z[y] (above) before any vector is written back: the
  // block barriers of the reduction order the read before these stores
  const float fac = mt == -INFINITY ? 0.f : ex2_fast((mt - M) * L2E) / S * inv_n;
#pragma unroll
  for (int k = 0; k < R; k++) {
    const int i = threadIdx.x + NT * k;
    if (i >= nvec) continue;
    const int v0 = 8 * i;
    __nv_bfloat162 *e = reinterpret_cast<__nv_bfloat162 *>(&q[k]);
#pragma unroll
    for (int t = 0; t < 4; t++) {
      const float2 f = __bfloat1622float2(e[t]);
      const int va = v0 + 2 * t, vb = va + 1;
      const float ga = f.x * fac - (va == y ? inv_n : 0.f);
      const float gb = f.y * fac - (vb == y ? inv_n : 0.f);
      e[t] = __floats2bfloat162_rn(ga, gb);
    }
    reinterpret_cast<uint4 *>(zr)[i] = q[k];
  }
}

// Streaming form (bf16, rows of at most 32768 columns): a persistent grid of
// one 512-thread block per SM walks groups of G = 16 / WPR consecutive rows
// (WPR warps per row, at most 8 vectors of 8 logits per thread).  Each group
// comes into one of CES_NBUF 64 KiB shared-memory buffers by one bulk copy
// (cp.async.bulk, completion counted on an mbarrier), so the next two groups
// load while the current one is reduced and its gradient stored (with two
// buffers, one 64 KiB row in flight per SM left the 350M step's 32000-wide
// rows at 0.48 of the copy rate); the row
// arithmetic is the register form's above (one exponential per logit, the
// terms kept as bf16, one (m, s) reduction per row in a fixed order).  Every
// wait is bounded: on time-out the block records FLAG_TIMEOUT, waits (again
// bounded) for its own copies and leaves.
constexpr int CES_THREADS = 512, CES_R = 8, CES_BUF = 64 * 1024, CES_NBUF = 3;
template <int WPR>
__global__ void __launch_bounds__(CES_THREADS, 1)
    k_cross_entropy_stream(__nv_bfloat16 *__restrict__ z, const int32_t *__restrict__ tgt,
                           float *__restrict__ rowloss, int64_t N, int V, int64_t ldz,
                           float inv_n, int *flag) {
  constexpr float L2E = 1.4426950408889634f;
  constexpr int G = 16 / WPR, TPR = 32 * WPR;
  extern __shared__ __align__(1024) uint8_t ce_buf[];  // [CES_NBUF][CES_BUF]
  __shared__ uint64_t full[CES_NBUF];
  __shared__ float red_m[16], red_s[16];
  __shared__ int stop_sh;
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int grow = warp / WPR, t = threadIdx.x - grow * TPR;
  const int64_t row_bytes = ldz * 2, ngroups = (N + G - 1) / G;
  const int nvec = (int)(ldz / 8);
  const uint32_t fb0 = tc::smem_u32(&full[0]);
  if (threadIdx.x == 0) {
    for (int bb = 0; bb < CES_NBUF; bb++) tc::mbar_init(fb0 + 8 * bb, 1);
    stop_sh = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // thread 0's record of the copy in flight into each buffer (for the drain)
  uint32_t issued = 0, par[CES_NBUF] = {};
  auto issue = [&](int64_t gi, int b) {
    const int64_t rows = min((int64_t)G, N - gi * G);
    const uint32_t bytes = (uint32_t)(rows * row_bytes);
    const uint32_t bar = fb0 + 8 * b;
    tc::mbar_arrive_expect_tx(bar, bytes);
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            tc::smem_u32(ce_buf + b * CES_BUF)),
        "l"(z + gi * G * ldz), "r"(bytes), "r"(bar)
        : "memory");
    issued |= 1u << b;
  };
  if (threadIdx.x == 0)
    for (int bb = 0; bb < CES_NBUF; bb++)
      if (blockIdx.x + (int64_t)bb * gridDim.x < ngroups) issue(blockIdx.x + (int64_t)bb * gridDim.x, bb);
  int k = 0;
  for (int64_t gi = blockIdx.x; gi < ngroups; gi += gridDim.x, k++) {
    const int b = k % CES_NBUF;
    const uint32_t ph = (k / CES_NBUF) & 1;
    // bounded wait for this group's rows, then a block-wide verdict
    bool ok = tc::mbar_try(fb0 + 8 * b, ph);
    if (!ok) {
      const unsigned long long t0 = tc::gtimer();
      while (!(ok = tc::mbar_try(fb0 + 8 * b, ph)) && tc::gtimer() - t0 < tc::WAIT_NS) {
      }
    }
    if (__syncthreads_or(!ok)) {
      if (threadIdx.x == 0) {
        atomicOr(flag, FLAG_TIMEOUT);
        for (int bb = 0; bb < CES_NBUF; bb++)
          if (issued & (1u << bb)) {
            const unsigned long long t0 = tc::gtimer();
            while (!tc::mbar_try(fb0 + 8 * bb, par[bb]) && tc::gtimer() - t0 < tc::WAIT_NS) {
            }
          }
      }
      return;
    }
    if (threadIdx.x == 0) {
      issued &= ~(1u << b);
      par[b] ^= 1u;
    }
    const int64_t row = gi * G + grow;
    const bool valid = row < N;
    const uint8_t *src = ce_buf + b * CES_BUF + grow * row_bytes;
    uint4 q[CES_R];
#pragma unroll
    for (int kk = 0; kk < CES_R; kk++) {
      const int i = t + TPR * kk;
      q[kk] = (valid && i < nvec) ? reinterpret_cast<const uint4 *>(src)[i] : make_uint4(0, 0, 0, 0);
    }
    int y = valid ? tgt[row] : 0;
    if (y < 0 || y >= V) {
      if (valid && t == 0) atomicOr(flag, FLAG_TOKEN);
      y = 0;
    }
    const float zy = valid ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(src)[y]) : 0.f;
    __syncthreads();  // buffer b is read: the group CES_NBUF ahead may land in it
    if (threadIdx.x == 0 && gi + CES_NBUF * (int64_t)gridDim.x < ngroups)
      issue(gi + CES_NBUF * (int64_t)gridDim.x, b);
    // this thread's maximum, its terms (kept as bf16) and their sum; a whole
    // vector inside [0, V) takes the unchecked form: three-input maxima and
    // packed f32x2 arithmetic (the kernel is issue-bound, not HBM-bound)
    float mt = -INFINITY;
#pragma unroll
    for (int kk = 0; kk < CES_R; kk++) {
      const int v0 = 8 * (t + TPR * kk);
      const __nv_bfloat162 *e = reinterpret_cast<const __nv_bfloat162 *>(&q[kk]);
      if (v0 + 8 <= V) {
#pragma unroll
        for (int u = 0; u < 4; u++) {
          const float2 f = __bfloat1622float2(e[u]);
          mt = tc::fmax3(mt, f.x, f.y);
        }
      } else {
#pragma unroll
        for (int u = 0; u < 4; u++) {
          const float2 f = __bfloat1622float2(e[u]);
          if (v0 + 2 * u < V) mt = fmaxf(mt, f.x);
          if (v0 + 2 * u + 1 < V) mt = fmaxf(mt, f.y);
        }
      }
    }
    const float mt2 = mt == -INFINITY ? 0.f : mt * L2E;
    const float2 l2e2 = make_float2(L2E, L2E), nm2 = make_float2(-mt2, -mt2);
    float2 st2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int kk = 0; kk < CES_R; kk++) {
      const int v0 = 8 * (t + TPR * kk);
      __nv_bfloat162 *e = reinterpret_cast<__nv_bfloat162 *>(&q[kk]);
      if (v0 + 8 <= V) {
#pragma unroll
        for (int u = 0; u < 4; u++) {
          const float2 x = __ffma2_rn(__bfloat1622float2(e[u]), l2e2, nm2);
          const float2 ex = make_float2(ex2_fast(x.x), ex2_fast(x.y));
          st2 = __fadd2_rn(st2, ex);
          e[u] = __floats2bfloat162_rn(ex.x, ex.y);
        }
      } else {
#pragma unroll
        for (int u = 0; u < 4; u++) {
          const float2 f = __bfloat1622float2(e[u]);
          const float ea = v0 + 2 * u < V ? ex2_fast(fmaf(f.x, L2E, -mt2)) : 0.f;
          const float eb = v0 + 2 * u + 1 < V ? ex2_fast(fmaf(f.y, L2E, -mt2)) : 0.f;
          st2.x += ea;
          st2.y += eb;
          e[u] = __floats2bfloat162_rn(ea, eb);
        }
      }
    }
    const float st = st2.x + st2.y;
    // the row's (M, S): warp tree, then the row's warps in order
    float M = mt, S = st;
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, M, o), s2 = __shfl_xor_sync(0xffffffffu, S, o);
      ms_combine(M, S, m2, s2);
    }
    if (WPR > 1) {
      if (lane == 0) {
        red_m[warp] = M;
        red_s[warp] = S;
      }
      __syncthreads();
      M = red_m[grow * WPR];
      S = red_s[grow * WPR];
      for (int w = 1; w < WPR; w++) ms_combine(M, S, red_m[grow * WPR + w], red_s[grow * WPR + w]);
      __syncthreads();  // red is reused by the next group
    }
    if (!valid) continue;
    const float lse = M + logf(S);
    if (t == 0) rowloss[row] = lse - zy;
    const float fac = mt == -INFINITY ? 0.f : ex2_fast((mt - M) * L2E) / S * inv_n;
    const float2 fac2 = make_float2(fac, fac);
    __nv_bfloat16 *zr = z + row * ldz;
#pragma unroll
    for (int kk = 0; kk < CES_R; kk++) {
      const int i = t + TPR * kk;
      if (i >= nvec) continue;
      const int v0 = 8 * i;
      __nv_bfloat162 *e = reinterpret_cast<__nv_bfloat162 *>(&q[kk]);
      if ((unsigned)(y - v0) >= 8u) {  // the target is not in this vector
#pragma unroll
        for (int u = 0; u < 4; u++) {
          const float2 g = __fmul2_rn(__bfloat1622float2(e[u]), fac2);
          e[u] = __floats2bfloat162_rn(g.x, g.y);
        }
      } else {
#pragma unroll
        for (int u = 0; u < 4; u++) {
          const float2 f = __bfloat1622float2(e[u]);
          const int va = v0 + 2 * u, vb = va + 1;
          e[u] = __floats2bfloat162_rn(f.x * fac - (va == y ? inv_n : 0.f),
                                       f.y * fac - (vb == y ? inv_n : 0.f));
        }
      }
      reinterpret_cast<uint4 *>(zr)[i] = q[kk];
    }
  }
}

void cross_entropy(void *logits, DType dt, const int32_t *tgt, float *rowloss, int64_t N, int V,
                   int64_t ldz, float inv_n, int *flag, cudaStream_t s) {
  constexpr int NT = 256, R = 16;
  if (dt == DT_BF16 && ldz % 8 == 0 && ((uintptr_t)logits & 15) == 0 && ldz <= 32768) {
    // warps per row: the fewest (a power of two) that keep 8 vectors a thread
    const int64_t nvec = ldz / 8;
    int wpr = 1;
    while ((int64_t)32 * wpr * CES_R < nvec) wpr *= 2;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t groups = (N + 16 / wpr - 1) / (16 / wpr);
    const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(groups, sms));
    const int smem = CES_NBUF * CES_BUF;
#define CES(W)                                                                                    \
  do {                                                                                            \
    smem_optin((const void *)k_cross_entropy_stream<W>, smem);                                   \
    k_cross_entropy_stream<W><<<grid, CES_THREADS, smem, s>>>((__nv_bfloat16 *)logits, tgt,      \
                                                             rowloss, N, V, ldz, inv_n, flag);   \
  } while (0)
    switch (wpr) {
      case 1: CES(1); break;
      case 2: CES(2); break;
      case 4: CES(4); break;
      case 8: CES(8); break;
      default: CES(16); break;
    }
#undef CES
    count_launch();
    return;
  }
  if (dt == DT_BF16 && ldz % 8 == 0 && ((uintptr_t)logits & 15) == 0 && ldz <= (int64_t)NT * R * 8) {
    k_cross_entropy_reg<NT, R><<<(unsigned)N, NT, 0, s>>>((__nv_bfloat16 *)logits, tgt, rowloss, V,
                                                         ldz, inv_n, flag);
    count_launch();
    return;
  }
  if (dt == DT_BF16)
    k_cross_entropy<__nv_bfloat16, 256><<<(unsigned)N, 256, 0, s>>>((__nv_bfloat16 *)logits, tgt,
                                                                   rowloss, V, ldz, inv_n, flag);
  else
    k_cross_entropy<float, 256><<<(unsigned)N, 256, 0, s>>>((float *)logits, tgt, rowloss, V, ldz,
                                                           inv_n, flag);
  count_launch();
}

// Mean of the row losses in a fixed order; a non-finite mean sets
// FLAG_NONFINITE.
__global__ void k_loss_reduce(const float *__restrict__ rowloss, int64_t N, float *loss, int *flag) {
  __shared__ double sh[1024];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < N; i += blockDim.x) s += (double)rowloss[i];
  sh[threadIdx.x] = s;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if ((int)threadIdx.x < o) sh[threadIdx.x] += sh[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    float l = (float)(sh[0] / (double)N);
    *loss = l;
    if (!isfinite(l)) atomicOr(flag, FLAG_NONFINITE);
  }
}
void loss_reduce(const float *rowloss, int64_t N, float *loss, int *flag, cudaStream_t s) {
  k_loss_reduce<<<1, 1024, 0, s>>>(rowloss, N, loss, flag);
  count_launch();
}

template <typename A>
__global__ void k_logits_out(const A *__restrict__ z, float *__restrict__ out, int64_t N, int V,
                             int64_t ldz) {
  int64_t n = N * V;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    out[i] = to_f(z[(i / V) * ldz + i % V]);
}
void logits_out(const void *logits, DType dt, float *out, int64_t N, int V, int64_t ldz,
                cudaStream_t s) {
  unsigned grid = min(cdiv(N * V, 256), 148u * 32);
  if (dt == DT_BF16)
    k_logits_out<<<grid, 256, 0, s>>>((const __nv_bfloat16 *)logits, out, N, V, ldz);
  else
    k_logits_out<<<grid, 256, 0, s>>>((const float *)logits, out, N, V, ldz);
  count_launch();
}

// -------------------------------------------------------------------- AdamW
// Hephaistos, Architecture at a glance (Optimizer); strata (AdamW, decoupled
// and bias-corrected).  m = b1 m + (1-b1) g; v = b2 v + (1-b2) g^2;
// p -= lr wd p + lr (m/bc1) / (sqrt(v/bc2) + eps), bc = 1 - beta^t.
// The flat buffers hold every tensor back to back, so one launch covers all.
// Skipped entirely when the step's flag is non-zero.  The per-step scalars
// (lr, wd, bc1, bc2) are read from device memory, written by k_set_hyper
// before the step, so a captured step graph replays with new values.
__global__ void k_set_hyper(float *hyper, float lr, float wd, float bc1, float bc2) {
  hyper[0] = lr;
  hyper[1] = wd;
  hyper[2] = bc1;
  hyper[3] = bc2;
}
void set_hyper(float *hyper, float lr, float wd, float bc1, float bc2, cudaStream_t s) {
  k_set_hyper<<<1, 1, 0, s>>>(hyper, lr, wd, bc1, bc2);
  count_launch();
}
__global__ void k_adamw(float *__restrict__ p, const float *__restrict__ g, float *__restrict__ m,
                        float *__restrict__ v, int64_t n, const float *__restrict__ hyper,
                        float b1, float b2, float eps, const int *flag) {
  if (*flag) return;
  const float lr = hyper[0], wd = hyper[1], bc1 = hyper[2], bc2 = hyper[3];
  int64_t n4 = n / 4;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    float4 pp = reinterpret_cast<float4 *>(p)[i];
    float4 gg = reinterpret_cast<const float4 *>(g)[i];
    float4 mm = reinterpret_cast<float4 *>(m)[i];
    float4 vv = reinterpret_cast<float4 *>(v)[i];
#define ADAM1(c)                                                         \
    mm.c = b1 * mm.c + (1.f - b1) * gg.c;                                \
    vv.c = b2 * vv.c + (1.f - b2) * gg.c * gg.c;                         \
    pp.c = pp.c - lr * wd * pp.c - lr * (mm.c / bc1) / (sqrtf(vv.c / bc2) + eps);
    ADAM1(x) ADAM1(y) ADAM1(z) ADAM1(w)
#undef ADAM1
    reinterpret_cast<float4 *>(p)[i] = pp;
    reinterpret_cast<float4 *>(m)[i] = mm;
    reinterpret_cast<float4 *>(v)[i] = vv;
  }
  for (int64_t i = n4 * 4 + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    float gi = g[i];
    float mi = b1 * m[i] + (1.f - b1) * gi;
    float vi = b2 * v[i] + (1.f - b2) * gi * gi;
    m[i] = mi;
    v[i] = vi;
    p[i] = p[i] - lr * wd * p[i] - lr * (mi / bc1) / (sqrtf(vi / bc2) + eps);
  }
}
void adamw(float *p, const float *g, float *m, float *v, int64_t n, const float *hyper, float b1,
           float b2, float eps, const int *flag, cudaStream_t s) {
  unsigned grid = min(cdiv(n / 4 + 1, 256), 148u * 8);
  k_adamw<<<grid, 256, 0, s>>>(p, g, m, v, n, hyper, b1, b2, eps, flag);
  count_launch();
}

// ------------------------------------------------------------ wgrad finish
// grad[r, c] = sum over splits k (in order) of part[k, r, cp(c)]; mode 1 maps
// the interleaved W1 | W3 columns back.  One block per row (grid-stride), 4
// columns per thread: an aligned group of 4 columns has 4 contiguous
// partial-sum columns in both modes (SWIGLU_BLOCK and h multiples of 4).
// Partial slabs of at most 32 MB (still in L2 from the GEMM that wrote
// them) go to k_wgrad_finish_flat instead: one thread per group of 4 columns
// over the whole gradient, four splits' loads in flight, the same sums in the
// same order.  Measured in the step (per-class CUDA events): the split-K
// finish of the 512-wide GQA workload 0.356 -> 0.323 ms, of the 256-wide one
// 0.262 -> 0.239 ms with the flat kernel; at 350M (slabs of 34-131 MB read
// mostly from HBM) this kernel is faster, 1.48 against 1.64 ms.
__global__ void k_wgrad_finish(const float *__restrict__ part, int splits, int64_t part_rows,
                               int64_t ldp, float *__restrict__ grad, int64_t rows, int64_t cols,
                               int mode, int64_t h, bool vec) {
  const int64_t pstride = part_rows * ldp;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const float *pr = part + r * ldp;
    float *gr = grad + r * cols;
    for (int64_t c = 4 * (int64_t)threadIdx.x; c < cols; c += 4 * (int64_t)blockDim.x) {
      if (vec && c + 4 <= cols) {
        const int64_t cp = mode == 1 ? ((c < h) ? w1_col(c) : w1_col(c - h) + SWIGLU_BLOCK) : c;
        float4 acc = *reinterpret_cast<const float4 *>(pr + cp);
        for (int k = 1; k < splits; k++) {
          const float4 q = *reinterpret_cast<const float4 *>(pr + k * pstride + cp);
          acc.x += q.x; acc.y += q.y; acc.z += q.z; acc.w += q.w;
        }
        *reinterpret_cast<float4 *>(gr + c) = acc;
      } else {
        for (int64_t cc = c; cc < c + 4 && cc < cols; cc++) {
          const int64_t cp = mode == 1 ? ((cc < h) ? w1_col(cc) : w1_col(cc - h) + SWIGLU_BLOCK) : cc;
          float acc = 0.f;
          for (int k = 0; k < splits; k++) acc += pr[k * pstride + cp];
          gr[cc] = acc;
        }
      }
    }
  }
}
LLM_DEV float4 add4(float4 a, float4 b) { return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w); }
__global__ void __launch_bounds__(256)
    k_wgrad_finish_flat(const float *__restrict__ part, int splits, int64_t part_rows, int64_t ldp,
                   float *__restrict__ grad, int64_t rows, int64_t cols, int mode, int64_t h,
                   bool vec) {
  const int64_t pstride = part_rows * ldp;
  const int64_t cq = (cols + 3) / 4, n = rows * cq;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / cq, c = 4 * (i - r * cq);
    const float *pr = part + r * ldp;
    float *gr = grad + r * cols;
    if (vec && c + 4 <= cols) {
      const int64_t cp = mode == 1 ? ((c < h) ? w1_col(c) : w1_col(c - h) + SWIGLU_BLOCK) : c;
      const float4 *p4 = reinterpret_cast<const float4 *>(pr + cp);
      const int64_t ps4 = pstride / 4;
      float4 acc = p4[0];
      int k = 1;
      for (; k + 4 <= splits; k += 4) {
        const float4 q1 = p4[k * ps4], q2 = p4[(k + 1) * ps4], q3 = p4[(k + 2) * ps4],
                     q4 = p4[(k + 3) * ps4];
        acc = add4(add4(add4(add4(acc, q1), q2), q3), q4);
      }
      for (; k < splits; k++) acc = add4(acc, p4[k * ps4]);
      *reinterpret_cast<float4 *>(gr + c) = acc;
    } else {
      for (int64_t cc = c; cc < c + 4 && cc < cols; cc++) {
        const int64_t cp = mode == 1 ? ((cc < h) ? w1_col(cc) : w1_col(cc - h) + SWIGLU_BLOCK) : cc;
        float acc = 0.f;
        for (int k = 0; k < splits; k++) acc += pr[k * pstride + cp];
        gr[cc] = acc;
      }
    }
  }
}
void wgrad_finish(const float *part, int splits, int64_t part_rows, int64_t ldp, float *grad,
                  int64_t rows, int64_t cols, int mode, int64_t h, cudaStream_t s) {
  const bool vec = ((uintptr_t)part & 15) == 0 && ((uintptr_t)grad & 15) == 0 && ldp % 4 == 0 &&
                   cols % 4 == 0 && (mode == 0 || h % 4 == 0) && (part_rows * ldp) % 4 == 0;
  if ((int64_t)splits * part_rows * ldp * 4 <= (int64_t(32) << 20)) {
    const int64_t groups = rows * ((cols + 3) / 4);
    const unsigned grid = (unsigned)std::min<int64_t>((groups + 255) / 256, 148 * 8);
    k_wgrad_finish_flat<<<grid, 256, 0, s>>>(part, splits, part_rows, ldp, grad, rows, cols, mode,
                                             h, vec);
  } else {
    const unsigned grid = (unsigned)std::min<int64_t>(rows, 148 * 8);
    k_wgrad_finish<<<grid, 256, 0, s>>>(part, splits, part_rows, ldp, grad, rows, cols, mode, h,
                                        vec);
  }
  count_launch();
}

// ------------------------------------------------------- embedding backward
// dwte[v,:] = sum_{i : tok_i = v} dx[i,:] in a fixed order, so the result
// does not depend on scheduling.  The token ids are sorted stably
// (least-significant-digit radix sort, 8-bit digits) together with their
// positions, giving each vocabulary row its run of positions in increasing
// order.  A run of at most EMB_LONG rows is summed in that order; a longer run
// (the frequent ids: Zipf puts thousands of rows on id 0) is cut into
// EMB_PARTS contiguous parts (part k = rows [c k / P, c (k + 1) / P) of its c
// rows), each part summed in order from zero by one warp, and the part sums
// are added in part order -- a fixed order with a dependent-load chain P
// times shorter (32 parts: ~80 rows per warp for the 2600-row run of the most
// frequent of 8192 Zipf(1.1) ids in 16384 tokens).
constexpr int RADIX_BLOCK = 256;
constexpr int EMB_LONG = 64, EMB_PARTS = 32;

__global__ void k_radix_hist(const int32_t *__restrict__ keys, int64_t N, int shift,
                             int32_t *__restrict__ hist, int nblk) {
  __shared__ int cnt[256];
  cnt[threadIdx.x] = 0;
  __syncthreads();
  int64_t i = (int64_t)blockIdx.x * RADIX_BLOCK + threadIdx.x;
  if (i < N) atomicAdd(&cnt[(keys[i] >> shift) & 255], 1);
  __syncthreads();
  hist[(int64_t)threadIdx.x * nblk + blockIdx.x] = cnt[threadIdx.x];
}
// Exclusive scan of n ints in place (one block of 1024 threads): chunks of
// SCAN_PER * 1024 (one chunk for the radix histogram of 16384 keys),
// SCAN_PER consecutive elements per thread, a warp-shuffle scan of the thread
// sums, then one warp scans the 32 warp totals; the running total of the
// chunks before carries over.  Integer sums: the result is exact.
constexpr int SCAN_PER = 16;
__global__ void __launch_bounds__(1024) k_scan_excl(int32_t *a, int64_t n) {
  __shared__ int32_t wtot[32];
  __shared__ int32_t carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int64_t base = 0; base < n; base += SCAN_PER * 1024) {
    const int64_t i0 = base + SCAN_PER * (int64_t)threadIdx.x;
    int32_t v[SCAN_PER], t = 0;
#pragma unroll
    for (int k = 0; k < SCAN_PER; k++) {
      v[k] = i0 + k < n ? a[i0 + k] : 0;
      t += v[k];
    }
    int32_t inc = t;  // inclusive scan of the thread sums within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t u = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += u;
    }
    if (lane == 31) wtot[warp] = inc;
    __syncthreads();
    if (warp == 0) {
      const int32_t w = wtot[lane];
      int32_t wi = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t u = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += u;
      }
      wtot[lane] = wi - w;  // exclusive warp offsets
    }
    __syncthreads();
    int32_t run = carry + wtot[warp] + inc - t;
#pragma unroll
    for (int k = 0; k < SCAN_PER; k++) {
      if (i0 + k < n) a[i0 + k] = run;
      run += v[k];
    }
    __syncthreads();  // every thread read carry and wtot
    if (threadIdx.x == 1023) carry = run;  // the last thread's running total is the chunk's end
    __syncthreads();
  }
}
__global__ void k_radix_scatter(const int32_t *__restrict__ keys, const int32_t *__restrict__ vals,
                                int64_t N, int shift, const int32_t *__restrict__ offs, int nblk,
                                int32_t *__restrict__ keys_out, int32_t *__restrict__ vals_out) {
  __shared__ int wcnt[RADIX_BLOCK / 32][256];
  int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < (RADIX_BLOCK / 32) * 256; i += RADIX_BLOCK) (&wcnt[0][0])[i] = 0;
  __syncthreads();
  int64_t i = (int64_t)blockIdx.x * RADIX_BLOCK + threadIdx.x;
  bool valid = i < N;
  int key = valid ? keys[i] : 0;
  int dig = valid ? ((key >> shift) & 255) : 256 + lane;  // invalid lanes never match
  unsigned peers = __match_any_sync(0xffffffffu, dig);
  int rank = __popc(peers & ((1u << lane) - 1));
  if (valid && rank == 0) wcnt[warp][dig] = __popc(peers);
  __syncthreads();
  if (valid) {
    int before = 0;
    for (int w = 0; w < warp; w++) before += wcnt[w][dig];
    int pos = offs[(int64_t)dig * nblk + blockIdx.x] + before + rank;
    keys_out[pos] = key;
    vals_out[pos] = vals ? vals[i] : (int32_t)i;
  }
}
__global__ void k_clamp_keys(const int32_t *__restrict__ tok, int32_t *__restrict__ keys,
                             int32_t *__restrict__ counts, int64_t N, int V) {
  int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= N) return;
  int t = tok[i];
  if (t < 0 || t >= V) t = 0;
  keys[i] = t;
  atomicAdd(&counts[t], 1);
}
// The vocabulary rows whose run is longer than EMB_LONG, listed in any order
// (each is summed the same way wherever it is listed).
__global__ void k_long_runs(const int32_t *__restrict__ offs, int V, int32_t *__restrict__ list,
                            int32_t *__restrict__ count) {
  const int v = blockIdx.x * blockDim.x + threadIdx.x;
  if (v < V && offs[v + 1] - offs[v] > EMB_LONG) list[atomicAdd(count, 1)] = v;
}
// Rows [p, e) of a run, in order, into s: lane = 4 columns (float4 c4), with
// the next 16 rows' loads in flight.
LLM_DEV float4 run_sum4(const int32_t *__restrict__ order, const float *__restrict__ dx, int d,
                        int c4, bool on, int p, int e) {
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  for (; p + 16 <= e; p += 16) {
    float4 t[16];
#pragma unroll
    for (int u = 0; u < 16; u++)
      t[u] = on ? reinterpret_cast<const float4 *>(dx + (int64_t)order[p + u] * d)[c4]
                : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int u = 0; u < 16; u++) {
      s.x += t[u].x; s.y += t[u].y; s.z += t[u].z; s.w += t[u].w;
    }
  }
  for (; p < e; p++) {
    if (!on) continue;
    const float4 t = reinterpret_cast<const float4 *>(dx + (int64_t)order[p] * d)[c4];
    s.x += t.x; s.y += t.y; s.z += t.z; s.w += t.w;
  }
  return s;
}
// Warp items (vocabulary row v, 128-column chunk), taken in order of v by a
// grid of whole blocks; lane = 4 columns.  Runs of at most EMB_LONG rows
// (and absent ids: zero rows); longer runs are left to k_embed_long.
__global__ void __launch_bounds__(256) k_embed_rows(const int32_t *__restrict__ order,
                                                   const int32_t *__restrict__ offs,
                                                   const float *__restrict__ dx,
                                                   float *__restrict__ dwte, int d, int V) {
  const int nchunk = (d + 127) / 128;
  const int64_t items = (int64_t)V * nchunk;
  const int lane = threadIdx.x & 31;
  const int64_t wid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t it = wid; it < items; it += nw) {
    const int v = (int)(it / nchunk), ch = (int)(it % nchunk);
    const int c4 = ch * 32 + lane;  // float4 column index
    const bool on = 4 * c4 < d;
    const int b = offs[v], e = offs[v + 1];
    if (e - b > EMB_LONG) continue;
    const float4 s = run_sum4(order, dx, d, c4, on, b, e);
    if (on) reinterpret_cast<float4 *>(dwte + (int64_t)v * d)[c4] = s;
  }
}
// Block (listed long run, 128-column chunk): warp k sums part k of the run,
// warp 0 adds the part sums in part order.
__global__ void __launch_bounds__(32 * EMB_PARTS)
    k_embed_long(const int32_t *__restrict__ list, const int32_t *__restrict__ count,
                 const int32_t *__restrict__ order, const int32_t *__restrict__ offs,
                 const float *__restrict__ dx, float *__restrict__ dwte, int d) {
  __shared__ float4 part[EMB_PARTS][32];
  if ((int)blockIdx.x >= *count) return;
  const int v = list[blockIdx.x];
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int c4 = blockIdx.y * 32 + lane;
  const bool on = 4 * c4 < d;
  const int b = offs[v];
  const int64_t c = offs[v + 1] - b;
  const int p0 = b + (int)(c * warp / EMB_PARTS), p1 = b + (int)(c * (warp + 1) / EMB_PARTS);
  part[warp][lane] = run_sum4(order, dx, d, c4, on, p0, p1);
  __syncthreads();
  if (warp == 0 && on) {
    float4 t = part[0][lane];
#pragma unroll
    for (int k = 1; k < EMB_PARTS; k++) {
      const float4 q = part[k][lane];
      t.x += q.x; t.y += q.y; t.z += q.z; t.w += q.w;
    }
    reinterpret_cast<float4 *>(dwte + (int64_t)v * d)[c4] = t;
  }
}
// Same sums and order for any d or alignment (one thread per column).
__global__ void k_embed_rows_scalar(const int32_t *__restrict__ order,
                                    const int32_t *__restrict__ offs, const float *__restrict__ dx,
                                    float *__restrict__ dwte, int d) {
  const int v = blockIdx.x;
  const int b = offs[v], e = offs[v + 1];
  const int64_t c = e - b;
  const int np = c > EMB_LONG ? EMB_PARTS : 1;
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    float total = 0.f;
    for (int k = 0; k < np; k++) {
      float sum = 0.f;
      for (int p = b + (int)(c * k / np); p < b + (int)(c * (k + 1) / np); p++)
        sum += dx[(int64_t)order[p] * d + j];
      total = k == 0 ? sum : total + sum;
    }
    dwte[(int64_t)v * d + j] = total;
  }
}
int64_t embed_bwd_scratch_ints(int64_t N, int V) {
  int64_t nblk = (N + RADIX_BLOCK - 1) / RADIX_BLOCK;
  return 4 * N + 256 * nblk + (V + 1) + 1 + (N / EMB_LONG + 1) + 64;
}
void embed_bwd(const int32_t *tok, const float *dx, float *dwte, int64_t N, int d, int V,
               int32_t *scratch, cudaStream_t s) {
  int nblk = (int)cdiv(N, RADIX_BLOCK);
  int32_t *k0 = scratch, *v0 = k0 + N, *k1 = v0 + N, *v1 = k1 + N;
  int32_t *hist = v1 + N, *offs = hist + 256 * (int64_t)nblk;
  int32_t *nlong = offs + V + 1, *list = nlong + 1;  // long runs: count, then vocabulary ids
  cudaMemsetAsync(offs, 0, sizeof(int32_t) * (V + 2), s);  // counts and the long-run count
  k_clamp_keys<<<cdiv(N, 256), 256, 0, s>>>(tok, k0, offs, N, V);
  count_launch();
  int bits = 1;
  while ((1 << bits) < V) bits++;
  const int32_t *kin = k0, *vin = nullptr;
  int32_t *kout = k1, *vout = v1;
  for (int shift = 0; shift < bits; shift += 8) {
    k_radix_hist<<<nblk, RADIX_BLOCK, 0, s>>>(kin, N, shift, hist, nblk);
    k_scan_excl<<<1, 1024, 0, s>>>(hist, 256 * (int64_t)nblk);
    k_radix_scatter<<<nblk, RADIX_BLOCK, 0, s>>>(kin, vin, N, shift, hist, nblk, kout, vout);
    count_launch(3);
    // ping-pong
    const int32_t *nk = kout, *nv = vout;
    kout = (kout == k1) ? k0 : k1;
    vout = (vout == v1) ? v0 : v1;
    kin = nk;
    vin = nv;
  }
  k_scan_excl<<<1, 1024, 0, s>>>(offs, V + 1);
  count_launch();
  if ((d & 3) == 0 && ((uintptr_t)dx & 15) == 0 && ((uintptr_t)dwte & 15) == 0) {
    k_long_runs<<<cdiv(V, 256), 256, 0, s>>>(offs, V, list, nlong);
    k_embed_rows<<<(unsigned)std::min<int64_t>(((int64_t)V * cdiv(d, 128) + 7) / 8, 148 * 8), 256,
                   0, s>>>(vin, offs, dx, dwte, d, V);
    const int64_t slots = std::max<int64_t>(1, N / EMB_LONG);  // at most N / EMB_LONG long runs
    k_embed_long<<<dim3((unsigned)slots, cdiv(d, 128)), 32 * EMB_PARTS, 0, s>>>(
        list, nlong, vin, offs, dx, dwte, d);
    count_launch(3);
  } else {
    k_embed_rows_scalar<<<V, min(256, ((d + 31) / 32) * 32), 0, s>>>(vin, offs, dx, dwte, d);
    count_launch();
  }
}

// ------------------------------------------------------------ initialisation
// Counter-based normal draws for llm_init: Philox4x32-10 (Salmon, Moraes,
// Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011) keyed
// by the seed, counter = element index; two 32-bit outputs give one normal by
// the Box-Muller transform.
__global__ void k_init(float *__restrict__ p, int64_t n, uint32_t k0, uint32_t k1, uint64_t base,
                       float std, int one) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    if (one) { p[i] = 1.f; continue; }
    uint64_t ctr = base + (uint64_t)i;
    uint32_t c[4] = {(uint32_t)ctr, (uint32_t)(ctr >> 32), 0u, 0u};
    philox4x32_10(c, k0, k1);
    double u1 = ((double)c[0] + 1.0) / 4294967296.0;  // (0, 1]
    double u2 = (double)c[1] / 4294967296.0;          // [0, 1)
    double z = sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
    p[i] = (float)(z * std);
  }
}
void init_params(float *p, int64_t n, uint64_t seed, uint64_t counter_base, float std,
                 int constant_one, cudaStream_t s) {
  unsigned grid = min(cdiv(n, 256), 148u * 8);
  k_init<<<grid, 256, 0, s>>>(p, n, (uint32_t)seed, (uint32_t)(seed >> 32), counter_base, std,
                              constant_one);
  count_launch();
}

// ------------------------------------------------------------------ dropout
// Hephaistos, Architecture at a glance (Regularization): inverted dropout,
// masks reused by the backward (the factor of an element is a pure function
// of its index, the site and the step, so the backward draws it again).
// A thread takes whole-batch groups of four consecutive elements, one
// generator call each: the context's elements are a.e0 .. a.e0 + n - 1, so
// group g holds its local elements 4g - a.e0 .. 4g - a.e0 + 3 that lie in
// [0, n) (a.e0 need not be a multiple of 4).
template <typename F>
LLM_DEV void for_drop_groups(const DropArgs &a, int64_t n, F f) {
  const uint32_t step = (uint32_t)*a.step;
  const uint64_t g0 = a.e0 >> 2;
  const int64_t ng = (int64_t)(((a.e0 + (uint64_t)n + 3) >> 2) - g0);
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < ng;
       t += (int64_t)gridDim.x * blockDim.x) {
    const uint64_t g = g0 + (uint64_t)t;
    const uint32_t keep = drop_bits4(a, g, step);
    const int64_t i0 = (int64_t)(g * 4) - (int64_t)a.e0;
#pragma unroll
    for (int j = 0; j < 4; j++)
      if (i0 + j >= 0 && i0 + j < n) f(i0 + j, (keep >> j) & 1u ? a.scale : 0.f);
  }
}
__global__ void k_drop_rows(float *__restrict__ x, int64_t n, const DropArgs a) {
  for_drop_groups(a, n, [&](int64_t i, float fac) { x[i] *= fac; });
}
__global__ void k_drop_add(const float *__restrict__ x, const float *__restrict__ y,
                           float *__restrict__ out, int64_t n, const DropArgs a) {
  for_drop_groups(a, n, [&](int64_t i, float fac) { out[i] = x[i] + fac * y[i]; });
}
template <typename A>
__global__ void k_drop_to_act(const float *__restrict__ dx, A *__restrict__ out, int64_t n,
                              const DropArgs a) {
  for_drop_groups(a, n, [&](int64_t i, float fac) { out[i] = from_f<A>(fac * dx[i]); });
}
// groups of the launch: at most n / 4 + 2 (n = 0 still launches one block)
static unsigned drop_grid(int64_t n) { return min(cdiv(n / 4 + 2, 256), 148u * 16); }
void drop_rows(float *x, int64_t n, const DropArgs &a, cudaStream_t s) {
  k_drop_rows<<<drop_grid(n), 256, 0, s>>>(x, n, a);
  count_launch();
}
void drop_add(const float *x, const float *y, float *out, int64_t n, const DropArgs &a,
              cudaStream_t s) {
  k_drop_add<<<drop_grid(n), 256, 0, s>>>(x, y, out, n, a);
  count_launch();
}
void drop_to_act(const float *dx, void *out, DType dt, int64_t n, const DropArgs &a,
                 cudaStream_t s) {
  const unsigned grid = drop_grid(n);
  if (dt == DT_BF16) k_drop_to_act<<<grid, 256, 0, s>>>(dx, (__nv_bfloat16 *)out, n, a);
  else k_drop_to_act<<<grid, 256, 0, s>>>(dx, (float *)out, n, a);
  count_launch();
}

// ------------------------------------------------------- gradient clipping
// MicroGPT in Rust, Gradient Clipping: the norm of all gradients together;
// when it exceeds max_norm every gradient is scaled by max_norm / norm.
// Squares are summed in double: per block in a fixed order over a fixed grid,
// then the block sums in order by one block, so the norm is reproducible.
constexpr int CLIP_BLOCKS = 148 * 4, CLIP_THREADS = 256;
LLM_DEV double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
LLM_DEV double block_sum_d(double v, double *ws) {  // ws: CLIP_THREADS / 32 doubles
  v = warp_sum_d(v);
  if ((threadIdx.x & 31) == 0) ws[threadIdx.x >> 5] = v;
  __syncthreads();
  double s = 0.0;
  if (threadIdx.x == 0)
    for (int w = 0; w < CLIP_THREADS / 32; w++) s += ws[w];
  return s;  // valid in thread 0
}
// g is 16-byte aligned; elements past the last whole float4 go to block 0.
__global__ void __launch_bounds__(CLIP_THREADS)
    k_sumsq(const float *__restrict__ g, int64_t n, double *__restrict__ part) {
  __shared__ double ws[CLIP_THREADS / 32];
  const int64_t n4 = n / 4;
  const float4 *g4 = reinterpret_cast<const float4 *>(g);
  double acc = 0.0;
  for (int64_t i = blockIdx.x * (int64_t)CLIP_THREADS + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * CLIP_THREADS) {
    const float4 v = g4[i];
    acc += (double)v.x * v.x + (double)v.y * v.y + (double)v.z * v.z + (double)v.w * v.w;
  }
  if (blockIdx.x == 0 && threadIdx.x < (int)(n & 3)) {
    const double v = g[n4 * 4 + threadIdx.x];
    acc += v * v;
  }
  const double s = block_sum_d(acc, ws);
  if (threadIdx.x == 0) part[blockIdx.x] = s;
}
__global__ void __launch_bounds__(CLIP_THREADS)
    k_clip_scale(const double *__restrict__ part, int nblk, float max_norm,
                 double *__restrict__ norm, float *__restrict__ scale) {
  __shared__ double ws[CLIP_THREADS / 32];
  double acc = 0.0;
  for (int i = threadIdx.x; i < nblk; i += CLIP_THREADS) acc += part[i];
  const double s = block_sum_d(acc, ws);
  if (threadIdx.x == 0) {
    const double nm = sqrt(s);
    *norm = nm;
    *scale = nm > (double)max_norm ? (float)((double)max_norm / nm) : 1.0f;
  }
}
__global__ void __launch_bounds__(CLIP_THREADS)
    k_scale_grads(float *__restrict__ g, int64_t n, const float *__restrict__ scale) {
  const float sc = *scale;
  const int64_t n4 = n / 4;
  float4 *g4 = reinterpret_cast<float4 *>(g);
  for (int64_t i = blockIdx.x * (int64_t)CLIP_THREADS + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * CLIP_THREADS) {
    float4 v = g4[i];
    v.x *= sc; v.y *= sc; v.z *= sc; v.w *= sc;
    g4[i] = v;
  }
  if (blockIdx.x == 0 && threadIdx.x < (int)(n & 3)) g[n4 * 4 + threadIdx.x] *= sc;
}
// randyGPT, Training: clipping by the L-infinity norm -- the largest |g| --
// with the same rule.  A maximum does not depend on the order it is taken in.
// A NaN anywhere makes the norm NaN (as the L2 sum does), so the scale stays 1.
LLM_DEV float nan_max(float a, float b) { return a != a ? a : ((b != b || b > a) ? b : a); }
__global__ void __launch_bounds__(CLIP_THREADS)
    k_absmax(const float *__restrict__ g, int64_t n, float *__restrict__ part) {
  __shared__ float ws[CLIP_THREADS / 32];
  float mx = 0.f;
  for (int64_t i = blockIdx.x * (int64_t)CLIP_THREADS + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * CLIP_THREADS)
    mx = nan_max(mx, fabsf(g[i]));
  for (int o = 16; o > 0; o >>= 1) mx = nan_max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) ws[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.f;
    for (int w = 0; w < CLIP_THREADS / 32; w++) m = nan_max(m, ws[w]);
    part[blockIdx.x] = m;
  }
}
__global__ void k_clip_scale_inf(const float *__restrict__ part, int nblk, float max_norm,
                                 double *__restrict__ norm, float *__restrict__ scale) {
  if (threadIdx.x != 0) return;
  float m = 0.f;
  for (int i = 0; i < nblk; i++) m = nan_max(m, part[i]);
  *norm = (double)m;
  *scale = m > max_norm ? (float)((double)max_norm / (double)m) : 1.0f;
}
void clip_grads_inf(float *g, int64_t n, float max_norm, double *part, double *norm,
                    float *scale, cudaStream_t s) {
  float *fpart = reinterpret_cast<float *>(part);  // CLIP_BLOCKS floats fit in the doubles
  k_absmax<<<CLIP_BLOCKS, CLIP_THREADS, 0, s>>>(g, n, fpart);
  k_clip_scale_inf<<<1, 32, 0, s>>>(fpart, CLIP_BLOCKS, max_norm, norm, scale);
  k_scale_grads<<<CLIP_BLOCKS, CLIP_THREADS, 0, s>>>(g, n, scale);
  count_launch(3);
}

// g *= sc (the mean of summed gradients: sc = 1 / ranks)
__global__ void __launch_bounds__(CLIP_THREADS)
    k_scale_grads_by(float *__restrict__ g, int64_t n, float sc) {
  const int64_t n4 = n / 4;
  float4 *g4 = reinterpret_cast<float4 *>(g);
  for (int64_t i = blockIdx.x * (int64_t)CLIP_THREADS + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * CLIP_THREADS) {
    float4 v = g4[i];
    v.x *= sc; v.y *= sc; v.z *= sc; v.w *= sc;
    g4[i] = v;
  }
  if (blockIdx.x == 0 && threadIdx.x < (int)(n & 3)) g[n4 * 4 + threadIdx.x] *= sc;
}
void scale_grads(float *g, int64_t n, float sc, cudaStream_t s) {
  k_scale_grads_by<<<CLIP_BLOCKS, CLIP_THREADS, 0, s>>>(g, n, sc);
  count_launch();
}
int clip_part_blocks() { return CLIP_BLOCKS; }
void clip_grads(float *g, int64_t n, float max_norm, double *part, double *norm, float *scale,
                cudaStream_t s) {
  k_sumsq<<<CLIP_BLOCKS, CLIP_THREADS, 0, s>>>(g, n, part);
  k_clip_scale<<<1, CLIP_THREADS, 0, s>>>(part, CLIP_BLOCKS, max_norm, norm, scale);
  k_scale_grads<<<CLIP_BLOCKS, CLIP_THREADS, 0, s>>>(g, n, scale);
  count_launch(3);
}

// Clipping with the gradient spread over ranks (sharded optimiser): each rank
// reduces its own range to one double -- the sum of squares (L2) or the
// largest |g| (L-infinity) -- the ranks combine those (sum or max), and every
// rank derives the same norm and scale from the combined value.
__global__ void __launch_bounds__(CLIP_THREADS)
    k_part_total(const double *__restrict__ part, int nblk, int accumulate, double *out) {
  __shared__ double ws[CLIP_THREADS / 32];
  double acc = 0.0;
  for (int i = threadIdx.x; i < nblk; i += CLIP_THREADS) acc += part[i];
  const double s = block_sum_d(acc, ws);
  if (threadIdx.x == 0) *out = accumulate ? *out + s : s;
}
__global__ void k_part_max(const float *__restrict__ part, int nblk, int accumulate, double *out) {
  if (threadIdx.x != 0) return;
  float m = 0.f;
  for (int i = 0; i < nblk; i++) m = nan_max(m, part[i]);
  const double dm = (double)m;
  if (!accumulate) *out = dm;
  else {
    const double o = *out;  // NaN wins, as in nan_max
    *out = o != o ? o : ((dm != dm || dm > o) ? dm : o);
  }
}
void grad_norm_part(float *g, int64_t n, float sc, int linf, int accumulate, double *part,
                    double *out, cudaStream_t s) {
  if (sc != 1.0f) scale_grads(g, n, sc, s);
  if (linf) {
    float *fpart = reinterpret_cast<float *>(part);
    k_absmax<<<CLIP_BLOCKS, CLIP_THREADS, 0, s>>>(g, n, fpart);
    k_part_max<<<1, 32, 0, s>>>(fpart, CLIP_BLOCKS, accumulate, out);
  } else {
    k_sumsq<<<CLIP_BLOCKS, CLIP_THREADS, 0, s>>>(g, n, part);
    k_part_total<<<1, CLIP_THREADS, 0, s>>>(part, CLIP_BLOCKS, accumulate, out);
  }
  count_launch(2);
}
__global__ void k_clip_from_total(const double *__restrict__ total, int linf, float max_norm,
                                  double *__restrict__ norm, float *__restrict__ scale) {
  if (threadIdx.x != 0) return;
  const double nm = linf ? *total : sqrt(*total);
  *norm = nm;
  *scale = nm > (double)max_norm ? (float)((double)max_norm / nm) : 1.0f;
}
void clip_from_total(float *g, int64_t n, const double *total, int linf, float max_norm,
                     double *norm, float *scale, cudaStream_t s) {
  k_clip_from_total<<<1, 32, 0, s>>>(total, linf, max_norm, norm, scale);
  k_scale_grads<<<CLIP_BLOCKS, CLIP_THREADS, 0, s>>>(g, n, scale);
  count_launch(2);
}

// -------------------------------------------------------------------- flags
__global__ void k_or_flag(const int *src, int *dst) { if (*src) atomicOr(dst, *src); }
void set_flag_zero(int *flag, cudaStream_t s) { cudaMemsetAsync(flag, 0, sizeof(int), s); }
void or_flag(const int *src, int *dst, cudaStream_t s) {
  k_or_flag<<<1, 1, 0, s>>>(src, dst);
  count_launch();
}

}  // namespace llm
