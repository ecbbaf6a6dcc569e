// Head-indexed tensor maps and TMEM load helpers of the tcgen05 attention
// kernels.
//
// A row of q|k|v (or of O, dO, dq|dk|dv) is a sequence of heads of hd
// bf16 values; the maps below describe it as [rows][heads][hd], so a tile is
// addressed as (0, head, row) and its box is always 64 values wide with
// 128-byte swizzle, the layout the kernels' UMMA descriptors expect.  For
// hd = 64 the box is exactly one head.  For hd = 32 the box reaches past the
// head's 32 values, which lie outside the tensor's innermost extent: a load
// fills them with zeros (so Q K^T, P V, dO V^T and the row sums dO . O are
// the head-32 values, and the products' columns 32..63 are zero) and a store
// skips them (only the head's own 32 columns are written).
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdint>

#include "common.cuh"

namespace llm {
namespace attn_maps {

LLM_DEV void tma_load_3d(uint32_t dst, const CUtensorMap *map, int x, int y, int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"((uint64_t)map), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}
// Bulk tensor store of a staged box (the caller commits the group).
LLM_DEV void tma_store_4d(const CUtensorMap *map, uint32_t src, int x, int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%1, %2, %3, %4}], [%5];" ::"l"(
          (uint64_t)map),
      "r"(x), "r"(y), "r"(z), "r"(w), "r"(src)
      : "memory");
}

// TMEM loads without their own wait (32x32b shape: lane = row, N columns
// of 32 bits), so several can be in flight; tmem_wait_regs waits for all of
// them and re-defines each loaded register after the wait, so no use of one
// can be scheduled before it.
template <int N>
LLM_DEV void tmem_ld_raw(uint32_t taddr, uint32_t (&r)[N]) {
  static_assert(N == 8 || N == 16 || N == 32, "8, 16 or 32 columns");
  if constexpr (N == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
  } else if constexpr (N == 16) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
  } else {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
  }
}
// A pair of equal loads (two TMEM regions of this thread's lane) under one wait.
template <int N>
LLM_DEV void tmem_ld_pair(uint32_t a, uint32_t b, float (&va)[N], float (&vb)[N]) {
  uint32_t ra[N], rb[N];
  tmem_ld_raw<N>(a, ra);
  tmem_ld_raw<N>(b, rb);
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < N; i++) {
    asm volatile("" : "+r"(ra[i]), "+r"(rb[i]));
    va[i] = __uint_as_float(ra[i]);
    vb[i] = __uint_as_float(rb[i]);
  }
}
LLM_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
template <int N>
LLM_DEV void tmem_after_wait(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; i++) asm volatile("" : "+r"(r[i]));
}

inline PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = [] {
    cudaDriverEntryPointQueryResult q;
    void *fn = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
    return (PFN_cuTensorMapEncodeTiled_v12000)fn;
  }();
  return encode;
}

// Loads: [rows][heads][hd] over a row-major [rows][ld] bf16 array (ld =
// heads * hd), box 64 x 1 head x box_rows rows.
inline bool head_map_load(CUtensorMap *map, const void *base, int hd, int64_t heads, int64_t rows,
                          int64_t ld, int box_rows) {
  auto encode = encoder();
  if (!encode || ((uintptr_t)base & 15) || (hd != 32 && hd != 64) || ld != heads * hd) return false;
  cuuint64_t dims[3] = {(cuuint64_t)hd, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)hd * 2, (cuuint64_t)ld * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t es[3] = {1, 1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Stores: [batches][T][heads][hd] over a row-major [batches * T][ld] bf16
// array, box 64 x 1 head x box_rows rows x 1 batch (rows past T, and a
// head-32 box's upper 32 values, are not written).
inline bool head_map_store(CUtensorMap *map, void *base, int hd, int64_t heads, int64_t T,
                           int64_t batches, int64_t ld, int box_rows) {
  auto encode = encoder();
  if (!encode || ((uintptr_t)base & 15) || (hd != 32 && hd != 64) || ld != heads * hd) return false;
  cuuint64_t dims[4] = {(cuuint64_t)hd, (cuuint64_t)heads, (cuuint64_t)T, (cuuint64_t)batches};
  cuuint64_t strides[3] = {(cuuint64_t)hd * 2, (cuuint64_t)ld * 2, (cuuint64_t)(ld * T * 2)};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace attn_maps
}  // namespace llm
