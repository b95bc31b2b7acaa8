// Tensor-memory-accelerator (TMA) tile loads into 128-byte-swizzled shared
// memory, and the tcgen05 shared-memory descriptors that read such tiles.
//
// A 2-D bf16 tensor [rows][cols] (cols contiguous) is described by a tensor map
// whose box is 64 columns (128 bytes) by `box_rows` rows, with the 128-byte
// swizzle. A box lands in shared memory (1024-byte aligned) as box_rows rows of
// 128 bytes, the 16-byte chunk c of row r stored at chunk c ^ (r % 8): eight
// rows form one 1024-byte swizzle atom. Read by the tensor core:
//   K-major operand (rows = M or N, the 64 columns = K): SBO = 1024 between
//     8-row groups; the K step of 16 elements (32 bytes) advances the start
//     address by 32 bytes inside the 128-byte row (the swizzle is applied to the
//     final address bits, as the TMA unit applied it when writing), and a new
//     64-column box starts a new tile.
//   MN-major operand (rows = K, the 64 columns = M or N): SBO = 1024 between
//     8-row groups along K, LBO = the distance between 64-column boxes along
//     M/N; the K step of 16 rows advances the start by 2048 bytes.
// Loads only, never with cluster multicast.
#pragma once

#include <cuda.h>

#include "tc.cuh"

namespace muir {

// One 2-D box of `tmap` at element coordinates (x = column, y = row) into shared
// memory at dst, completing as transaction bytes on bar. x * 2 bytes must be a
// multiple of 16 (x a multiple of 8 for bf16).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* tmap, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

}  // namespace muir

// ---- host: tensor maps ------------------------------------------------------

namespace muir_host {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once through the runtime (no link
// dependency on the driver library). Returns nullptr if unavailable.
inline EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// Tensor map of a row-major bf16 matrix [rows][cols] (row pitch `pitch`
// elements, a multiple of 8) with a box of 64 columns x box_rows rows and the
// 128-byte swizzle. Rows or columns past the end read as zeros. Returns false if
// the encoder is unavailable or rejects the arguments.
inline bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t pitch,
                           uint32_t box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch * 2u};
  const cuuint32_t box[2] = {64u, box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace muir_host
