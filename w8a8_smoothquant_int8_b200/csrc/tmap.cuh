// Host-side helper: 2D tiled TMA descriptors (cuTensorMapEncodeTiled through
// the runtime's driver entry point, so the library needs no -lcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace sq {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn lookup_encode_fn() {
  void *p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<EncodeTiledFn>(p);
  return nullptr;
}

// looked up once per process (a function-local static: thread-safe)
static EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = lookup_encode_fn();
  return fn;
}

// 2D row-major tensor [outer, inner] of `esize`-byte elements, 128B swizzle
// unless another is given (the box's inner extent must fit the swizzle span).
static bool make_tmap(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int esize,
                      uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer,
                      CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * static_cast<uint64_t>(esize)};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D view of a row-major int8 matrix [rows, K] (K a multiple of 128) as
// K/128 blocks of 128 bytes: dims {128, rows, K/128}, strides {K, 128} bytes.
// A box {128, box_rows, box_kb} lands in shared memory as box_kb slabs of
// box_rows rows of 128 bytes (128-byte swizzle inside each slab), so one
// copy brings several K blocks of a tile.
static bool make_tmap_kblocks(CUtensorMap *m, const void *base, uint64_t K, uint64_t rows,
                              uint32_t box_rows, uint32_t box_kb) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || K % 128 != 0) return false;
  cuuint64_t dims[3] = {128, rows, K / 128};
  cuuint64_t strides[2] = {K, 128};
  cuuint32_t box[3] = {128, box_rows, box_kb};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace sq
