// Host-side creation of TMA tensor maps through the driver entry point
// (no link-time dependency on libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sdpa {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3-D map over a row-major [n2][n1][n0] tensor of `elem_bytes` elements:
// dim0 (contiguous) n0, dim1 n1 with stride s1 bytes, dim2 n2 with stride s2
// bytes; box {b0, b1, 1}; 128-byte swizzle when b0*elem_bytes == 128.
// Out-of-range elements of a box read as zero.  Returns false if the driver
// rejects the map (alignment, strides, box).
inline bool make_tmap_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem_bytes,
                         uint64_t n0, uint64_t n1, uint64_t n2, uint64_t s1, uint64_t s2, uint32_t b0,
                         uint32_t b1, bool swizzle128) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {n0, n1, n2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  (void)elem_bytes;
  CUresult r = fn(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 4-D map over a tensor of `elem_bytes` elements with dims {n0, n1, n2, n3}
// (dim0 contiguous) and byte strides s1, s2, s3 of dims 1..3, in any order of
// magnitude (e.g. head_dim, token, head, batch of a "bshd" tensor); box
// {b0, b1, 1, 1}; 128-byte swizzle when asked.  Out-of-range elements of a box
// read as zero.  Returns false if the driver rejects the map.
inline bool make_tmap_4d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint64_t n0,
                         uint64_t n1, uint64_t n2, uint64_t n3, uint64_t s1, uint64_t s2, uint64_t s3,
                         uint32_t b0, uint32_t b1, bool swizzle128) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[4] = {n0, n1, n2, n3};
  cuuint64_t strides[3] = {s1, s2, s3};
  cuuint32_t box[4] = {b0, b1, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace sdpa
