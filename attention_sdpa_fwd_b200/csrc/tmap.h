// Host-side creation of TMA tensor maps through the driver entry point
// (no link-time dependency on libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

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

// Encoded maps, cached by every argument of the encode call (base address,
// type, rank, extents, byte strides, box, swizzle mode).  A map is a pure function
// of those arguments, so a repeated call on the same tensor -- the usual case
// for a layer run step after step -- copies the cached 128-byte map instead of
// calling the driver.  Fixed size, round-robin replacement, one mutex.
struct TmapKey {
  const void* base;
  uint64_t dims[4];
  uint64_t strides[3];
  uint32_t box[2];
  int dt, rank, swizzle;
};

class TmapCache {
 public:
  static constexpr int kEntries = 64;
  bool find(const TmapKey& k, CUtensorMap* out) {
    std::lock_guard<std::mutex> lock(mu_);
    for (int i = 0; i < used_; ++i)
      if (memcmp(&keys_[i], &k, sizeof(TmapKey)) == 0) {
        *out = maps_[i];
        return true;
      }
    return false;
  }
  void put(const TmapKey& k, const CUtensorMap& m) {
    std::lock_guard<std::mutex> lock(mu_);
    const int i = used_ < kEntries ? used_++ : (next_++ % kEntries);
    keys_[i] = k;
    maps_[i] = m;
  }

 private:
  std::mutex mu_;
  TmapKey keys_[kEntries];
  CUtensorMap maps_[kEntries];
  int used_ = 0;
  unsigned next_ = 0;
};

inline TmapCache& tmap_cache() {
  static TmapCache c;
  return c;
}

inline TmapKey tmap_key(const void* base, CUtensorMapDataType dt, int rank, const cuuint64_t* dims,
                        const cuuint64_t* strides, const cuuint32_t* box, int swizzle) {
  TmapKey k;
  memset(&k, 0, sizeof(k));  // padding included: keys compare with memcmp
  k.base = base;
  for (int i = 0; i < rank; ++i) k.dims[i] = dims[i];
  for (int i = 0; i + 1 < rank; ++i) k.strides[i] = strides[i];
  k.box[0] = box[0];
  k.box[1] = box[1];
  k.dt = (int)dt;
  k.rank = rank;
  k.swizzle = swizzle;
  return k;
}

// One encode through the cache; false if the driver rejects the map.
inline bool encode_cached(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int rank,
                          const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                          CUtensorMapSwizzle swz) {
  const TmapKey key = tmap_key(base, dt, rank, dims, strides, box, (int)swz);
  if (tmap_cache().find(key, map)) return true;
  EncodeTiledFn fn = encode_tiled_fn();
  if (fn == nullptr) return false;
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, dt, (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  tmap_cache().put(key, *map);
  return true;
}

// 3-D map over a row-major [n2][n1][n0] tensor of `elem_bytes` elements:
// dim0 (contiguous) n0, dim1 n1 with stride s1 bytes, dim2 n2 with stride s2
// bytes; box {b0, b1, 1}; 128-byte swizzle when b0*elem_bytes == 128.
// Out-of-range elements of a box read as zero.  Returns false if the driver
// rejects the map (alignment, strides, box).
inline bool make_tmap_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem_bytes,
                         uint64_t n0, uint64_t n1, uint64_t n2, uint64_t s1, uint64_t s2, uint32_t b0,
                         uint32_t b1, bool swizzle128) {
  cuuint64_t dims[3] = {n0, n1, n2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, 1};
  (void)elem_bytes;
  return encode_cached(map, base, dt, 3, dims, strides, box,
                       swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
}

// 4-D map over a tensor of `elem_bytes` elements with dims {n0, n1, n2, n3}
// (dim0 contiguous) and byte strides s1, s2, s3 of dims 1..3, in any order of
// magnitude (e.g. head_dim, token, head, batch of a "bshd" tensor); box
// {b0, b1, 1, 1}; the given swizzle mode (or, with a bool, the 128-byte
// swizzle when asked).  Out-of-range elements of a box read as zero.  Returns
// false if the driver rejects the map.
inline bool make_tmap_4d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint64_t n0,
                         uint64_t n1, uint64_t n2, uint64_t n3, uint64_t s1, uint64_t s2, uint64_t s3,
                         uint32_t b0, uint32_t b1, CUtensorMapSwizzle swz) {
  cuuint64_t dims[4] = {n0, n1, n2, n3};
  cuuint64_t strides[3] = {s1, s2, s3};
  cuuint32_t box[4] = {b0, b1, 1, 1};
  return encode_cached(map, base, dt, 4, dims, strides, box, swz);
}
inline bool make_tmap_4d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint64_t n0,
                         uint64_t n1, uint64_t n2, uint64_t n3, uint64_t s1, uint64_t s2, uint64_t s3,
                         uint32_t b0, uint32_t b1, bool swizzle128) {
  return make_tmap_4d(map, base, dt, n0, n1, n2, n3, s1, s2, s3, b0, b1,
                      swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
}

}  // namespace sdpa
