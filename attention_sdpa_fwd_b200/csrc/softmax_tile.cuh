// Per-row pieces of the online softmax that both tensor-core kernels
// (flash_tc.cu, flash_persist.cu) run, one thread per query row = TMEM lane:
// the row max of a score tile, the exponentials packed to bf16 P with their
// sum, the rescale of the O accumulator in TMEM, the P store into TMEM and
// the O / l epilogue.  Scores are in log2 units (softmax with exp2); the
// rel_h term of the decomposed rel-pos bias is constant over a key-grid row
// and enters as one offset per row of the tile (goff).
#pragma once

#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "sm100.cuh"

namespace sdpa {
namespace tile {

using namespace sm100;

// Max over a tile of x (pairs) taken NG key-grid rows at a time (GW keys
// each), the row's goff added to each row's max: three-input max over pairs,
// four independent chains per row.
template <int NG, int GW>
__device__ __forceinline__ float row_max(const uint64_t* x2, const float* goff) {
  float mx = -INFINITY;
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    float a[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int i = 0; i < GW / 2; ++i) {
      float lo, hi;
      f2_split(x2[g * GW / 2 + i], lo, hi);
      a[i & 3] = max3(a[i & 3], lo, hi);
    }
    mx = fmaxf(mx, fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3])) + goff[g]);
  }
  return mx;
}

// p = 2^(x + goff - m) for the BN keys of a tile (key-grid rows of GW keys),
// packed to bf16 pairs in pk; returns the sum of the p (fp32, two chains).
// An x of -inf gives p = 0.
template <int BN, int GW>
__device__ __forceinline__ float exp_pack(const uint64_t* x2, const float* goff, float m_use, uint32_t* pk) {
  uint64_t sum2[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
  for (int i = 0; i < BN / 2; ++i) {
    const float nmo = goff[(2 * i) / GW] - m_use;
    const uint64_t y2 = f2_add(x2[i], f2(nmo, nmo));
    float lo, hi;
    f2_split(y2, lo, hi);
    const float p0 = ex2_approx(lo);
    const float p1 = ex2_approx(hi);
    sum2[i & 1] = f2_add(sum2[i & 1], f2(p0, p1));
    pk[i] = pack_bf16x2(p0, p1);
  }
  float a0, a1, b0, b1;
  f2_split(sum2[0], a0, a1);
  f2_split(sum2[1], b0, b1);
  return (a0 + a1) + (b0 + b1);
}

// The D accumulator columns of this thread's row of O, at o_addr in TMEM,
// times alpha (warp-collective; alpha is 1 where the max did not move).
template <int D>
__device__ __forceinline__ void rescale_o(uint32_t o_addr, float alpha) {
#pragma unroll
  for (int c0 = 0; c0 < D; c0 += 32) {
    uint32_t r[32];
    tmem_ld32(o_addr + c0, r);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
    tmem_st32(o_addr + c0, r);
  }
}

// P of a tile (BN keys as BN / 2 packed bf16 pairs) into TMEM at p_addr.
template <int BN>
__device__ __forceinline__ void store_p(uint32_t p_addr, const uint32_t* pk) {
#pragma unroll
  for (int c0 = 0; c0 < BN / 2; c0 += 8) tmem_st8p(p_addr + c0, pk + c0);
}

// Epilogue of a row: O / l (inv = 1 / l) from the D TMEM columns at o_addr,
// rounded to bf16 and written as 16-byte pieces to orow; the TMEM loads are
// warp-collective, the store is skipped for a row past Tq.
template <int D>
__device__ __forceinline__ void store_o_row(uint32_t o_addr, float inv, __nv_bfloat16* orow, bool row_valid) {
#pragma unroll
  for (int c0 = 0; c0 < D; c0 += 32) {
    uint32_t r[32];
    tmem_ld32(o_addr + c0, r);
    tmem_wait_ld();
    if (row_valid) {
#pragma unroll
      for (int c = 0; c < 32; c += 8) {
        uint4 v;
        v.x = pack_bf16x2(__uint_as_float(r[c + 0]) * inv, __uint_as_float(r[c + 1]) * inv);
        v.y = pack_bf16x2(__uint_as_float(r[c + 2]) * inv, __uint_as_float(r[c + 3]) * inv);
        v.z = pack_bf16x2(__uint_as_float(r[c + 4]) * inv, __uint_as_float(r[c + 5]) * inv);
        v.w = pack_bf16x2(__uint_as_float(r[c + 6]) * inv, __uint_as_float(r[c + 7]) * inv);
        *reinterpret_cast<uint4*>(orow + c0 + c) = v;
      }
    }
  }
}

// The same epilogue into shared memory for a TMA store: the row's D bf16
// values as 128-byte pieces of 64 columns (panel p at srow + p * panel_bytes),
// each in the 128-byte swizzle of a tensor map with 128-byte rows -- 16-byte
// chunk c at position c ^ (r & 7), r the row's index in its 1024-byte-aligned
// block (so a warp's 32 rows hit every bank group).
template <int D>
__device__ __forceinline__ void stage_o_row_sw128(uint32_t o_addr, float inv, uint8_t* srow, int r,
                                                  int panel_bytes) {
  static_assert(D % 64 == 0, "whole 64-column panels");
#pragma unroll
  for (int c0 = 0; c0 < D; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(o_addr + c0, v);
    tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < 32; c += 8) {
      uint4 w;
      w.x = pack_bf16x2(__uint_as_float(v[c + 0]) * inv, __uint_as_float(v[c + 1]) * inv);
      w.y = pack_bf16x2(__uint_as_float(v[c + 2]) * inv, __uint_as_float(v[c + 3]) * inv);
      w.z = pack_bf16x2(__uint_as_float(v[c + 4]) * inv, __uint_as_float(v[c + 5]) * inv);
      w.w = pack_bf16x2(__uint_as_float(v[c + 6]) * inv, __uint_as_float(v[c + 7]) * inv);
      const int col = c0 + c;  // first of the 8 columns
      const int chunk = (col & 63) >> 3;
      *reinterpret_cast<uint4*>(srow + (col >> 6) * panel_bytes + ((chunk ^ (r & 7)) << 4)) = w;
    }
  }
}

}  // namespace tile
}  // namespace sdpa
