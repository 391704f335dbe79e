// Exact CUDA-core SDPA forward: every feature, fp32 and bf16 I/O, fp32 math.
//
// One warp owns one query row.  The warp walks the row's visible keys 32 at a
// time (one key per lane for the score, then the 32 probabilities are
// broadcast lane to lane for the value sum, each lane owning d/32 output
// columns), keeping the online-softmax state (running max m, running sum l,
// accumulator) so the T_q x T_kv score matrix is never stored -- the fusion
// the mlx-examples issue "segment_anything: fuse attention ..." asks for.
// The rel-pos projections rel_h[i,:] and rel_w[i,:] of the row are computed
// once into shared memory from the unscaled query (SAM add_decomposed_rel_pos,
// candle PR term_h / term_w) and added to each score before the max.
//
// This is the fp32 I/O path (no TF32 anywhere) and the reference-quality
// fallback for shapes the tensor-core kernels do not take.
#include <math.h>

#include "common.cuh"
#include "pdl_launch.cuh"
#include "sm100.cuh"

namespace sdpa {
namespace {

constexpr int kWarps = 4;

template <typename T, int D>
__device__ __forceinline__ float dot_row(const float* __restrict__ qs, const T* __restrict__ row) {
  // 16-byte vector loads of the key row, fp32 products with the query in smem.
  constexpr int kVec = 16 / sizeof(T);
  float acc = 0.f;
#pragma unroll
  for (int c0 = 0; c0 < D; c0 += kVec) {
    uint4 raw = *reinterpret_cast<const uint4*>(row + c0);
    const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
    for (int t = 0; t < kVec; ++t) acc = fmaf(qs[c0 + t], to_f32(e[t]), acc);
  }
  return acc;
}

template <typename T>
__device__ __forceinline__ float dot_any(const float* __restrict__ qs, const T* __restrict__ row, int d) {
  float acc = 0.f;
  for (int c = 0; c < d; ++c) acc = fmaf(qs[c], to_f32(row[c]), acc);
  return acc;
}

// VPRE (one output column per lane only): a chunk's V column is loaded at the
// top of the chunk, with the K rows (one round trip per chunk), at about twice
// the registers; the host takes it for launches of at most one wave at that
// occupancy, where latency, not the number of resident warps, sets the time.
template <typename T, int D, bool VPRE>
__global__ void __launch_bounds__(kWarps * 32) exact_kernel(Params p) {
  // launched behind the previous grid in the stream (programmatic
  // serialization): wait for it before any global-memory access
  sm100::grid_dep_launch();
  sm100::grid_dep_wait();
  extern __shared__ float smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long i = (long long)blockIdx.x * kWarps + warp;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  if (i >= p.Tq) return;  // warp-uniform; no block barrier follows
  const int hk = h / p.group;
  if (!dcheck_q(p, b, h, i)) return;  // debug builds: the row is in q / out
  const int per_warp = D + (p.use_rel ? (p.kh_n + p.kw_n) : 0);
  float* qs = smem + warp * per_warp;
  float* relh = qs + D;
  float* relw = relh + p.kh_n;

  const T* qrow = static_cast<const T*>(p.q) + q_off(p, b, h, i);
  for (int c = lane; c < D; c += 32) qs[c] = to_f32(qrow[c]);
  __syncwarp();

  if (p.use_rel) {
    // rel_h[i, a] = q_i . Rh[qh - a + Kh - 1], rel_w[i, a] = q_i . Rw[qw - a + Kw - 1]
    const int qh = (int)(i / p.qw_n), qw = (int)(i % p.qw_n);
    const T* Rh = static_cast<const T*>(p.rel_h);
    const T* Rw = static_cast<const T*>(p.rel_w);
    for (int a = lane; a < p.kh_n; a += 32) {
      const long long r = qh - a + p.kh_n - 1;
      relh[a] = dcheck_idx(p.err, r, p.qh_n + p.kh_n - 1) ? dot_any<T>(qs, Rh + r * D, D) : 0.f;
    }
    for (int a = lane; a < p.kw_n; a += 32) {
      const long long r = qw - a + p.kw_n - 1;
      relw[a] = dcheck_idx(p.err, r, p.qw_n + p.kw_n - 1) ? dot_any<T>(qs, Rw + r * D, D) : 0.f;
    }
    __syncwarp();
  }

  long long lo, hi;
  key_range(p, i, lo, hi);

  constexpr int CPL = D >= 32 ? D / 32 : 1;  // output columns per lane
  const bool owns_cols = (D >= 32) || (lane < D);
  const int col0 = D >= 32 ? lane * CPL : lane;

  const T* kb = static_cast<const T*>(p.k) + k_off(p, b, hk, 0);
  const T* vb = static_cast<const T*>(p.v) + v_off(p, b, hk, 0);
  const long long mrow = (long long)b * p.msb + (long long)h * p.msh + i * p.msq;

  float m = -INFINITY, l = 0.f;
  float acc[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) acc[c] = 0.f;

  for (long long j0 = lo; j0 < hi; j0 += 32) {
    const long long j = j0 + lane;
    const int nk = (int)((hi - j0) < 32 ? (hi - j0) : 32);
    // one column per lane: the chunk's V column goes out with the K rows, so
    // the chunk costs one round trip to memory instead of one per KB keys
    constexpr bool kVpre = VPRE && CPL == 1;
    float vcol[kVpre ? 32 : 1];
    if constexpr (kVpre) {
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const bool live = t < nk && owns_cols && dcheck_kv(p, b, hk, j0 + t);
        vcol[t] = live ? to_f32(vb[(j0 + t) * p.svt + col0]) : 0.f;
      }
    }
    float s = -INFINITY;
    if (j < hi && dcheck_kv(p, b, hk, j)) {
      s = p.scale * (p.k_vec16 ? dot_row<T, D>(qs, kb + j * p.skt) : dot_any<T>(qs, kb + j * p.skt, D));
      if (p.use_rel) s += relh[j / p.kw_n] + relw[j % p.kw_n];
      if (p.mask_kind == SDPA_MASK_ADD_FLOAT) {
        s += to_f32(static_cast<const T*>(p.mask)[mrow + j]);
      } else if (p.mask_kind == SDPA_MASK_BOOL) {
        if (static_cast<const uint8_t*>(p.mask)[mrow + j] == 0) s = -INFINITY;
      }
    }
    float cmax = s;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
    const float mnew = fmaxf(m, cmax);
    if (mnew == -INFINITY) continue;  // nothing visible yet (warp-uniform)
    const float corr = expf(m - mnew);  // 0 when m == -inf
    const float pj = expf(s - mnew);    // 0 for excluded keys
    float psum = pj;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
    l = l * corr + psum;
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[c] *= corr;
    if constexpr (kVpre) {
#pragma unroll
      for (int t = 0; t < 32; ++t) acc[0] = fmaf(__shfl_sync(0xffffffffu, pj, t), vcol[t], acc[0]);
      m = mnew;
      continue;
    }
    // the value sum over the chunk's keys, KB at a time: the KB V loads go
    // out together, then the FMAs (one round trip per KB keys; 16 when a lane
    // owns one column)
    constexpr int KB = CPL == 1 ? 16 : 8;
    for (int t0 = 0; t0 < nk; t0 += KB) {
      float pt[KB], vv[KB][CPL];
#pragma unroll
      for (int u = 0; u < KB; ++u) {
        const int t = t0 + u;  // < 32
        pt[u] = __shfl_sync(0xffffffffu, pj, t);
        const bool live = t < nk && owns_cols && dcheck_kv(p, b, hk, j0 + t);
        const T* vr = vb + (j0 + (live ? t : 0)) * p.svt + col0;
#pragma unroll
        for (int c = 0; c < CPL; ++c) vv[u][c] = live ? to_f32(vr[c]) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < KB; ++u)
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[c] = fmaf(pt[u], vv[u][c], acc[c]);
    }
    m = mnew;
  }

  const float inv = l > 0.f ? 1.f / l : 0.f;
  T* orow = static_cast<T*>(p.out) + o_off(p, b, h, i);
  if (owns_cols) {
#pragma unroll
    for (int c = 0; c < CPL; ++c) orow[col0 + c] = from_f32<T>(acc[c] * inv);
  }
  if (p.lse != nullptr && lane == 0)
    p.lse[((long long)b * p.Hq + h) * p.Tq + i] = l > 0.f ? m + logf(l) : -INFINITY;
}

template <typename T, int D, bool VPRE>
cudaError_t launch_tv(const Params& p, dim3 grid, size_t smem, cudaStream_t stream) {
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(exact_kernel<T, D, VPRE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_serialized(exact_kernel<T, D, VPRE>, grid, dim3(kWarps * 32), smem, stream, p);
}

template <typename T, int D>
cudaError_t launch_t(const Params& p, cudaStream_t stream) {
  const int per_warp = D + (p.use_rel ? (p.kh_n + p.kw_n) : 0);
  const size_t smem = sizeof(float) * (size_t)per_warp * kWarps;
  dim3 grid((unsigned)((p.Tq + kWarps - 1) / kWarps), (unsigned)p.Hq, (unsigned)p.B);
  if constexpr (D <= 32) {
    // the V-column prefetch holds about twice the registers (three CTAs per
    // SM): taken while the whole grid fits one wave at that occupancy
    const long long ctas = (long long)grid.x * grid.y * grid.z;
    if (ctas <= 3LL * num_sms()) return launch_tv<T, D, true>(p, grid, smem, stream);
  }
  return launch_tv<T, D, false>(p, grid, smem, stream);
}

}  // namespace

cudaError_t launch_exact(const Params& p, sdpa_dtype_t dtype, cudaStream_t stream) {
  if (dtype == SDPA_F32) {
    switch (p.d) {
      case 16: return launch_t<float, 16>(p, stream);
      case 64: return launch_t<float, 64>(p, stream);
      case 128: return launch_t<float, 128>(p, stream);
    }
  } else {
    switch (p.d) {
      case 16: return launch_t<__nv_bfloat16, 16>(p, stream);
      case 64: return launch_t<__nv_bfloat16, 64>(p, stream);
      case 128: return launch_t<__nv_bfloat16, 128>(p, stream);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace sdpa
