// head_dim 16 kernels for the SAM mask decoder's attention shapes (mlx-examples
// issue "segment_anything: fuse attention ...": the TwoWayTransformer's
// Attention, the same matmul/softmax/matmul without a bias; candle PR "SDPA
// with Relative Positional Embeddings": head_dim 16 support and a packed
// vector kernel for it).  At head_dim 16 a 128-row tcgen05 tile would sit
// mostly idle and the work is a stream over Q/O or K/V, so the kernels are
// shaped for memory traffic, with the arithmetic on mma.sync tensor-core
// tiles (16 rows x 8 or 16 keys) wherever there are enough keys to fill them:
//
//  * small_d_kernel / small_d_mma_kernel: one thread per query row for the
//    global traffic (a 32-byte Q row in, an O row out), 128 consecutive rows
//    of one (batch, head) per CTA -- or of several heads when the query axis
//    is short -- and K/V rounds staged in shared memory.  The scalar kernel
//    serves short key axes (image->token: 4096 rows against 8 keys); from 64
//    keys on, the tensor-core instance.
//
//  * split_kv_kernel: few query rows against a long key axis.  The key axis
//    of every (batch, head) is split over enough CTAs to cover the SMs; each
//    CTA stages its K/V part, every warp computes the partial (m, l,
//    unnormalised O) of each row over its slice of the keys on the tensor
//    cores, the warps' partials merge in the CTA and go to a workspace, and
//    the last CTA of a (batch, head) to finish, detected with an atomic
//    ticket, merges the parts: O = sum_k 2^(m_k-M) O_k / sum_k 2^(m_k-M) l_k.
//    When the key axis fits in 8 parts (token->image: 8 rows against 4096
//    keys), split_kv_cluster_kernel does the same with the parts in one
//    thread-block cluster, merged through distributed shared memory instead
//    of a global workspace.
//
// All take every mask kind and GQA; none takes the rel-pos bias (the exact
// kernel does).
#include <math.h>

#include <mutex>

#include <cooperative_groups.h>

#include "common.cuh"
#include "pdl_launch.cuh"
#include "sm100.cuh"

namespace sdpa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int D16 = 16;

__device__ __forceinline__ void bf16x8_to_f32(const uint4& raw, float* f) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// additive mask term (log2 units) or -inf for key j of row i; 0 when none
__device__ __forceinline__ float mask_term(const Params& p, long long mrow, long long i, long long j) {
  if ((p.mask_kind == SDPA_MASK_ADD_FLOAT || p.mask_kind == SDPA_MASK_BOOL) &&
      !(dcheck_idx(p.err, i, p.Tq) && dcheck_idx(p.err, j, p.Tkv)))
    return -INFINITY;  // debug builds: an index outside the mask skips the load
  if (p.mask_kind == SDPA_MASK_ADD_FLOAT)
    return __bfloat162float(static_cast<const __nv_bfloat16*>(p.mask)[mrow + j]) * kLog2e;
  if (p.mask_kind == SDPA_MASK_BOOL)
    return static_cast<const uint8_t*>(p.mask)[mrow + j] ? 0.f : -INFINITY;
  if (p.mask_kind == SDPA_MASK_CAUSAL || p.mask_kind == SDPA_MASK_SLIDING) {
    if (j > i + p.offset) return -INFINITY;
    if (p.mask_kind == SDPA_MASK_SLIDING && j <= i + p.offset - p.window) return -INFINITY;
  }
  return 0.f;
}

// ------------------------------------------------------------------ small_d
constexpr int kRowsPerCta = 128;
constexpr int kKeyChunk = 128;

// One thread per query row.  Heads are packed when the query axis is short:
// a CTA's 128 threads form 2^hp_log2 groups of `rows` = 128 >> hp_log2
// threads, group g taking query head blockIdx.y * groups + g, so a decoder
// shape with 8 query rows runs 16 heads per CTA instead of leaving 120 of
// 128 threads idle.  Each group stages its own head's keys, `rows` per
// round, in its own slice of the shared K/V chunk.
__global__ void __launch_bounds__(kRowsPerCta, 7) small_d_kernel(Params p, int hp_log2) {
  // launched behind the previous grid in the stream (programmatic
  // serialization): wait for it before any global-memory access
  sm100::grid_dep_launch();
  sm100::grid_dep_wait();
  __shared__ float4 sk[kKeyChunk][D16 / 4];  // every thread of a group reads the same key: broadcast
  __shared__ float4 sv[kKeyChunk][D16 / 4];
  const int rows = kRowsPerCta >> hp_log2;  // threads (query rows) per head
  const int g = threadIdx.x >> (7 - hp_log2), r = threadIdx.x & (rows - 1);
  const int h = (blockIdx.y << hp_log2) + g, b = blockIdx.z;
  const bool head_ok = h < p.Hq;
  const int hk = (head_ok ? h : 0) / p.group;
  const long long i = (long long)blockIdx.x * rows + r;
  const bool valid = head_ok && i < p.Tq;
  const long long zq = (long long)b * p.Hq + h;
  const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(p.q) + q_off(p, b, head_ok ? h : 0, valid ? i : 0);
  float q[D16];
  bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(qrow)), q);
  bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(qrow) + 1), q + 8);
  const float sl = p.scale * kLog2e;
#pragma unroll
  for (int c = 0; c < D16; ++c) q[c] *= sl;

  // key range shared by the CTA (causal / sliding; every group covers the
  // same query rows), then per row
  long long lo = 0, hi = p.Tkv;
  if (p.mask_kind == SDPA_MASK_CAUSAL || p.mask_kind == SDPA_MASK_SLIDING) {
    const long long first = (long long)blockIdx.x * rows;
    const long long last = min(first + rows, (long long)p.Tq) - 1;
    hi = min(hi, last + p.offset + 1);
    if (p.mask_kind == SDPA_MASK_SLIDING) lo = max(0LL, first + p.offset - p.window + 1);
  }
  const bool elementwise = p.mask_kind != SDPA_MASK_NONE;
  const long long mrow = (long long)b * p.msb + (long long)h * p.msh + i * p.msq;
  const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(p.k) + k_off(p, b, hk, 0);
  const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(p.v) + v_off(p, b, hk, 0);

  float m = -INFINITY, l = 0.f, acc[D16];
#pragma unroll
  for (int c = 0; c < D16; ++c) acc[c] = 0.f;

  // this group's slice of the chunk: keys [j0, j0 + rows) at rows sg .. sg + rows - 1
  const int sg = g * rows;
  for (long long j0 = lo; j0 < hi; j0 += rows) {
    const int n = (int)min((long long)rows, hi - j0);
    __syncthreads();
    // stage the chunk: each thread moves one key's K row and V row (32 B each)
    if (head_ok && r < n && dcheck_kv(p, b, hk, j0 + r)) {
      const long long j = j0 + r;
      float f[D16];
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(kb + j * p.skt)), f);
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(kb + j * p.skt) + 1), f + 8);
#pragma unroll
      for (int c = 0; c < D16; c += 4) sk[threadIdx.x][c / 4] = make_float4(f[c], f[c + 1], f[c + 2], f[c + 3]);
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(vb + j * p.svt)), f);
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(vb + j * p.svt) + 1), f + 8);
#pragma unroll
      for (int c = 0; c < D16; c += 4) sv[threadIdx.x][c / 4] = make_float4(f[c], f[c + 1], f[c + 2], f[c + 3]);
    }
    __syncthreads();
    if (!valid) continue;
    // eight keys at a time: scores, their max, one rescale, then the sums
    for (int t0 = 0; t0 < n; t0 += 8) {
      float sc[8];
      float cmax = -INFINITY;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int t = t0 + u;
        float x = -INFINITY;
        if (t < n) {
          x = 0.f;
#pragma unroll
          for (int c = 0; c < D16; c += 4) {
            const float4 k4 = sk[sg + t][c / 4];
            x = fmaf(q[c], k4.x, fmaf(q[c + 1], k4.y, fmaf(q[c + 2], k4.z, fmaf(q[c + 3], k4.w, x))));
          }
          if (elementwise) x += mask_term(p, mrow, i, j0 + t);
        }
        sc[u] = x;
        cmax = fmaxf(cmax, x);
      }
      if (cmax == -INFINITY) continue;
      if (cmax > m) {
        const float corr = sm100::ex2_approx(m - cmax);  // 0 when m == -inf
        l *= corr;
#pragma unroll
        for (int c = 0; c < D16; ++c) acc[c] *= corr;
        m = cmax;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float pj = sm100::ex2_approx(sc[u] - m);  // 0 for -inf
        l += pj;
        if (t0 + u < n) {
#pragma unroll
          for (int c = 0; c < D16; c += 4) {
            const float4 v4 = sv[sg + t0 + u][c / 4];
            acc[c] = fmaf(pj, v4.x, acc[c]);
            acc[c + 1] = fmaf(pj, v4.y, acc[c + 1]);
            acc[c + 2] = fmaf(pj, v4.z, acc[c + 2]);
            acc[c + 3] = fmaf(pj, v4.w, acc[c + 3]);
          }
        }
      }
    }
  }
  if (!valid || !dcheck_q(p, b, h, i)) return;
  const float inv = l > 0.f ? 1.f / l : 0.f;
  uint4 o0, o1;
  o0.x = pack2(acc[0] * inv, acc[1] * inv);
  o0.y = pack2(acc[2] * inv, acc[3] * inv);
  o0.z = pack2(acc[4] * inv, acc[5] * inv);
  o0.w = pack2(acc[6] * inv, acc[7] * inv);
  o1.x = pack2(acc[8] * inv, acc[9] * inv);
  o1.y = pack2(acc[10] * inv, acc[11] * inv);
  o1.z = pack2(acc[12] * inv, acc[13] * inv);
  o1.w = pack2(acc[14] * inv, acc[15] * inv);
  uint4* orow = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + o_off(p, b, h, i));
  orow[0] = o0;
  orow[1] = o1;
  if (p.lse) p.lse[zq * p.Tq + i] = l > 0.f ? m * kLn2 + logf(l) : -INFINITY;
}

// ------------------------------------------------------------------ tensor-core fragments
// mma.sync m16n8k16, bf16 operands, fp32 accumulate.  Thread (g, t) =
// (lane / 4, lane % 4) of a warp holds: of a 16x16 A tile, rows g and g + 8 at
// columns 2t, 2t + 1 (registers 0, 1) and 2t + 8, 2t + 9 (registers 2, 3); of
// a 16x8 B tile, column g at rows 2t, 2t + 1 (register 0) and 2t + 8, 2t + 9
// (register 1); of the 16x8 fp32 accumulator, rows g (c0, c1) and g + 8
// (c2, c3) at columns 2t, 2t + 1.  The S = Q K^T accumulators of two 8-key
// tiles, packed to bf16, are exactly the A operand of O += P V over those 16
// keys, so P never leaves registers.  Operands come from shared memory
// through ldmatrix.
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
               "{%8, %9}, {%0, %1, %2, %3};"
               : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// Byte offset of 16-byte half h (d 0..7 or 8..15) of row r in a [rows][16]
// bf16 array: halves swap every 4 rows, so the 8 rows one ldmatrix matrix
// reads hit all 32 banks once.
__device__ __forceinline__ uint32_t sw32(int r, int h) { return (uint32_t)(r * 32 + ((h ^ ((r >> 2) & 1)) << 4)); }

// The A operand (rows row0 .. row0 + 15) of a [rows][16] bf16 array at base.
__device__ __forceinline__ void ldsm_a(uint32_t (&a)[4], uint32_t base, int row0, int lane) {
  ldsm_x4(a, base + sw32(row0 + (lane & 7) + ((lane >> 3) & 1) * 8, lane >> 4));
}
// K of keys key0 .. key0 + 15 as the B operands of two 8-key tiles of S = Q K^T:
// r[0], r[1] for keys key0 .. + 7, r[2], r[3] for keys key0 + 8 .. + 15.
__device__ __forceinline__ void ldsm_k(uint32_t (&r)[4], uint32_t base, int key0, int lane) {
  ldsm_x4(r, base + sw32(key0 + (lane & 7) + (lane >> 4) * 8, (lane >> 3) & 1));
}
// V of keys key0 .. key0 + 15 as the B operands of O += P V: r[0], r[1] for
// value columns 0 .. 7, r[2], r[3] for columns 8 .. 15.
__device__ __forceinline__ void ldsm_v(uint32_t (&r)[4], uint32_t base, int key0, int lane) {
  ldsm_x4_t(r, base + sw32(key0 + (lane & 7) + ((lane >> 3) & 1) * 8, lane >> 4));
}

constexpr int kPartStride = 20;  // floats per row partial: 16 O, m, l, pad

// One warp's partial of 16 query rows over NT tiles of 16 keys of a staged
// part: S = Q K^T on the tensor cores from the staged bf16 rows (Q rows
// qrow0 .. qrow0 + 15 of q_s; keys key0 .. key0 + 16 NT - 1 of k_s / v_s, of
// which those at or past n are absent), the scores in log2 units with the
// mask (the rows are query rows row0 .. row0 + 15, staged key kk is key
// jg0 + kk of the problem), the softmax over the warp's keys, and O = P V with
// P packed straight from the S accumulators.  For every row row0 + i < Tq,
// writes the unnormalised O (16 values), the max m (log2 units) and the sum l
// to wp + i * kPartStride.
template <int NT>
__device__ __forceinline__ void warp_slice_partial(const Params& p, int b, int h, uint32_t q_s, int qrow0,
                                                   uint32_t k_s, uint32_t v_s, int key0, int n, long long jg0,
                                                   long long row0, float* wp, int lane, float sl) {
  const int g = lane >> 2, t = lane & 3;
  uint32_t qa[4];
  ldsm_a(qa, q_s, qrow0, lane);
  float x[NT][2][4];
#pragma unroll
  for (int c = 0; c < NT; ++c) {
    uint32_t kf[4];
    ldsm_k(kf, k_s, key0 + 16 * c, lane);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      x[c][u][0] = x[c][u][1] = x[c][u][2] = x[c][u][3] = 0.f;
      mma16816(x[c][u], qa, kf[2 * u], kf[2 * u + 1]);
    }
  }
  // scores in log2 units with the mask; absent keys and rows past Tq score
  // -inf (a warp slice of present keys without a mask: the scale and the row test)
  const long long mrow_base = (long long)b * p.msb + (long long)h * p.msh;
  if (p.mask_kind == SDPA_MASK_NONE && key0 + 16 * NT <= n) {
    const bool ok0 = row0 + g < p.Tq, ok1 = row0 + g + 8 < p.Tq;
#pragma unroll
    for (int c = 0; c < NT; ++c)
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) x[c][u][e] = ((e >> 1) ? ok1 : ok0) ? x[c][u][e] * sl : -INFINITY;
  } else
#pragma unroll
  for (int c = 0; c < NT; ++c)
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const long long row = row0 + g + (e >> 1) * 8;
        const int kk = key0 + 16 * c + 8 * u + 2 * t + (e & 1);
        float v = x[c][u][e] * sl;
        if (kk >= n || row >= p.Tq)
          v = -INFINITY;
        else
          v += mask_term(p, mrow_base + row * p.msq, row, jg0 + kk);
        x[c][u][e] = v;
      }
  float mr[2], lr[2] = {0.f, 0.f}, o[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    float mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < NT; ++c)
      mx = fmaxf(mx, fmaxf(fmaxf(x[c][0][2 * r], x[c][0][2 * r + 1]), fmaxf(x[c][1][2 * r], x[c][1][2 * r + 1])));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mr[r] = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  }
#pragma unroll
  for (int c = 0; c < NT; ++c) {
    uint32_t pa[4];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float mu = mr[r] == -INFINITY ? 0.f : mr[r];  // nothing visible: every p is 0
      const float p00 = sm100::ex2_approx(x[c][0][2 * r] - mu), p01 = sm100::ex2_approx(x[c][0][2 * r + 1] - mu);
      const float p10 = sm100::ex2_approx(x[c][1][2 * r] - mu), p11 = sm100::ex2_approx(x[c][1][2 * r + 1] - mu);
      lr[r] += (p00 + p01) + (p10 + p11);
      pa[r] = pack2(p00, p01);      // keys 2t, 2t + 1 of the 16
      pa[r + 2] = pack2(p10, p11);  // keys 8 + 2t, 9 + 2t
    }
    uint32_t vf[4];
    ldsm_v(vf, v_s, key0 + 16 * c, lane);
    mma16816(o[0], pa, vf[0], vf[1]);
    mma16816(o[1], pa, vf[2], vf[3]);
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int i = g + 8 * r;
    float L = lr[r];
    L += __shfl_xor_sync(0xffffffffu, L, 1);
    L += __shfl_xor_sync(0xffffffffu, L, 2);
    if (row0 + i >= p.Tq) continue;
    float* pr = wp + i * kPartStride;
    pr[2 * t] = o[0][2 * r];
    pr[2 * t + 1] = o[0][2 * r + 1];
    pr[8 + 2 * t] = o[1][2 * r];
    pr[9 + 2 * t] = o[1][2 * r + 1];
    if (t == 0) {
      pr[16] = mr[r];
      pr[17] = L;
    }
  }
}

// The CTA's partial of a row from its warps' partials ws[k * wstride] (k <
// 8, each O, m, l as warp_slice_partial writes them): warp-collective; lane
// c < 16 returns column c of O relative to the returned max M, with den the
// matching sum.
__device__ __forceinline__ void combine_warp_partials(const float* ws, int wstride, int lane, float& num,
                                                      float& M, float& den) {
  float Mk = -INFINITY, lk = 0.f;
  if (lane < 8) {
    Mk = ws[lane * wstride + 16];
    lk = ws[lane * wstride + 17];
  }
  M = lk > 0.f ? Mk : -INFINITY;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float wk = lk > 0.f ? sm100::ex2_approx(Mk - M) : 0.f;
  den = wk * lk;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  num = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float w_k = __shfl_sync(0xffffffffu, wk, k);
    if (lane < D16 && w_k > 0.f) num = fmaf(w_k, ws[k * wstride + lane], num);
  }
}

// ------------------------------------------------------------------ small_d on the tensor cores
// The small-d kernel for longer key axes: the same global traffic (one 32-byte
// Q row in and one O row out per thread, K/V rows of the round staged with
// 16-byte loads, heads packed when the query axis is short) with the
// arithmetic on the tensor cores: each warp's 32 rows are two 16-row tiles
// for S = Q K^T and O += P V (mma.sync from ldmatrix fragments), 16 keys at a
// time, with the online softmax on the accumulator fragments; O goes back to
// its rows through stmatrix and shared memory.  The scalar kernel above costs
// a fixed time per key for every row and keeps the short key axes (8 keys:
// 5.9 against 6.8 us for the decoder's image->token shape); from 64 keys on
// this one is much faster.
__device__ __forceinline__ void stsm_x4(uint32_t addr, const uint32_t (&r)[4]) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(r[0]), "r"(r[1]),
               "r"(r[2]), "r"(r[3])
               : "memory");
}

template <bool MASKED>
__global__ void __launch_bounds__(kRowsPerCta, MASKED ? 4 : 6) small_d_mma_kernel(Params p, int hp_log2) {
  sm100::grid_dep_launch();  // programmatic serialization when launched with it, as small_d_kernel
  sm100::grid_dep_wait();
  __shared__ __align__(128) uint8_t sq[kRowsPerCta * 32];  // Q rows, then O rows (bf16, swizzled)
  __shared__ __align__(128) uint8_t sk[kRowsPerCta * 32];  // staged K rows
  __shared__ __align__(128) uint8_t sv[kRowsPerCta * 32];  // staged V rows
  const int rows = kRowsPerCta >> hp_log2;  // threads (query rows) per head
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int grp = tid >> (7 - hp_log2), r = tid & (rows - 1);
  const int h = (blockIdx.y << hp_log2) + grp, b = blockIdx.z;
  const bool head_ok = h < p.Hq;
  const int hk = (head_ok ? h : 0) / p.group;
  const long long i = (long long)blockIdx.x * rows + r;
  const bool valid = head_ok && i < p.Tq;
  const uint32_t q_s = sm100::smem_u32(sq), k_s = sm100::smem_u32(sk), v_s = sm100::smem_u32(sv);

  // this thread's Q row into shared memory (zeros past Tq)
  {
    uint4 a = make_uint4(0, 0, 0, 0), c = a;
    if (valid && dcheck_q(p, b, h, i)) {
      const uint4* qrow = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.q) + q_off(p, b, h, i));
      a = __ldg(qrow);
      c = __ldg(qrow + 1);
    }
    *reinterpret_cast<uint4*>(sq + sw32(tid, 0)) = a;
    *reinterpret_cast<uint4*>(sq + sw32(tid, 1)) = c;
  }
  // the warp's two 16-row tiles: rows (within the CTA) 32 warp + 16 m + [0, 16)
  // of group grp_m, whose keys sit at rows grp_m * rows + [0, rows) of sk / sv
  int kbase[2];
  long long row0[2];
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    const int cr = 32 * warp + 16 * m;
    const int gm = cr >> (7 - hp_log2);
    kbase[m] = gm * rows;
    row0[m] = (long long)blockIdx.x * rows + (cr & (rows - 1));
  }
  const int hm[2] = {(int)(blockIdx.y << hp_log2) + ((32 * warp) >> (7 - hp_log2)),
                     (int)(blockIdx.y << hp_log2) + ((32 * warp + 16) >> (7 - hp_log2))};
  __syncwarp();
  uint32_t qa[2][4];
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    const int qr = 32 * warp + 16 * m + (lane & 7) + ((lane >> 3) & 1) * 8;
    ldsm_x4(qa[m], q_s + sw32(qr, lane >> 4));
  }

  // key range shared by the CTA (causal / sliding; every group covers the
  // same query rows)
  long long lo = 0, hi = p.Tkv;
  if (p.mask_kind == SDPA_MASK_CAUSAL || p.mask_kind == SDPA_MASK_SLIDING) {
    const long long first = (long long)blockIdx.x * rows;
    const long long last = min(first + rows, (long long)p.Tq) - 1;
    hi = min(hi, last + p.offset + 1);
    if (p.mask_kind == SDPA_MASK_SLIDING) lo = max(0LL, first + p.offset - p.window + 1);
  }
  const float sl = p.scale * kLog2e;
  const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(p.k) + k_off(p, b, hk, 0);
  const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(p.v) + v_off(p, b, hk, 0);
  float mrun[2][2], lrun[2][2], o[2][2][4];  // [tile][row g / g + 8], [tile][d half][acc]
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    mrun[m][0] = mrun[m][1] = -INFINITY;
    lrun[m][0] = lrun[m][1] = 0.f;
#pragma unroll
    for (int dh = 0; dh < 2; ++dh) o[m][dh][0] = o[m][dh][1] = o[m][dh][2] = o[m][dh][3] = 0.f;
  }

  for (long long j0 = lo; j0 < hi; j0 += rows) {
    const int n = (int)min((long long)rows, hi - j0);
    __syncthreads();
    // stage the round: each thread moves one key's K and V rows of its
    // group's head (zeros past the range, so no stale value meets a zero P)
    {
      uint4 k0 = make_uint4(0, 0, 0, 0), k1 = k0, v0 = k0, v1 = k0;
      if (head_ok && r < n && dcheck_kv(p, b, hk, j0 + r)) {
        const uint4* kr = reinterpret_cast<const uint4*>(kb + (j0 + r) * p.skt);
        const uint4* vr = reinterpret_cast<const uint4*>(vb + (j0 + r) * p.svt);
        k0 = __ldg(kr);
        k1 = __ldg(kr + 1);
        v0 = __ldg(vr);
        v1 = __ldg(vr + 1);
      }
      *reinterpret_cast<uint4*>(sk + sw32(tid, 0)) = k0;
      *reinterpret_cast<uint4*>(sk + sw32(tid, 1)) = k1;
      *reinterpret_cast<uint4*>(sv + sw32(tid, 0)) = v0;
      *reinterpret_cast<uint4*>(sv + sw32(tid, 1)) = v1;
    }
    __syncthreads();
    for (int k0 = 0; k0 < n; k0 += 16) {
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        if (row0[m] >= p.Tq || hm[m] >= p.Hq) continue;  // warp-uniform
        uint32_t kf[4], vf[4];
        ldsm_x4(kf, k_s + sw32(kbase[m] + k0 + (lane & 7) + (lane >> 4) * 8, (lane >> 3) & 1));
        ldsm_x4_t(vf, v_s + sw32(kbase[m] + k0 + (lane & 7) + ((lane >> 3) & 1) * 8, lane >> 4));
        float x[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        mma16816(x[0], qa[m], kf[0], kf[1]);
        mma16816(x[1], qa[m], kf[2], kf[3]);
        const long long mrow_base = (long long)b * p.msb + (long long)hm[m] * p.msh;
        if (!MASKED && k0 + 16 <= n && row0[m] + 16 <= p.Tq) {
          // a whole tile of present keys and rows: only the scale
#pragma unroll
          for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int e = 0; e < 4; ++e) x[u][e] *= sl;
        } else
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const long long row = row0[m] + g + (e >> 1) * 8;
            const int kk = k0 + 8 * u + 2 * t + (e & 1);
            float v = x[u][e] * sl;
            if (kk >= n || row >= p.Tq)
              v = -INFINITY;
            else if (MASKED)
              v += mask_term(p, mrow_base + row * p.msq, row, j0 + kk);
            x[u][e] = v;
          }
        uint32_t pa[4];
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          float tm = fmaxf(fmaxf(x[0][2 * rr], x[0][2 * rr + 1]), fmaxf(x[1][2 * rr], x[1][2 * rr + 1]));
          tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 1));
          tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 2));
          const float mnew = fmaxf(mrun[m][rr], tm);
          const float mu = mnew == -INFINITY ? 0.f : mnew;  // nothing visible yet: every p is 0
          const float alpha = sm100::ex2_approx(mrun[m][rr] - mu);
          mrun[m][rr] = mnew;
          const float p00 = sm100::ex2_approx(x[0][2 * rr] - mu), p01 = sm100::ex2_approx(x[0][2 * rr + 1] - mu);
          const float p10 = sm100::ex2_approx(x[1][2 * rr] - mu), p11 = sm100::ex2_approx(x[1][2 * rr + 1] - mu);
          lrun[m][rr] = lrun[m][rr] * alpha + ((p00 + p01) + (p10 + p11));
#pragma unroll
          for (int dh = 0; dh < 2; ++dh) {
            o[m][dh][2 * rr] *= alpha;
            o[m][dh][2 * rr + 1] *= alpha;
          }
          pa[rr] = pack2(p00, p01);      // keys 2t, 2t + 1 of the 16
          pa[rr + 2] = pack2(p10, p11);  // keys 8 + 2t, 9 + 2t
        }
        mma16816(o[m][0], pa, vf[0], vf[1]);
        mma16816(o[m][1], pa, vf[2], vf[3]);
      }
    }
  }

  // O / l as bf16 into the warp's Q rows (read only by this warp), then each
  // thread stores its own row
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    float inv[2];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      float L = lrun[m][rr];
      L += __shfl_xor_sync(0xffffffffu, L, 1);
      L += __shfl_xor_sync(0xffffffffu, L, 2);
      inv[rr] = L > 0.f ? 1.f / L : 0.f;
      const long long row = row0[m] + g + 8 * rr;
      if (t == 0 && p.lse && row < p.Tq && hm[m] < p.Hq)
        p.lse[((long long)b * p.Hq + hm[m]) * p.Tq + row] =
            L > 0.f ? mrun[m][rr] * kLn2 + logf(L) : -INFINITY;
    }
    const uint32_t of[4] = {pack2(o[m][0][0] * inv[0], o[m][0][1] * inv[0]),
                            pack2(o[m][0][2] * inv[1], o[m][0][3] * inv[1]),
                            pack2(o[m][1][0] * inv[0], o[m][1][1] * inv[0]),
                            pack2(o[m][1][2] * inv[1], o[m][1][3] * inv[1])};
    const int orr = 32 * warp + 16 * m + (lane & 7) + ((lane >> 3) & 1) * 8;
    stsm_x4(q_s + sw32(orr, lane >> 4), of);
  }
  __syncwarp();
  if (!valid || !dcheck_q(p, b, h, i)) return;
  uint4* orow = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + o_off(p, b, h, i));
  orow[0] = *reinterpret_cast<const uint4*>(sq + sw32(tid, 0));
  orow[1] = *reinterpret_cast<const uint4*>(sq + sw32(tid, 1));
}

// ------------------------------------------------------------------ split_kv
constexpr int kSplitThreads = 256;  // 8 warps: one query row per warp at a time
constexpr int kSplitChunk = 256;    // keys per CTA part (at most)

struct SplitArgs {
  Params p;
  int nsplit;      // parts per (batch, head)
  int chunk;       // keys per part
  float* ws_o;     // [B*Hq][nsplit][Tq][16]
  float2* ws_ml;   // [B*Hq][nsplit][Tq]  (m in log2 units, l)
  int* ws_cnt;     // [B*Hq] tickets, zero between launches
};

constexpr int kWsRows = 32;  // query rows per block of the workspace kernel (two 16-row tiles)

__global__ void __launch_bounds__(kSplitThreads, 3) split_kv_kernel(SplitArgs a) {
  sm100::grid_dep_launch();  // programmatic serialization, as in small_d_kernel
  sm100::grid_dep_wait();
  const Params& p = a.p;
  constexpr int kWarps = kSplitThreads / 32;
  static_assert(kSplitChunk == kSplitThreads && kSplitChunk == kWarps * 32, "a key per thread, 32 per warp");
  __shared__ __align__(128) uint8_t sk[kSplitChunk * 32];  // staged K rows (bf16, swizzled halves)
  __shared__ __align__(128) uint8_t sv[kSplitChunk * 32];
  __shared__ __align__(128) uint8_t sq[kWsRows * 32];
  __shared__ float warp_s[kWarps][kWsRows][kPartStride];
  __shared__ int s_last;
  const int part = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int hk = h / p.group;
  const long long zq = (long long)b * p.Hq + h;
  const long long j0 = (long long)part * a.chunk;
  const int n = (int)max(0LL, min((long long)a.chunk, (long long)p.Tkv - j0));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t k_s = sm100::smem_u32(sk), v_s = sm100::smem_u32(sv), q_s = sm100::smem_u32(sq);
  {
    // stage this part's K and V rows, one key per thread (zeros past the part)
    uint4 k0 = make_uint4(0, 0, 0, 0), k1 = k0, v0 = k0, v1 = k0;
    if (tid < n && dcheck_kv(p, b, hk, j0 + tid)) {
      const uint4* kr = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.k) + k_off(p, b, hk, j0 + tid));
      const uint4* vr = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.v) + v_off(p, b, hk, j0 + tid));
      k0 = __ldg(kr);
      k1 = __ldg(kr + 1);
      v0 = __ldg(vr);
      v1 = __ldg(vr + 1);
    }
    *reinterpret_cast<uint4*>(sk + sw32(tid, 0)) = k0;
    *reinterpret_cast<uint4*>(sk + sw32(tid, 1)) = k1;
    *reinterpret_cast<uint4*>(sv + sw32(tid, 0)) = v0;
    *reinterpret_cast<uint4*>(sv + sw32(tid, 1)) = v1;
  }
  const float sl = p.scale * kLog2e;
  // query rows in blocks of 32: stage them, every warp's partial over its 32
  // keys (tensor cores), then the CTA's partial of each row into the workspace
  for (int rb = 0; rb < p.Tq; rb += kWsRows) {
    if (tid < kWsRows) {
      uint4 q0 = make_uint4(0, 0, 0, 0), q1 = q0;
      if (rb + tid < p.Tq && dcheck_q(p, b, h, rb + tid)) {
        const uint4* qr = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.q) + q_off(p, b, h, rb + tid));
        q0 = __ldg(qr);
        q1 = __ldg(qr + 1);
      }
      *reinterpret_cast<uint4*>(sq + sw32(tid, 0)) = q0;
      *reinterpret_cast<uint4*>(sq + sw32(tid, 1)) = q1;
    }
    __syncthreads();  // (the first block's barrier also covers the K/V staging)
#pragma unroll
    for (int m = 0; m < kWsRows / 16; ++m)
      if (rb + 16 * m < p.Tq)
        warp_slice_partial<2>(p, b, h, q_s, 16 * m, k_s, v_s, 32 * warp, n, j0, rb + 16 * m, &warp_s[warp][16 * m][0],
                              lane, sl);
    __syncthreads();
    for (int i = warp; i < kWsRows && rb + i < p.Tq; i += kWarps) {
      float num, M, den;
      combine_warp_partials(&warp_s[0][i][0], kWsRows * kPartStride, lane, num, M, den);
      const long long slot = (zq * a.nsplit + part) * p.Tq + rb + i;
      if (!dcheck_idx(p.err, slot, (long long)p.B * p.Hq * a.nsplit * p.Tq)) continue;
      if (lane < D16) __stcg(a.ws_o + slot * D16 + lane, num);
      if (lane == 0) __stcg(a.ws_ml + slot, make_float2(M, den));
    }
    __syncthreads();  // the next block's staging overwrites sq and warp_s
  }
  // the last part of this (batch, head) to finish merges all parts.  The CTA
  // barrier orders every thread's stores before thread 0's gpu-scope fence
  // and ticket increment (fences are cumulative); the last arriver's fence
  // after its increment acquires the other parts' stores.
  __syncthreads();
  if (threadIdx.x == 0) {
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    s_last = dcheck_idx(p.err, zq, (long long)p.B * p.Hq) && atomicAdd(a.ws_cnt + zq, 1) == a.nsplit - 1;
    if (s_last) asm volatile("fence.acq_rel.gpu;" ::: "memory");
  }
  __syncthreads();
  if (!s_last) return;
  const long long base = zq * a.nsplit;  // first part slot of this (batch, head)
  for (int i = warp; i < p.Tq; i += kSplitThreads / 32) {
    // M = max over parts (one part per lane), then lanes (c, half) = (lane & 15,
    // lane >> 4) sum column c over every other part: independent loads, no
    // chain of round trips through the parts
    float M = -INFINITY;
    for (int k = lane; k < a.nsplit; k += 32) {
      const float2 ml = __ldcg(a.ws_ml + (base + k) * p.Tq + i);
      if (ml.y > 0.f) M = fmaxf(M, ml.x);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const int c = lane & 15;
    float den = 0.f, num = 0.f;
#pragma unroll 4
    for (int k = lane >> 4; k < a.nsplit; k += 2) {
      const long long slot = (base + k) * p.Tq + i;
      const float2 ml = __ldcg(a.ws_ml + slot);
      const float o = __ldcg(a.ws_o + slot * D16 + c);
      if (ml.y > 0.f) {
        const float w = exp2f(ml.x - M);
        den = fmaf(w, ml.y, den);
        num = fmaf(w, o, num);
      }
    }
    den += __shfl_xor_sync(0xffffffffu, den, 16);
    num += __shfl_xor_sync(0xffffffffu, num, 16);
    const float val = den > 0.f ? num / den : 0.f;
    const float nb = __shfl_down_sync(0xffffffffu, val, 1);
    if (lane < D16 && (lane & 1) == 0 && dcheck_q(p, b, h, i)) {
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + o_off(p, b, h, i);
      *reinterpret_cast<uint32_t*>(orow + lane) = pack2(val, nb);
    }
    if (lane == 0 && p.lse) p.lse[zq * p.Tq + i] = den > 0.f ? M * kLn2 + logf(den) : -INFINITY;
  }
  if (threadIdx.x == 0) a.ws_cnt[zq] = 0;  // ready for the next launch
}

// ------------------------------------------------------------------ split_kv over a cluster
// The same split of the key axis, with the parts of one (batch, head) in one
// thread-block cluster: each CTA leaves its partial (O, m, l) per query row
// in its own shared memory, and the parts merge through distributed shared
// memory -- no global workspace, fence or ticket, so the whole forward is one
// pass over K and V.  Used when the key axis fits in the cluster's parts
// (4096 keys).  Inside a part, K and V are staged as bf16 with 16-byte loads
// (CHUNK / 256 keys per thread), and each warp takes CHUNK / 8 of the keys:
// for every 16-row tile of query rows, S = Q K^T, the softmax over its keys
// and O = P V run on the tensor cores (mma.sync).  The warps' partials merge
// in the CTA, the CTAs' through the cluster.  Two sizes: 8 parts of 512 keys,
// and 4 parts of 1024 keys for grids beyond one wave of two CTAs per SM, where
// fewer and larger CTAs spread their fixed costs over more keys (token->image
// at batch 128: 128 against 187 us; at batch 4: 8.2 against 7.5 us).
constexpr int kClusterKeys = 4096;  // keys a cluster covers (at most)
constexpr int kRowsMax = 64;        // query rows the partial areas hold

template <int NCL>
struct ClLayout {
  static constexpr int kChunk = kClusterKeys / NCL;                 // keys per CTA (at most)
  static constexpr int kWarpKeys = kChunk / (kSplitThreads / 32);   // keys per warp
  static constexpr int kKeysPerThread = kChunk / kSplitThreads;
  // dynamic shared memory: K and V (bf16 rows), Q rows, the warps' partials,
  // the CTA's partials
  static constexpr int kK = 0, kV = kChunk * 32, kQ = 2 * kChunk * 32;
  static constexpr int kWarp = kQ + kRowsMax * 32;
  static constexpr int kPart = kWarp + (kSplitThreads / 32) * kRowsMax * kPartStride * 4;
  static constexpr int kBytes = kPart + kRowsMax * kPartStride * 4;
  static_assert(kChunk % kSplitThreads == 0 && kWarpKeys % 16 == 0, "whole keys per thread, 16-key tiles");
};

struct ClusterArgs {
  Params p;
  int ncl;    // parts = cluster size
  int chunk;  // keys per part
};

template <int NCL>
__global__ void __launch_bounds__(kSplitThreads, 2) split_kv_cluster_kernel(ClusterArgs a) {
  sm100::grid_dep_launch();  // programmatic serialization, as in small_d_kernel
  sm100::grid_dep_wait();
  namespace cg = cooperative_groups;
  using CL = ClLayout<NCL>;
  const Params& p = a.p;
  constexpr int kWarps = kSplitThreads / 32;
  extern __shared__ __align__(128) uint8_t cl_smem[];
  float* warp_s = reinterpret_cast<float*>(cl_smem + CL::kWarp);  // [kWarps][kRowsMax][kPartStride]
  float* part_s = reinterpret_cast<float*>(cl_smem + CL::kPart);  // [kRowsMax][kPartStride], read by the cluster
  const uint32_t k_s = sm100::smem_u32(cl_smem + CL::kK), v_s = sm100::smem_u32(cl_smem + CL::kV);
  const uint32_t q_s = sm100::smem_u32(cl_smem + CL::kQ);
  cg::cluster_group cluster = cg::this_cluster();
  const int part = (int)cluster.block_rank(), h = blockIdx.y, b = blockIdx.z;
  const int hk = h / p.group;
  const long long zq = (long long)b * p.Hq + h;
  const long long j0 = (long long)part * a.chunk;
  const int n = (int)max(0LL, min((long long)a.chunk, (long long)p.Tkv - j0));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int mrows = (p.Tq + 15) & ~15;  // query rows rounded up to whole 16-row tiles
  {
    // stage K and V rows tid, tid + 256, ... (zeros past the part) and Q rows
    // (zeros past Tq), all loads issued before the first store
    constexpr int KPT = CL::kKeysPerThread;
    uint4 kv[KPT][4], qv[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
      const int tk = tid + u * kSplitThreads;
      kv[u][0] = kv[u][1] = kv[u][2] = kv[u][3] = make_uint4(0, 0, 0, 0);
      if (tk < n && dcheck_kv(p, b, hk, j0 + tk)) {
        const uint4* kr = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.k) + k_off(p, b, hk, j0 + tk));
        const uint4* vr = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.v) + v_off(p, b, hk, j0 + tk));
        kv[u][0] = __ldg(kr);
        kv[u][1] = __ldg(kr + 1);
        kv[u][2] = __ldg(vr);
        kv[u][3] = __ldg(vr + 1);
      }
    }
    if (tid < mrows && tid < p.Tq && dcheck_q(p, b, h, tid)) {
      const uint4* qr = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.q) + q_off(p, b, h, tid));
      qv[0] = __ldg(qr);
      qv[1] = __ldg(qr + 1);
    }
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
      const int tk = tid + u * kSplitThreads;
      *reinterpret_cast<uint4*>(cl_smem + CL::kK + sw32(tk, 0)) = kv[u][0];
      *reinterpret_cast<uint4*>(cl_smem + CL::kK + sw32(tk, 1)) = kv[u][1];
      *reinterpret_cast<uint4*>(cl_smem + CL::kV + sw32(tk, 0)) = kv[u][2];
      *reinterpret_cast<uint4*>(cl_smem + CL::kV + sw32(tk, 1)) = kv[u][3];
    }
    if (tid < mrows) {
      *reinterpret_cast<uint4*>(cl_smem + CL::kQ + sw32(tid, 0)) = qv[0];
      *reinterpret_cast<uint4*>(cl_smem + CL::kQ + sw32(tid, 1)) = qv[1];
    }
  }
  __syncthreads();
  const float sl = p.scale * kLog2e;
  const int kw0 = warp * CL::kWarpKeys;  // this warp's keys within the part
  float* wp = warp_s + warp * kRowsMax * kPartStride;
  for (int row0 = 0; row0 < p.Tq; row0 += 16)
    warp_slice_partial<CL::kWarpKeys / 16>(p, b, h, q_s, row0, k_s, v_s, kw0, n, j0, row0, wp + row0 * kPartStride, lane,
                                       sl);
  __syncthreads();
  // the CTA's partial of row i from its warps' (warp i % 8 combines row i)
  for (int i = warp; i < p.Tq; i += kWarps) {
    float num, M, den;
    combine_warp_partials(warp_s + i * kPartStride, kRowsMax * kPartStride, lane, num, M, den);
    if (lane < D16) part_s[i * kPartStride + lane] = num;
    if (lane == 0) {
      part_s[i * kPartStride + 16] = M;
      part_s[i * kPartStride + 17] = den;
    }
  }
  // every part's partials are in its shared memory; row i is merged by part
  // i % ncl, which reads the row's partials from all parts (distributed
  // shared memory) and writes it: the merge is spread over the whole cluster
  cluster.sync();
  for (int i = part + a.ncl * warp; i < p.Tq; i += a.ncl * kWarps) {
    float Mk = -INFINITY, lk = 0.f;
    if (lane < a.ncl) {
      const float* pr = cluster.map_shared_rank(part_s, lane) + i * kPartStride;
      Mk = pr[16];
      lk = pr[17];
    }
    float M = lk > 0.f ? Mk : -INFINITY;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float wk = (lk > 0.f) ? sm100::ex2_approx(Mk - M) : 0.f;
    float den = wk * lk;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    // lane c (< 16) sums column c over the parts
    float num = 0.f;
#pragma unroll
    for (int k = 0; k < NCL; ++k) {
      const float w_k = __shfl_sync(0xffffffffu, wk, k);
      if (k < a.ncl && lane < D16 && w_k > 0.f)
        num = fmaf(w_k, cluster.map_shared_rank(part_s, k)[i * kPartStride + lane], num);
    }
    const float val = den > 0.f ? num / den : 0.f;
    const float nb = __shfl_down_sync(0xffffffffu, val, 1);
    if (lane < D16 && (lane & 1) == 0 && dcheck_q(p, b, h, i)) {
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + o_off(p, b, h, i);
      *reinterpret_cast<uint32_t*>(orow + lane) = pack2(val, nb);
    }
    if (lane == 0 && p.lse) p.lse[zq * p.Tq + i] = den > 0.f ? M * kLn2 + logf(den) : -INFINITY;
  }
  // keep every part's shared memory alive until every part has read it
  cluster.sync();
}

}  // namespace

int small_d_check(const Params& p, sdpa_dtype_t dtype) {
  if (dtype != SDPA_BF16 || p.d != 16) return SDPA_ERR_UNSUPPORTED;
  if (p.use_rel) return SDPA_ERR_UNSUPPORTED;
  if (p.B > 65535 || p.Hq > 65535) return SDPA_ERR_UNSUPPORTED;
  const uintptr_t m = reinterpret_cast<uintptr_t>(p.q) | reinterpret_cast<uintptr_t>(p.k) |
                      reinterpret_cast<uintptr_t>(p.v) | reinterpret_cast<uintptr_t>(p.out);
  if (m & 15) return SDPA_ERR_MISALIGNED;
  if (!strides_multiple_of(p, 8)) return SDPA_ERR_MISALIGNED;  // 16-byte row loads / stores
  return SDPA_OK;
}

// Heads per CTA, as a power of two: the most (up to 16, so at least 8 rows
// per head) whose query rows still fit the CTA's 128 threads, no more than
// there are query heads, and never so many that the grid drops below one
// CTA per SM (below a full wave, packing only lengthens each CTA: measured
// 2.7 against 2.9 us for 32 heads of 8 rows, and 10.6 against 4.5 us for
// 4096 heads packed 8 to a CTA).
static int small_d_pack_log2(const Params& p) {
  int hp = 0;  // (a packed query axis fits one block, so the grid is B x head groups)
  while (hp < 4 && ((long long)p.Tq << (hp + 1)) <= kRowsPerCta && (1 << (hp + 1)) <= p.Hq &&
         (long long)p.B * ((p.Hq + (1 << (hp + 1)) - 1) >> (hp + 1)) >= num_sms())
    ++hp;
  return hp;
}

// Key axes from this length on take the tensor-core small-d kernel.
constexpr int kSmallDMmaKeys = 64;

cudaError_t launch_small_d(const Params& p, cudaStream_t stream) {
  const bool mma = p.Tkv >= kSmallDMmaKeys;
  const int hp = mma ? min(small_d_pack_log2(p), 3) : small_d_pack_log2(p);  // >= 16 rows a head on the tensor cores
  const int rows = kRowsPerCta >> hp;
  dim3 grid((unsigned)((p.Tq + rows - 1) / rows), (unsigned)((p.Hq + (1 << hp) - 1) >> hp), (unsigned)p.B);
  if (!mma) return launch_serialized(small_d_kernel, grid, dim3(kRowsPerCta), 0, stream, p, hp);
  // The tensor-core instance runs long on grids that leave SM slots free
  // (1024 x 2048 rows x keys at 4 x 8 heads: 256 CTAs of 79 us): serialized
  // launches would place the next grid's waiting CTAs into those slots at
  // once, unevenly over the SMs, and that grid then ran 60 % longer.  Plain
  // launches place a grid on empty SMs (its grid_dep_* calls are no-ops then).
  if (p.mask_kind == SDPA_MASK_NONE)
    small_d_mma_kernel<false><<<grid, kRowsPerCta, 0, stream>>>(p, hp);
  else
    small_d_mma_kernel<true><<<grid, kRowsPerCta, 0, stream>>>(p, hp);
  return cudaGetLastError();
}

int split_kv_check(const Params& p, sdpa_dtype_t dtype) { return small_d_check(p, dtype); }

// Parts per (batch, head): enough CTAs for two per SM, parts of at most
// kSplitChunk keys.
static void split_shape(const Params& p, int* nsplit, int* chunk) {
  const long long bh = (long long)p.B * p.Hq;
  const long long want = (2LL * num_sms() + bh - 1) / bh;
  long long ns = max(1LL, min(want, (long long)(p.Tkv + 31) / 32));
  long long ch = (p.Tkv + ns - 1) / ns;
  if (ch > kSplitChunk) {
    ch = kSplitChunk;
    ns = (p.Tkv + ch - 1) / ch;
  }
  *nsplit = (int)ns;
  *chunk = (int)ch;
}

void split_kv_workspace_bytes(const Params& p, size_t* cnt_bytes, size_t* data_bytes) {
  int ns, ch;
  split_shape(p, &ns, &ch);
  const long long bh = (long long)p.B * p.Hq;
  const size_t nml = (size_t)bh * ns * p.Tq * sizeof(float2);
  const size_t no = (size_t)bh * ns * p.Tq * D16 * sizeof(float);
  *cnt_bytes = (size_t)bh * sizeof(int);
  *data_bytes = ((nml + 255) & ~size_t(255)) + no;
}

cudaError_t launch_split_kv_ws(const Params& p, int* cnt, void* data, cudaStream_t stream) {
  SplitArgs a;
  a.p = p;
  split_shape(p, &a.nsplit, &a.chunk);
  const long long bh = (long long)p.B * p.Hq;
  const size_t nml = (size_t)bh * a.nsplit * p.Tq * sizeof(float2);
  a.ws_cnt = cnt;
  a.ws_ml = static_cast<float2*>(data);
  a.ws_o = reinterpret_cast<float*>(static_cast<char*>(data) + ((nml + 255) & ~size_t(255)));
  dim3 grid((unsigned)a.nsplit, (unsigned)p.Hq, (unsigned)p.B);
  return launch_serialized(split_kv_kernel, grid, dim3(kSplitThreads), 0, stream, a);
}

template <int NCL>
static cudaError_t launch_cluster(const Params& p, cudaStream_t stream) {
  using CL = ClLayout<NCL>;
  ClusterArgs a;
  a.p = p;
  a.ncl = NCL;
  a.chunk = (p.Tkv + NCL - 1) / NCL;
  const size_t smem = (size_t)CL::kBytes;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [&] {
    attr = cudaFuncSetAttribute(split_kv_cluster_kernel<NCL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  });
  if (attr != cudaSuccess) return attr;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)NCL, (unsigned)p.Hq, (unsigned)p.B);
  cfg.blockDim = dim3(kSplitThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = (unsigned)NCL;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  // programmatic serialization: the kernel waits for the previous grid first
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, split_kv_cluster_kernel<NCL>, a);
}

cudaError_t launch_split_kv(const Params& p, cudaStream_t stream) {
  // one cluster of parts per (batch, head) when the key axis fits: 8 parts,
  // or 4 larger ones once 8-part clusters would not fit one wave of two CTAs
  // per SM
  if (p.Tq <= kRowsMax && p.Tkv >= 1 && p.Tkv <= (long long)kClusterKeys && p.B <= 65535 && p.Hq <= 65535) {
    if ((long long)p.B * p.Hq * 8 > 2LL * num_sms()) return launch_cluster<4>(p, stream);
    return launch_cluster<8>(p, stream);
  }
  size_t cb = 0, db = 0;
  split_kv_workspace_bytes(p, &cb, &db);
  void *cnt = nullptr, *data = nullptr;
  if (workspace_get(cb, db, &cnt, &data, stream) != SDPA_OK) return cudaErrorMemoryAllocation;
  return launch_split_kv_ws(p, static_cast<int*>(cnt), data, stream);
}

}  // namespace sdpa
