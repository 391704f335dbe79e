// head_dim 16 kernels for the SAM mask decoder's attention shapes (mlx-examples
// issue "segment_anything: fuse attention ...": the TwoWayTransformer's
// Attention, the same matmul/softmax/matmul without a bias; candle PR "SDPA
// with Relative Positional Embeddings": head_dim 16 support and a packed
// vector kernel for it).  At head_dim 16 a 128-row tensor-core tile would sit
// mostly idle and the work is a stream over Q/O or K/V, so both kernels run
// on CUDA cores and are shaped for HBM bandwidth:
//
//  * small_d_kernel: one thread per query row (16 values of q, the running
//    max/sum and a 16-wide accumulator in registers), 128 consecutive rows of
//    one (batch, head) per CTA so Q and O move as fully coalesced 32-byte
//    rows.  K/V of the kv head stream through shared memory in chunks as fp32
//    and are read by every thread as broadcasts.  Used when there are many
//    query rows (image->token: 4096 rows against 8 keys; self-attention).
//
//  * split_kv_kernel: few query rows against a long key axis (token->image: 8
//    rows against 4096 keys).  The key axis of every (batch, head) is split
//    over enough CTAs to cover the SMs; each CTA stages its K/V chunk in
//    shared memory, one warp per query row runs the online softmax over the
//    chunk (lanes stride the keys), and writes (m, l, unnormalised O) for its
//    part.  The last CTA of a (batch, head) to finish, detected with an
//    atomic ticket, merges the parts: O = sum_k 2^(m_k-M) O_k / sum_k 2^(m_k-M) l_k.
//    When the key axis fits in 8 parts, split_kv_cluster_kernel does the
//    same with the parts in one thread-block cluster, merged through
//    distributed shared memory instead of a global workspace.
//
// Both take every mask kind and GQA; neither takes the rel-pos bias (the
// exact kernel does).
#include <math.h>

#include <mutex>

#include <cooperative_groups.h>

#include "common.cuh"
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

__global__ void __launch_bounds__(kSplitThreads, 4) split_kv_kernel(SplitArgs a) {
  const Params& p = a.p;
  // key t's row as four float4 at [t][f ^ ((t >> 1) & 3)]: eight consecutive
  // lanes reading the same f of consecutive keys hit all 32 banks once
  __shared__ float4 sk[kSplitChunk][D16 / 4];
  __shared__ float4 sv[kSplitChunk][D16 / 4];
  __shared__ int s_last;
  const int part = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int hk = h / p.group;
  const long long zq = (long long)b * p.Hq + h;
  const long long j0 = (long long)part * a.chunk;
  const int n = (int)max(0LL, min((long long)a.chunk, (long long)p.Tkv - j0));
  const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(p.k) + k_off(p, b, hk, 0);
  const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(p.v) + v_off(p, b, hk, 0);
  for (int t = threadIdx.x; t < n; t += kSplitThreads) {
    if (!dcheck_kv(p, b, hk, j0 + t)) continue;
    float f[D16];
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(kb + (j0 + t) * p.skt)), f);
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(kb + (j0 + t) * p.skt) + 1), f + 8);
#pragma unroll
    for (int c = 0; c < D16; c += 4) sk[t][(c / 4) ^ ((t >> 1) & 3)] = make_float4(f[c], f[c + 1], f[c + 2], f[c + 3]);
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(vb + (j0 + t) * p.svt)), f);
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(vb + (j0 + t) * p.svt) + 1), f + 8);
#pragma unroll
    for (int c = 0; c < D16; c += 4) sv[t][(c / 4) ^ ((t >> 1) & 3)] = make_float4(f[c], f[c + 1], f[c + 2], f[c + 3]);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float sl = p.scale * kLog2e;
  for (int i = warp; i < p.Tq; i += kSplitThreads / 32) {
    const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(p.q) + q_off(p, b, h, i);
    float q[D16];
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(qrow)), q);
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(qrow) + 1), q + 8);
    const long long mrow = (long long)b * p.msb + (long long)h * p.msh + (long long)i * p.msq;
    float m = -INFINITY, l = 0.f, acc[D16];
#pragma unroll
    for (int c = 0; c < D16; ++c) acc[c] = 0.f;
    // this lane's keys (lane, lane + 32, ... : at most kSplitChunk / 32 of
    // them): scores, their max, then the sums
    float sc[kSplitChunk / 32];
#pragma unroll
    for (int u = 0; u < kSplitChunk / 32; ++u) {
      const int t = lane + 32 * u;
      float x = -INFINITY;
      if (t < n) {
        x = 0.f;
#pragma unroll
        for (int c = 0; c < D16; c += 4) {
          const float4 k4 = sk[t][(c / 4) ^ ((t >> 1) & 3)];
          x = fmaf(q[c], k4.x, fmaf(q[c + 1], k4.y, fmaf(q[c + 2], k4.z, fmaf(q[c + 3], k4.w, x))));
        }
        x = x * sl + mask_term(p, mrow, i, j0 + t);
      }
      sc[u] = x;
      m = fmaxf(m, x);
    }
    if (m != -INFINITY) {
#pragma unroll
      for (int u = 0; u < kSplitChunk / 32; ++u) {
        const int t = lane + 32 * u;
        const float pj = sm100::ex2_approx(sc[u] - m);  // 0 for -inf
        l += pj;
        if (t < n) {
#pragma unroll
          for (int c = 0; c < D16; c += 4) {
            const float4 v4 = sv[t][(c / 4) ^ ((t >> 1) & 3)];
            acc[c] = fmaf(pj, v4.x, acc[c]);
            acc[c + 1] = fmaf(pj, v4.y, acc[c + 1]);
            acc[c + 2] = fmaf(pj, v4.z, acc[c + 2]);
            acc[c + 3] = fmaf(pj, v4.w, acc[c + 3]);
          }
        }
      }
    }
    // combine the 32 lanes
    float M = m;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float w = (m == -INFINITY) ? 0.f : exp2f(m - M);
    l *= w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    // sum the 16 columns over the 32 lanes as a butterfly reduce-scatter:
    // at each step a lane keeps half of its columns and adds its partner's
    // half (8 + 4 + 2 + 1 + 1 shuffles instead of 16 x 5); lane pair
    // (2k, 2k+1) ends with column col = bits 4..1 of the lane
#pragma unroll
    for (int c = 0; c < D16; ++c) acc[c] *= w;
    const long long slot = (zq * a.nsplit + part) * p.Tq + i;
    const bool slot_ok = dcheck_idx(p.err, slot, (long long)p.B * p.Hq * a.nsplit * p.Tq);
    float r8[8], r4[4], r2[2], r1;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const bool hi = lane & 16;
      r8[k] = (hi ? acc[k + 8] : acc[k]) + __shfl_xor_sync(0xffffffffu, hi ? acc[k] : acc[k + 8], 16);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const bool hi = lane & 8;
      r4[k] = (hi ? r8[k + 4] : r8[k]) + __shfl_xor_sync(0xffffffffu, hi ? r8[k] : r8[k + 4], 8);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const bool hi = lane & 4;
      r2[k] = (hi ? r4[k + 2] : r4[k]) + __shfl_xor_sync(0xffffffffu, hi ? r4[k] : r4[k + 2], 4);
    }
    {
      const bool hi = lane & 2;
      r1 = (hi ? r2[1] : r2[0]) + __shfl_xor_sync(0xffffffffu, hi ? r2[0] : r2[1], 2);
    }
    r1 += __shfl_xor_sync(0xffffffffu, r1, 1);
    if ((lane & 1) == 0 && slot_ok) {
      const int col = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
      __stcg(a.ws_o + slot * D16 + col, r1);
    }
    if (lane == 0 && slot_ok) __stcg(a.ws_ml + slot, make_float2(M, l));
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
// in its own shared memory, and CTA 0 of the cluster merges them through
// distributed shared memory -- no global workspace, fence or ticket, so the
// whole forward is one pass over K and V.  Used when the key axis fits in 8
// parts of at most 512 keys.
constexpr int kClusterMax = 8;      // portable cluster size
constexpr int kClusterChunk = 512;  // keys per CTA (at most)
constexpr int kRowsMax = 64;        // query rows the partial area holds
constexpr int kPartStride = 20;     // floats per row partial: 16 O, m, l, pad

struct ClusterArgs {
  Params p;
  int ncl;    // parts = cluster size
  int chunk;  // keys per part
};

__global__ void __launch_bounds__(kSplitThreads, 2) split_kv_cluster_kernel(ClusterArgs a) {
  namespace cg = cooperative_groups;
  const Params& p = a.p;
  extern __shared__ float4 cl_smem[];
  float4 (*sk)[D16 / 4] = reinterpret_cast<float4 (*)[D16 / 4]>(cl_smem);
  float4 (*sv)[D16 / 4] = reinterpret_cast<float4 (*)[D16 / 4]>(cl_smem + kClusterChunk * (D16 / 4));
  float* part_s = reinterpret_cast<float*>(cl_smem + 2 * kClusterChunk * (D16 / 4));  // [Tq][2 halves][kPartStride]
  cg::cluster_group cluster = cg::this_cluster();
  const int part = (int)cluster.block_rank(), h = blockIdx.y, b = blockIdx.z;
  const int hk = h / p.group;
  const long long zq = (long long)b * p.Hq + h;
  const long long j0 = (long long)part * a.chunk;
  const int n = (int)max(0LL, min((long long)a.chunk, (long long)p.Tkv - j0));
  const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(p.k) + k_off(p, b, hk, 0);
  const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(p.v) + v_off(p, b, hk, 0);
  // stage the part: each thread moves the K and V rows (32 B each) of keys
  // tid and tid + 256, all eight 16-byte loads issued before the first
  // conversion
  static_assert(kClusterChunk == 2 * kSplitThreads, "two keys per thread");
  {
    uint4 raw[2][4];
    bool have[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int t = threadIdx.x + u * kSplitThreads;
      have[u] = t < n && dcheck_kv(p, b, hk, j0 + t);
      if (have[u]) {
        const uint4* kr = reinterpret_cast<const uint4*>(kb + (j0 + t) * p.skt);
        const uint4* vr = reinterpret_cast<const uint4*>(vb + (j0 + t) * p.svt);
        raw[u][0] = __ldg(kr);
        raw[u][1] = __ldg(kr + 1);
        raw[u][2] = __ldg(vr);
        raw[u][3] = __ldg(vr + 1);
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int t = threadIdx.x + u * kSplitThreads;
      if (!have[u]) continue;
      float f[D16];
      bf16x8_to_f32(raw[u][0], f);
      bf16x8_to_f32(raw[u][1], f + 8);
#pragma unroll
      for (int c = 0; c < D16; c += 4) sk[t][(c / 4) ^ ((t >> 1) & 3)] = make_float4(f[c], f[c + 1], f[c + 2], f[c + 3]);
      bf16x8_to_f32(raw[u][2], f);
      bf16x8_to_f32(raw[u][3], f + 8);
#pragma unroll
      for (int c = 0; c < D16; c += 4) sv[t][(c / 4) ^ ((t >> 1) & 3)] = make_float4(f[c], f[c + 1], f[c + 2], f[c + 3]);
    }
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float sl = p.scale * kLog2e;
  // Warp w takes two query rows, 2 (w & 3) + 8 r and the next, over one half
  // of the part's keys (w >> 2): every K and V row read from shared memory
  // serves two query rows, and each row's two key halves become two partials.
  const int kh = warp >> 2;
  for (int i0 = 2 * (warp & 3); i0 < p.Tq; i0 += 8) {
    const int ir[2] = {i0, min(i0 + 1, p.Tq - 1)};
    const bool live1 = i0 + 1 < p.Tq;
    float q[2][D16];
    long long mrow[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(p.q) + q_off(p, b, h, ir[r]);
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(qrow)), q[r]);
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(qrow) + 1), q[r] + 8);
      mrow[r] = (long long)b * p.msb + (long long)h * p.msh + (long long)ir[r] * p.msq;
    }
    // this lane's eight keys of the half (lane + 32 u): scores of both rows,
    // their maxima, then the sums
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f}, acc[2][D16];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int c = 0; c < D16; ++c) acc[r][c] = 0.f;
    float sc[2][8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int t = lane + 32 * (kh * 8 + u);
      float x0 = -INFINITY, x1 = -INFINITY;
      if (t < n) {
        x0 = 0.f;
        x1 = 0.f;
#pragma unroll
        for (int c = 0; c < D16; c += 4) {
          const float4 k4 = sk[t][(c / 4) ^ ((t >> 1) & 3)];
          x0 = fmaf(q[0][c], k4.x, fmaf(q[0][c + 1], k4.y, fmaf(q[0][c + 2], k4.z, fmaf(q[0][c + 3], k4.w, x0))));
          x1 = fmaf(q[1][c], k4.x, fmaf(q[1][c + 1], k4.y, fmaf(q[1][c + 2], k4.z, fmaf(q[1][c + 3], k4.w, x1))));
        }
        x0 = x0 * sl + mask_term(p, mrow[0], ir[0], j0 + t);
        x1 = x1 * sl + mask_term(p, mrow[1], ir[1], j0 + t);
      }
      sc[0][u] = x0;
      sc[1][u] = x1;
      m[0] = fmaxf(m[0], x0);
      m[1] = fmaxf(m[1], x1);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int t = lane + 32 * (kh * 8 + u);
      const float p0 = m[0] == -INFINITY ? 0.f : sm100::ex2_approx(sc[0][u] - m[0]);  // 0 for -inf
      const float p1 = m[1] == -INFINITY ? 0.f : sm100::ex2_approx(sc[1][u] - m[1]);
      l[0] += p0;
      l[1] += p1;
      if (t < n) {
#pragma unroll
        for (int c = 0; c < D16; c += 4) {
          const float4 v4 = sv[t][(c / 4) ^ ((t >> 1) & 3)];
          acc[0][c] = fmaf(p0, v4.x, acc[0][c]);
          acc[0][c + 1] = fmaf(p0, v4.y, acc[0][c + 1]);
          acc[0][c + 2] = fmaf(p0, v4.z, acc[0][c + 2]);
          acc[0][c + 3] = fmaf(p0, v4.w, acc[0][c + 3]);
          acc[1][c] = fmaf(p1, v4.x, acc[1][c]);
          acc[1][c + 1] = fmaf(p1, v4.y, acc[1][c + 1]);
          acc[1][c + 2] = fmaf(p1, v4.z, acc[1][c + 2]);
          acc[1][c + 3] = fmaf(p1, v4.w, acc[1][c + 3]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      // combine the 32 lanes: max, sum, and the 16 columns by a butterfly
      // reduce-scatter (lane pair (2k, 2k+1) ends with column bits 4..1 of the lane)
      float M = m[r];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      const float w = (m[r] == -INFINITY) ? 0.f : sm100::ex2_approx(m[r] - M);
      float lr = l[r] * w;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) lr += __shfl_xor_sync(0xffffffffu, lr, o);
      float r8[8], r4[4], r2[2], r1;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const bool hi = lane & 16;
        const float lo_v = acc[r][k] * w, hi_v = acc[r][k + 8] * w;
        r8[k] = (hi ? hi_v : lo_v) + __shfl_xor_sync(0xffffffffu, hi ? lo_v : hi_v, 16);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const bool hi = lane & 8;
        r4[k] = (hi ? r8[k + 4] : r8[k]) + __shfl_xor_sync(0xffffffffu, hi ? r8[k] : r8[k + 4], 8);
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const bool hi = lane & 4;
        r2[k] = (hi ? r4[k + 2] : r4[k]) + __shfl_xor_sync(0xffffffffu, hi ? r4[k] : r4[k + 2], 4);
      }
      {
        const bool hi = lane & 2;
        r1 = (hi ? r2[1] : r2[0]) + __shfl_xor_sync(0xffffffffu, hi ? r2[0] : r2[1], 2);
      }
      r1 += __shfl_xor_sync(0xffffffffu, r1, 1);
      if ((r == 1 && !live1) || !dcheck_idx(p.err, ir[r], kRowsMax)) continue;
      float* pr = part_s + (ir[r] * 2 + kh) * kPartStride;
      if ((lane & 1) == 0) pr[((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1)] = r1;
      if (lane == 0) {
        pr[16] = M;
        pr[17] = lr;
      }
    }
  }
  // every part's partials (two key halves per row) are in its shared memory;
  // row i is merged by part i % ncl, which reads the row's partials from all
  // parts (distributed shared memory) and writes it: the merge of a row of 8
  // query rows is spread over the whole cluster
  cluster.sync();
  {
    const int nslot = 2 * a.ncl;  // (part, half) partials per row
    for (int i = part + a.ncl * warp; i < p.Tq; i += a.ncl * (kSplitThreads / 32)) {
      float Mk = -INFINITY, lk = 0.f;
      if (lane < nslot) {
        const float* pr = cluster.map_shared_rank(part_s, lane >> 1) + (i * 2 + (lane & 1)) * kPartStride;
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
      // lane c (< 16) sums column c over the partials
      float num = 0.f;
#pragma unroll
      for (int k = 0; k < 2 * kClusterMax; ++k) {
        const float w_k = __shfl_sync(0xffffffffu, wk, k);
        if (k < nslot && lane < D16 && w_k > 0.f)
          num = fmaf(w_k, cluster.map_shared_rank(part_s, k >> 1)[(i * 2 + (k & 1)) * kPartStride + lane], num);
      }
      const float val = den > 0.f ? num / den : 0.f;
      const float nb = __shfl_down_sync(0xffffffffu, val, 1);
      if (lane < D16 && (lane & 1) == 0 && dcheck_q(p, b, h, i)) {
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + o_off(p, b, h, i);
        *reinterpret_cast<uint32_t*>(orow + lane) = pack2(val, nb);
      }
      if (lane == 0 && p.lse) p.lse[zq * p.Tq + i] = den > 0.f ? M * kLn2 + logf(den) : -INFINITY;
    }
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

cudaError_t launch_small_d(const Params& p, cudaStream_t stream) {
  const int hp = small_d_pack_log2(p);
  const int rows = kRowsPerCta >> hp;
  dim3 grid((unsigned)((p.Tq + rows - 1) / rows), (unsigned)((p.Hq + (1 << hp) - 1) >> hp), (unsigned)p.B);
  small_d_kernel<<<grid, kRowsPerCta, 0, stream>>>(p, hp);
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
  split_kv_kernel<<<grid, kSplitThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_split_kv(const Params& p, cudaStream_t stream) {
  // one cluster of up to 8 parts per (batch, head) when the key axis fits
  if (p.Tq <= kRowsMax && p.Tkv >= 1 && p.Tkv <= (long long)kClusterMax * kClusterChunk && p.B <= 65535 &&
      p.Hq <= 65535) {
    ClusterArgs a;
    a.p = p;
    a.ncl = kClusterMax;
    a.chunk = (p.Tkv + kClusterMax - 1) / kClusterMax;
    const size_t smem = (size_t)2 * kClusterChunk * (D16 / 4) * sizeof(float4) + (size_t)kRowsMax * 2 * kPartStride * 4;
    static std::once_flag once;
    static cudaError_t attr = cudaSuccess;
    std::call_once(once, [&] {
      attr = cudaFuncSetAttribute(split_kv_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    });
    if (attr != cudaSuccess) return attr;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.ncl, (unsigned)p.Hq, (unsigned)p.B);
    cfg.blockDim = dim3(kSplitThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)a.ncl;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, split_kv_cluster_kernel, a);
  }
  size_t cb = 0, db = 0;
  split_kv_workspace_bytes(p, &cb, &db);
  void *cnt = nullptr, *data = nullptr;
  if (workspace_get(cb, db, &cnt, &data, stream) != SDPA_OK) return cudaErrorMemoryAllocation;
  return launch_split_kv_ws(p, static_cast<int*>(cnt), data, stream);
}

}  // namespace sdpa
