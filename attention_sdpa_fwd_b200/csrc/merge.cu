// sdpa_merge: combine attention results over disjoint key subsets of the same
// queries into the result over their union (split-key / KV-chunked attention).
//
// Part i holds out_i = sum_j p_ij v_j / l_i and its log-sum-exp
// lse_i = m_i + log l_i over its own keys.  Over the union the normaliser is
// L = log sum_i exp(lse_i) and part i's unnormalised sum is exp(lse_i) out_i,
// so out = sum_i exp(lse_i - L) out_i -- the softmax numerators of every key
// summed (Axon PR "Add scaled_dot_product_attention": softmax(Q.K^T*scale +
// mask).V over the whole key axis).  A row with no visible key in any part
// gets zeros and L = -inf.
//
// HBM-bound elementwise work: one thread per 16-byte piece of an output row
// reads that piece of every part and the parts' lse of its row (a row's
// pieces are consecutive threads of one CTA, so the lse loads hit L1).
#include <math.h>

#include "common.cuh"

namespace sdpa {
namespace {

constexpr int kMergeThreads = 256;

struct MergeArgs {
  const void* outs[kMaxMergeParts];
  const float* lses[kMaxMergeParts];
  int n;
  void* out;
  float* lse;
  long long rows;  // B * Hq * Tq
  int pieces;      // 16-byte pieces per row
};

template <typename T>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const MergeArgs a) {
  constexpr int E = 16 / sizeof(T);  // elements per piece
  const long long idx = (long long)blockIdx.x * kMergeThreads + threadIdx.x;
  const long long row = idx / a.pieces;
  const int piece = (int)(idx - row * a.pieces);
  const bool live = row < a.rows;
  float s[kMaxMergeParts];
  float top = -INFINITY;
#pragma unroll
  for (int i = 0; i < kMaxMergeParts; ++i) {
    s[i] = (live && i < a.n) ? __ldg(a.lses[i] + row) : -INFINITY;
    top = fmaxf(top, s[i]);
  }
  float tot = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxMergeParts; ++i) {
    s[i] = (top == -INFINITY) ? 0.f : expf(s[i] - top);  // exp(-inf) = 0 for empty parts
    tot += s[i];
  }
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  if (live && top != -INFINITY) {
    const float inv = 1.f / tot;
#pragma unroll
    for (int i = 0; i < kMaxMergeParts; ++i) {
      if (i < a.n && s[i] > 0.f) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(static_cast<const T*>(a.outs[i]) + row * a.pieces * E) + piece);
        const T* v = reinterpret_cast<const T*>(&raw);
        const float w = s[i] * inv;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(w, to_f32(v[e]), acc[e]);
      }
    }
  }
  // every thread of the CTA has read its parts (out / lse may be part 0)
  __syncthreads();
  if (!live) return;
  uint4 res;
  T* r = reinterpret_cast<T*>(&res);
#pragma unroll
  for (int e = 0; e < E; ++e) r[e] = from_f32<T>(acc[e]);
  reinterpret_cast<uint4*>(static_cast<T*>(a.out) + row * a.pieces * E)[piece] = res;
  if (piece == 0 && a.lse) a.lse[row] = top == -INFINITY ? -INFINITY : top + logf(tot);
}

}  // namespace

cudaError_t launch_merge(const void* const* outs, const float* const* lses, int n, void* out, float* lse,
                         sdpa_dtype_t dtype, long long rows, int d, cudaStream_t stream) {
  MergeArgs a;
  memset(&a, 0, sizeof(a));
  for (int i = 0; i < n; ++i) {
    a.outs[i] = outs[i];
    a.lses[i] = lses[i];
  }
  a.n = n;
  a.out = out;
  a.lse = lse;
  a.rows = rows;
  const int esz = dtype == SDPA_F32 ? 4 : 2;
  a.pieces = d * esz / 16;
  const long long threads = rows * a.pieces;
  const unsigned blocks = (unsigned)((threads + kMergeThreads - 1) / kMergeThreads);
  if (dtype == SDPA_F32)
    merge_kernel<float><<<blocks, kMergeThreads, 0, stream>>>(a);
  else
    merge_kernel<__nv_bfloat16><<<blocks, kMergeThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace sdpa
