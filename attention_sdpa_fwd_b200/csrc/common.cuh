// Shared host/device definitions of libsdpa's kernels (not part of the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sdpa.h"

namespace sdpa {

// Everything a kernel needs, filled on the host after validation.
struct Params {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* lse;        // optional [B, Hq, Tq]
  int B, Hq, Hkv, Tq, Tkv, d;
  int group;         // Hq / Hkv
  float scale;
  int mask_kind;
  long long offset, window;
  const void* mask;  // ADD_FLOAT (I/O dtype) or BOOL (uint8)
  long long msb, msh, msq;
  const void* rel_h;
  const void* rel_w;
  int use_rel;
  int qh_n, qw_n, kh_n, kw_n;  // query / key patch grids (height, width)
  int* err;          // device error word (bounded waits report here)
  int k_vec16;       // k's rows are 16-byte aligned (vector loads allowed)
  // element strides of the batch, head and token axes (head_dim contiguous)
  long long sqb, sqh, sqt, skb, skh, skt, svb, svh, svt, sob, soh, sot;
};

// Element offsets of row t of (batch b, head h) in q / k / v / out.
__host__ __device__ __forceinline__ long long q_off(const Params& p, long long b, long long h, long long t) {
  return b * p.sqb + h * p.sqh + t * p.sqt;
}
__host__ __device__ __forceinline__ long long k_off(const Params& p, long long b, long long h, long long t) {
  return b * p.skb + h * p.skh + t * p.skt;
}
__host__ __device__ __forceinline__ long long v_off(const Params& p, long long b, long long h, long long t) {
  return b * p.svb + h * p.svh + t * p.svt;
}
__host__ __device__ __forceinline__ long long o_off(const Params& p, long long b, long long h, long long t) {
  return b * p.sob + h * p.soh + t * p.sot;
}
// Every stride of q, k, v and out is a multiple of n elements.
__host__ __device__ __forceinline__ bool strides_multiple_of(const Params& p, long long n) {
  const long long s[12] = {p.sqb, p.sqh, p.sqt, p.skb, p.skh, p.skt, p.svb, p.svh, p.svt, p.sob, p.soh, p.sot};
  for (int i = 0; i < 12; ++i)
    if (s[i] % n != 0) return false;
  return true;
}

enum ErrBits { ERR_WAIT_TIMEOUT = 1, ERR_INDEX = 2 };

// Device-side index checks.  A build compiled with SDPA_DEBUG tests each
// index a kernel derives (query / key rows, rel-pos table rows, mask and
// workspace slots, shared-memory slots of the scatter) against its extent
// before the access; an index outside it sets ERR_INDEX in the error word and
// the access is skipped (no trap, no fault).  Without SDPA_DEBUG every check
// is the constant true and compiles away.
#ifdef SDPA_DEBUG
__device__ __noinline__ inline void dcheck_fail(int* err) {
  if (err != nullptr) atomicOr(err, ERR_INDEX);
}
__device__ __forceinline__ bool dcheck(int* err, bool ok) {
  if (!ok) dcheck_fail(err);
  return ok;
}
// 0 <= i < n
__device__ __forceinline__ bool dcheck_idx(int* err, long long i, long long n) { return dcheck(err, i >= 0 && i < n); }
// row t of (batch b, query head h): q, out, lse
__device__ __forceinline__ bool dcheck_q(const Params& p, long long b, long long h, long long t) {
  return dcheck(p.err, b >= 0 && b < p.B && h >= 0 && h < p.Hq && t >= 0 && t < p.Tq);
}
// row t of (batch b, key/value head hk): k, v
__device__ __forceinline__ bool dcheck_kv(const Params& p, long long b, long long hk, long long t) {
  return dcheck(p.err, b >= 0 && b < p.B && hk >= 0 && hk < p.Hkv && t >= 0 && t < p.Tkv);
}
#else
__device__ __forceinline__ constexpr bool dcheck(int*, bool) { return true; }
__device__ __forceinline__ constexpr bool dcheck_idx(int*, long long, long long) { return true; }
__device__ __forceinline__ constexpr bool dcheck_q(const Params&, long long, long long, long long) { return true; }
__device__ __forceinline__ constexpr bool dcheck_kv(const Params&, long long, long long, long long) { return true; }
#endif

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Visible key range [lo, hi) of query row i under CAUSAL / SLIDING; the whole
// key axis otherwise.
__host__ __device__ __forceinline__ void key_range(const Params& p, long long i, long long& lo,
                                                   long long& hi) {
  lo = 0;
  hi = p.Tkv;
  if (p.mask_kind == SDPA_MASK_CAUSAL || p.mask_kind == SDPA_MASK_SLIDING) {
    long long top = i + p.offset + 1;  // exclusive upper bound
    if (top < hi) hi = top;
    if (p.mask_kind == SDPA_MASK_SLIDING) {
      long long bot = i + p.offset - p.window + 1;
      if (bot > lo) lo = bot;
    }
    if (hi < lo) hi = lo;
  }
}

// Launchers (one per kernel family); each returns a cudaError_t of the launch.
cudaError_t launch_exact(const Params& p, sdpa_dtype_t dtype, cudaStream_t stream);
int tc_check(const Params& p, sdpa_dtype_t dtype);  // SDPA_OK or why the tensor-core kernel cannot run
// Library-owned scratch of the current device: a counter area of at least
// `cnt_bytes` that is zero when the next kernel on `stream` starts (kernels
// taking tickets from it leave it zero again) and a data area of at least
// `data_bytes`.  Returns SDPA_OK or SDPA_ERR_CUDA.
int workspace_get(size_t cnt_bytes, size_t data_bytes, void** cnt, void** data, cudaStream_t stream);
int small_d_check(const Params& p, sdpa_dtype_t dtype);
cudaError_t launch_small_d(const Params& p, cudaStream_t stream);
int split_kv_check(const Params& p, sdpa_dtype_t dtype);
cudaError_t launch_split_kv(const Params& p, cudaStream_t stream);
// scratch the split-KV kernel needs for this problem (tickets that must be
// zero at launch, and partial results) and the launch on given scratch
void split_kv_workspace_bytes(const Params& p, size_t* cnt_bytes, size_t* data_bytes);
cudaError_t launch_split_kv_ws(const Params& p, int* cnt, void* data, cudaStream_t stream);
// split-KV on the fixed-size static scratch (no allocation); an sdpa_status
int split_kv_static(const Params& p, sdpa_dtype_t dtype, cudaStream_t stream);
// One bounded mbarrier wait that runs out (nothing arrives); sets *err.
int selftest_wait_timeout(unsigned long long limit_ns, int* err, cudaStream_t stream);
// One index check of i against [0, n) on the device, no memory access at i.
int selftest_index_check(long long i, long long n, int* err, cudaStream_t stream);
int num_sms();
cudaError_t launch_tc(const Params& p, cudaStream_t stream);
// persistent form of the tensor-core kernel (one CTA per SM over many short problems)
int tc_persist_check(const Params& p, sdpa_dtype_t dtype);
bool tc_persist_preferred(const Params& p);
cudaError_t launch_tc_persist(const Params& p, cudaStream_t stream);

// Division by a divisor d >= 1 fixed at launch, as a multiply-high, an add
// and a shift (Granlund and Montgomery, "Division by Invariant Integers using
// Multiplication", 1994, section 4, unsigned division by a run-time invariant
// divisor): with l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1 (which
// fits in 32 bits), n / d = (umulhi(m, n) + n) >> l for every 32-bit unsigned
// n, the sum taken in 64 bits.  The kernels decode their work unit with it:
// a generic 32-bit division is a long dependent chain at the head of every CTA.
struct FastDiv {
  uint32_t d, m, l;
};
inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d < 1 ? 1 : d;
  uint32_t l = 0;
  while ((1ull << l) < f.d) ++l;
  f.l = l;
  f.m = (uint32_t)((((1ull << 32) * ((1ull << l) - f.d)) / f.d) + 1);
  return f;
}
__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
  return (uint32_t)(((uint64_t)__umulhi(f.m, n) + n) >> f.l);
}

// Parts sdpa_merge combines at most.
constexpr int kMaxMergeParts = 16;
cudaError_t launch_merge(const void* const* outs, const float* const* lses, int n, void* out, float* lse,
                         sdpa_dtype_t dtype, long long rows, int d, cudaStream_t stream);

}  // namespace sdpa
