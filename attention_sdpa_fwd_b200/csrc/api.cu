// C ABI of libsdpa: argument validation, kernel-family selection, launch.
// Declarations and the meaning of every argument: include/sdpa.h.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace sdpa {

// Bit set by kernels whose bounded waits expire; read and cleared by
// sdpa_last_device_error().
__device__ int g_error_word;

namespace {

constexpr int kMaxDevices = 64;

int* error_word_ptr() {
  static int* ptrs[kMaxDevices] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int*>(p);
  }
  return ptrs[dev];
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Scratch for split key ranges, one per device, grown on demand and never
// shrunk: a counter area that is zero between launches (every kernel that
// takes tickets from it puts them back to zero) and a separate data area for
// partial results.  `dirty` is set when a kernel may have left counters
// non-zero (a device-side wait gave up); the next user clears them first.
struct Workspace {
  void* cnt = nullptr;
  size_t cnt_cap = 0;
  void* data = nullptr;
  size_t data_cap = 0;
  bool dirty = false;
};
Workspace g_ws[kMaxDevices];
std::mutex g_ws_mu;

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (a == nullptr || b == nullptr || na == 0 || nb == 0) return false;
  uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

struct Problem {
  Params p;
  sdpa_dtype_t dtype;
  size_t esz;
  bool empty_out;  // nothing to write
};

// Validates everything that can be checked on the host and fills the kernel
// parameters.  Pointers are only checked for NULL, alignment to the element
// size and overlap of `out` with the inputs.
int build_problem(const void* q, const void* k, const void* v, void* out, sdpa_dtype_t dtype, int B,
                  int Hq, int Hkv, int Tq, int Tkv, int d, float scale, int mask_kind,
                  const void* mask_ptr, const void* rel_pos_h, const void* rel_pos_w,
                  const int* q_hw, const int* k_hw, float* lse, Problem* pr,
                  const sdpa_strides_t* const* strides = nullptr) {
  memset(pr, 0, sizeof(*pr));
  if (dtype != SDPA_F32 && dtype != SDPA_BF16) return SDPA_ERR_INVALID_ARG;
  if (B < 0 || Hq < 1 || Hkv < 1 || Tq < 0 || Tkv < 0) return SDPA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return SDPA_ERR_INVALID_ARG;
  if (!(d == 16 || d == 64 || d == 128)) return SDPA_ERR_UNSUPPORTED;
  if (!isfinite(scale)) return SDPA_ERR_INVALID_ARG;
  if (mask_kind < SDPA_MASK_NONE || mask_kind > SDPA_MASK_BOOL) return SDPA_ERR_INVALID_ARG;
  const size_t esz = dtype == SDPA_F32 ? 4 : 2;
  Params& p = pr->p;
  p.q = q; p.k = k; p.v = v; p.out = out; p.lse = lse;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Tq = Tq; p.Tkv = Tkv; p.d = d;
  p.group = Hq / Hkv;
  p.scale = scale;
  p.mask_kind = mask_kind;
  const long long rows = (long long)B * Hq * Tq;
  pr->empty_out = rows == 0;
  pr->dtype = dtype;
  pr->esz = esz;
  // strides: dense bhsd unless given
  {
    const long long dq[3] = {(long long)Hq * Tq * d, (long long)Tq * d, d};
    const long long dk[3] = {(long long)Hkv * Tkv * d, (long long)Tkv * d, d};
    long long* dst[4][3] = {{&p.sqb, &p.sqh, &p.sqt}, {&p.skb, &p.skh, &p.skt},
                            {&p.svb, &p.svh, &p.svt}, {&p.sob, &p.soh, &p.sot}};
    for (int a = 0; a < 4; ++a) {
      const long long* def = (a == 1 || a == 2) ? dk : dq;
      const sdpa_strides_t* st = strides ? strides[a] : nullptr;
      if (st == nullptr) {
        for (int x = 0; x < 3; ++x) *dst[a][x] = def[x];
      } else {
        const long long given[3] = {st->b, st->h, st->t};
        for (int x = 0; x < 3; ++x) {
          if (given[x] < 1 || given[x] > (1LL << 40)) return SDPA_ERR_INVALID_ARG;
          *dst[a][x] = given[x];
        }
      }
    }
  }

  const sdpa_mask_t* m = static_cast<const sdpa_mask_t*>(mask_ptr);
  if (mask_kind == SDPA_MASK_CAUSAL) {
    p.offset = m ? m->offset : 0;
  } else if (mask_kind == SDPA_MASK_SLIDING) {
    if (m == nullptr || m->window < 1) return SDPA_ERR_INVALID_ARG;
    p.offset = m->offset;
    p.window = m->window;
  } else if (mask_kind == SDPA_MASK_ADD_FLOAT || mask_kind == SDPA_MASK_BOOL) {
    if (m == nullptr) return SDPA_ERR_INVALID_ARG;
    if (m->stride_b < 0 || m->stride_h < 0 || m->stride_q < 0) return SDPA_ERR_INVALID_ARG;
    if (!pr->empty_out && Tkv > 0 && m->data == nullptr) return SDPA_ERR_INVALID_ARG;
    const size_t mesz = mask_kind == SDPA_MASK_BOOL ? 1 : esz;
    if (m->data && !aligned(m->data, mesz)) return SDPA_ERR_MISALIGNED;
    p.mask = m->data;
    p.msb = m->stride_b; p.msh = m->stride_h; p.msq = m->stride_q;
  }
  if (p.offset > (1LL << 40) || p.offset < -(1LL << 40) || p.window > (1LL << 40))
    return SDPA_ERR_INVALID_ARG;

  if ((rel_pos_h == nullptr) != (rel_pos_w == nullptr)) return SDPA_ERR_INVALID_ARG;
  if (rel_pos_h != nullptr) {
    if (q_hw == nullptr || k_hw == nullptr) return SDPA_ERR_INVALID_ARG;
    if (q_hw[0] < 1 || q_hw[1] < 1 || k_hw[0] < 1 || k_hw[1] < 1) return SDPA_ERR_INVALID_ARG;
    if ((long long)q_hw[0] * q_hw[1] != Tq || (long long)k_hw[0] * k_hw[1] != Tkv)
      return SDPA_ERR_INVALID_ARG;
    if (!aligned(rel_pos_h, esz) || !aligned(rel_pos_w, esz)) return SDPA_ERR_MISALIGNED;
    p.use_rel = 1;
    p.rel_h = rel_pos_h; p.rel_w = rel_pos_w;
    p.qh_n = q_hw[0]; p.qw_n = q_hw[1]; p.kh_n = k_hw[0]; p.kw_n = k_hw[1];
  }

  if (!pr->empty_out) {
    if (q == nullptr || out == nullptr) return SDPA_ERR_INVALID_ARG;
    if (Tkv > 0 && (k == nullptr || v == nullptr)) return SDPA_ERR_INVALID_ARG;
    if (!aligned(q, esz) || !aligned(out, esz) || (k && !aligned(k, esz)) || (v && !aligned(v, esz)))
      return SDPA_ERR_MISALIGNED;
    if (lse && !aligned(lse, 4)) return SDPA_ERR_MISALIGNED;
    // address span of each tensor: last element + 1, in bytes
    auto span = [&](long long sb, long long sh, long long st, int H, int T) -> size_t {
      if (B == 0 || T == 0) return 0;
      return (size_t)((B - 1) * sb + (long long)(H - 1) * sh + (long long)(T - 1) * st + d) * esz;
    };
    const size_t nq = span(p.sqb, p.sqh, p.sqt, Hq, Tq), no = span(p.sob, p.soh, p.sot, Hq, Tq);
    const size_t nk = span(p.skb, p.skh, p.skt, Hkv, Tkv), nv = span(p.svb, p.svh, p.svt, Hkv, Tkv);
    if (overlaps(out, no, q, nq) || overlaps(out, no, k, nk) || overlaps(out, no, v, nv))
      return SDPA_ERR_INVALID_ARG;
    // lse is written while other CTAs still read q, k, v and the mask: no overlap with any of them
    size_t nm = 0;
    if (p.mask != nullptr && Tkv > 0) {
      const long long last = (long long)(B - 1) * p.msb + (long long)(Hq - 1) * p.msh +
                             (long long)(Tq - 1) * p.msq + Tkv;
      nm = (size_t)last * (mask_kind == SDPA_MASK_BOOL ? 1 : esz);
    }
    const size_t nl = (size_t)rows * 4;
    if (lse && (overlaps(lse, nl, out, no) || overlaps(lse, nl, q, nq) || overlaps(lse, nl, k, nk) ||
                overlaps(lse, nl, v, nv) || overlaps(lse, nl, p.mask, nm)))
      return SDPA_ERR_INVALID_ARG;
  }
  p.k_vec16 = (k != nullptr && aligned(k, 16) && (p.skb * (long long)esz) % 16 == 0 &&
               (p.skh * (long long)esz) % 16 == 0 && (p.skt * (long long)esz) % 16 == 0)
                  ? 1 : 0;
  return SDPA_OK;
}

int choose_path(const Problem& pr) {
  const Params& p = pr.p;
  if (p.Tkv == 0) return SDPA_PATH_EXACT;
  if (tc_check(p, pr.dtype) == SDPA_OK) {
    // many short problems: one persistent CTA per SM walks them
    if (tc_persist_check(p, pr.dtype) == SDPA_OK && tc_persist_preferred(p)) return SDPA_PATH_TC_PERSISTENT;
    return SDPA_PATH_TCGEN05;
  }
  if (small_d_check(p, pr.dtype) == SDPA_OK) {
    // a long key axis against at most a sixteenth as many query rows: split
    // the keys over the SMs.  The small-d kernel walks the keys in rounds of
    // 128 per CTA, so with few query rows (few CTAs) those rounds are the whole
    // time.  Measured at 4 x 8 heads, split-KV against small-d: 64 x 1024 rows
    // x keys 13.9 against 34.2 us, 128 x 2048 51.6 against about 69, 128 x 1024
    // 50.8 against 34.4, 256 x 2048 98.8 against 66.7, 512 x 4096 268 against 131.
    if (p.Tkv >= 1024 && (long long)p.Tq * 16 <= p.Tkv) return SDPA_PATH_SPLIT_KV;
    return SDPA_PATH_SMALL_D;
  }
  return SDPA_PATH_EXACT;
}

int run(const Problem& pr, int path, cudaStream_t stream) {
  if (pr.empty_out) return SDPA_OK;
  Params p = pr.p;
  if (path == SDPA_PATH_AUTO) path = choose_path(pr);
  // a forced family that cannot take the problem says so before any device work
  int rc = SDPA_OK;
  switch (path) {
    case SDPA_PATH_EXACT: break;
    case SDPA_PATH_TCGEN05: rc = tc_check(p, pr.dtype); break;
    case SDPA_PATH_TC_PERSISTENT: rc = tc_persist_check(p, pr.dtype); break;
    case SDPA_PATH_SMALL_D: rc = small_d_check(p, pr.dtype); break;
    case SDPA_PATH_SPLIT_KV: rc = split_kv_check(p, pr.dtype); break;
    default: return SDPA_ERR_INVALID_ARG;
  }
  if (rc != SDPA_OK) return rc;
  p.err = error_word_ptr();
  if (p.err == nullptr) return SDPA_ERR_CUDA;
  cudaError_t e = cudaErrorInvalidValue;
  switch (path) {
    case SDPA_PATH_EXACT: e = launch_exact(p, pr.dtype, stream); break;
    case SDPA_PATH_TCGEN05: e = launch_tc(p, stream); break;
    case SDPA_PATH_TC_PERSISTENT: e = launch_tc_persist(p, stream); break;
    case SDPA_PATH_SMALL_D: e = launch_small_d(p, stream); break;
    case SDPA_PATH_SPLIT_KV: e = launch_split_kv(p, stream); break;
  }
  return e == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

}  // namespace

int workspace_get(size_t cnt_bytes, size_t data_bytes, void** cnt, void** data, cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SDPA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_ws_mu);
  Workspace& w = g_ws[dev];
  auto round_mb = [](size_t x) { return (x + (1u << 20) - 1) & ~size_t((1u << 20) - 1); };
  if (w.cnt_cap < cnt_bytes || w.data_cap < data_bytes) {
    // earlier launches may still use the old buffers
    if ((w.cnt || w.data) && cudaDeviceSynchronize() != cudaSuccess) return SDPA_ERR_CUDA;
  }
  if (w.cnt_cap < cnt_bytes) {
    if (w.cnt) cudaFree(w.cnt);
    w.cnt = nullptr;
    w.cnt_cap = 0;
    const size_t cap = round_mb(cnt_bytes);
    if (cudaMalloc(&w.cnt, cap) != cudaSuccess) return SDPA_ERR_CUDA;
    if (cudaMemset(w.cnt, 0, cap) != cudaSuccess) return SDPA_ERR_CUDA;
    w.cnt_cap = cap;
  }
  if (w.data_cap < data_bytes) {
    if (w.data) cudaFree(w.data);
    w.data = nullptr;
    w.data_cap = 0;
    const size_t cap = round_mb(data_bytes);
    if (cudaMalloc(&w.data, cap) != cudaSuccess) return SDPA_ERR_CUDA;
    w.data_cap = cap;
  }
  if (w.dirty) {
    if (cudaMemsetAsync(w.cnt, 0, w.cnt_cap, stream) != cudaSuccess) return SDPA_ERR_CUDA;
    w.dirty = false;
  }
  *cnt = w.cnt;
  *data = w.data;
  return SDPA_OK;
}

int num_sms() {
  static int cached[kMaxDevices] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

void mark_workspace_dirty() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return;
  std::lock_guard<std::mutex> lock(g_ws_mu);
  g_ws[dev].dirty = true;
}

}  // namespace sdpa

using namespace sdpa;

extern "C" int sdpa_fwd_ex(const void* q, const void* k, const void* v, void* out, sdpa_dtype_t dtype,
                           int B, int Hq, int Hkv, int Tq, int Tkv, int d, float scale, int mask_kind,
                           const void* mask_ptr, const void* rel_pos_h, const void* rel_pos_w,
                           const int* q_hw, const int* k_hw, float* lse, int path, cudaStream_t stream) {
  if (path < SDPA_PATH_AUTO || path > SDPA_PATH_TC_PERSISTENT) return SDPA_ERR_INVALID_ARG;
  Problem pr;
  int rc = build_problem(q, k, v, out, dtype, B, Hq, Hkv, Tq, Tkv, d, scale, mask_kind, mask_ptr,
                         rel_pos_h, rel_pos_w, q_hw, k_hw, lse, &pr);
  if (rc != SDPA_OK) return rc;
  return run(pr, path, stream);
}

extern "C" int sdpa_fwd_strided(const void* q, const sdpa_strides_t* q_strides, const void* k,
                                const sdpa_strides_t* k_strides, const void* v, const sdpa_strides_t* v_strides,
                                void* out, const sdpa_strides_t* out_strides, sdpa_dtype_t dtype, int B, int Hq,
                                int Hkv, int Tq, int Tkv, int d, float scale, int mask_kind, const void* mask_ptr,
                                const void* rel_pos_h, const void* rel_pos_w, const int* q_hw, const int* k_hw,
                                float* lse, int path, cudaStream_t stream) {
  if (path < SDPA_PATH_AUTO || path > SDPA_PATH_TC_PERSISTENT) return SDPA_ERR_INVALID_ARG;
  const sdpa_strides_t* st[4] = {q_strides, k_strides, v_strides, out_strides};
  Problem pr;
  int rc = build_problem(q, k, v, out, dtype, B, Hq, Hkv, Tq, Tkv, d, scale, mask_kind, mask_ptr,
                         rel_pos_h, rel_pos_w, q_hw, k_hw, lse, &pr, st);
  if (rc != SDPA_OK) return rc;
  return run(pr, path, stream);
}

extern "C" int sdpa_merge(const void* const* outs, const float* const* lses, int nparts, void* out, float* lse,
                          sdpa_dtype_t dtype, int B, int Hq, int Tq, int d, cudaStream_t stream) {
  if (dtype != SDPA_F32 && dtype != SDPA_BF16) return SDPA_ERR_INVALID_ARG;
  if (nparts < 1 || nparts > kMaxMergeParts || outs == nullptr || lses == nullptr) return SDPA_ERR_INVALID_ARG;
  if (B < 0 || Hq < 1 || Tq < 0) return SDPA_ERR_INVALID_ARG;
  if (!(d == 16 || d == 64 || d == 128)) return SDPA_ERR_UNSUPPORTED;
  const long long rows = (long long)B * Hq * Tq;
  if (rows == 0) return SDPA_OK;
  if (out == nullptr) return SDPA_ERR_INVALID_ARG;
  const size_t esz = dtype == SDPA_F32 ? 4 : 2;
  const size_t no = (size_t)rows * d * esz, nl = (size_t)rows * 4;
  if (!aligned(out, 16) || (lse && !aligned(lse, 4))) return SDPA_ERR_MISALIGNED;
  for (int i = 0; i < nparts; ++i) {
    if (outs[i] == nullptr || lses[i] == nullptr) return SDPA_ERR_INVALID_ARG;
    if (!aligned(outs[i], 16) || !aligned(lses[i], 4)) return SDPA_ERR_MISALIGNED;
    // out may be part 0 exactly (in place); no other overlap
    if (!(i == 0 && outs[i] == out) && overlaps(out, no, outs[i], no)) return SDPA_ERR_INVALID_ARG;
    if (overlaps(out, no, lses[i], nl)) return SDPA_ERR_INVALID_ARG;
    if (lse && !(i == 0 && lses[i] == lse) && overlaps(lse, nl, lses[i], nl)) return SDPA_ERR_INVALID_ARG;
    if (lse && overlaps(lse, nl, outs[i], no)) return SDPA_ERR_INVALID_ARG;
  }
  if (lse && overlaps(lse, nl, out, no)) return SDPA_ERR_INVALID_ARG;
  const cudaError_t e = launch_merge(outs, lses, nparts, out, lse, dtype, rows, d, stream);
  return e == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

extern "C" int sdpa_fwd(const void* q, const void* k, const void* v, void* out, sdpa_dtype_t dtype,
                        int B, int Hq, int Hkv, int Tq, int Tkv, int d, float scale, int mask_kind,
                        const void* mask_ptr, const void* rel_pos_h, const void* rel_pos_w,
                        const int* q_hw, const int* k_hw, cudaStream_t stream) {
  return sdpa_fwd_ex(q, k, v, out, dtype, B, Hq, Hkv, Tq, Tkv, d, scale, mask_kind, mask_ptr,
                     rel_pos_h, rel_pos_w, q_hw, k_hw, nullptr, SDPA_PATH_AUTO, stream);
}

extern "C" int sdpa_select_path(const void* q, const void* k, const void* v, void* out,
                                sdpa_dtype_t dtype, int B, int Hq, int Hkv, int Tq, int Tkv, int d,
                                int mask_kind, const void* mask_ptr, const void* rel_pos_h,
                                const void* rel_pos_w, const int* q_hw, const int* k_hw) {
  Problem pr;
  int rc = build_problem(q, k, v, out, dtype, B, Hq, Hkv, Tq, Tkv, d, 1.0f, mask_kind, mask_ptr,
                         rel_pos_h, rel_pos_w, q_hw, k_hw, nullptr, &pr);
  if (rc != SDPA_OK) return rc;
  return choose_path(pr);
}


namespace sdpa {
namespace {

// Slabs the host entry point pipelines a problem into: three measured best
// for SAM global attention (545 us per call against 568 with six and 608
// with one, on one B200 machine): fewer slabs overlap less of the uploads with
// the kernels, more slabs pay a fixed cost per copy and run kernels too
// small to fill the GPU.
constexpr int kHostChunks = 3;

// Device staging buffer of sdpa_fwd_host, one per device, grown on demand,
// with the two copy streams and the events that order the pipeline.
struct Staging {
  void* buf = nullptr;
  size_t cap = 0;
  bool pipe_ready = false;
  cudaStream_t up = nullptr, down = nullptr;
  cudaEvent_t start = nullptr, landed[kHostChunks] = {}, computed[kHostChunks] = {};
};

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace
}  // namespace sdpa

extern "C" int sdpa_fwd_host(const void* q, const void* k, const void* v, void* out, sdpa_dtype_t dtype,
                             int B, int Hq, int Hkv, int Tq, int Tkv, int d, float scale, int mask_kind,
                             const void* mask_ptr, const void* rel_pos_h, const void* rel_pos_w,
                             const int* q_hw, const int* k_hw, int path, cudaStream_t stream) {
  if (path < SDPA_PATH_AUTO || path > SDPA_PATH_TC_PERSISTENT) return SDPA_ERR_INVALID_ARG;
  Problem pr;
  int rc = build_problem(q, k, v, out, dtype, B, Hq, Hkv, Tq, Tkv, d, scale, mask_kind, mask_ptr,
                         rel_pos_h, rel_pos_w, q_hw, k_hw, nullptr, &pr);
  if (rc != SDPA_OK) return rc;
  if (pr.empty_out) return SDPA_OK;
  static Staging staging[kMaxDevices];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SDPA_ERR_CUDA;

  const size_t esz = pr.esz;
  const size_t nq = (size_t)B * Hq * Tq * d * esz;
  const size_t nk = (size_t)B * Hkv * Tkv * d * esz;
  size_t nrh = 0, nrw = 0, nmask = 0;
  if (pr.p.use_rel) {
    nrh = (size_t)(pr.p.qh_n + pr.p.kh_n - 1) * d * esz;
    nrw = (size_t)(pr.p.qw_n + pr.p.kw_n - 1) * d * esz;
  }
  const bool tensor_mask = mask_kind == SDPA_MASK_ADD_FLOAT || mask_kind == SDPA_MASK_BOOL;
  if (tensor_mask && Tkv > 0) {
    const size_t mesz = mask_kind == SDPA_MASK_BOOL ? 1 : esz;
    const long long last = (long long)(B - 1) * pr.p.msb + (long long)(Hq - 1) * pr.p.msh +
                           (long long)(Tq - 1) * pr.p.msq + Tkv;
    nmask = (size_t)last * mesz;
  }
  const size_t oq = 0, ok = round_up(oq + nq, 256), ov = round_up(ok + nk, 256),
               oo = round_up(ov + nk, 256), orh = round_up(oo + nq, 256),
               orw = round_up(orh + nrh, 256), om = round_up(orw + nrw, 256),
               total = round_up(om + nmask, 256);

  std::lock_guard<std::mutex> lock(mu);
  Staging& st = staging[dev];
  if (st.cap < total) {
    if (st.buf) cudaFree(st.buf);
    st.buf = nullptr;
    st.cap = 0;
    if (cudaMalloc(&st.buf, total) != cudaSuccess) return SDPA_ERR_CUDA;
    st.cap = total;
  }
  if (!st.pipe_ready) {
    if (cudaStreamCreateWithFlags(&st.up, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&st.down, cudaStreamNonBlocking) != cudaSuccess)
      return SDPA_ERR_CUDA;
    for (int i = 0; i < kHostChunks; ++i)
      if (cudaEventCreateWithFlags(&st.landed[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&st.computed[i], cudaEventDisableTiming) != cudaSuccess)
        return SDPA_ERR_CUDA;
    if (cudaEventCreateWithFlags(&st.start, cudaEventDisableTiming) != cudaSuccess) return SDPA_ERR_CUDA;
    st.pipe_ready = true;
  }
  char* base = static_cast<char*>(st.buf);
  // Everything this call queues on the copy streams comes after the work
  // already queued on the caller's stream.
  if (cudaEventRecord(st.start, stream) != cudaSuccess || cudaStreamWaitEvent(st.up, st.start, 0) != cudaSuccess)
    return SDPA_ERR_CUDA;
  auto h2d = [&](size_t off, const void* src, size_t n) {
    return n == 0 || cudaMemcpyAsync(base + off, src, n, cudaMemcpyHostToDevice, st.up) == cudaSuccess;
  };
  if (!h2d(orh, rel_pos_h, nrh) || !h2d(orw, rel_pos_w, nrw)) return SDPA_ERR_CUDA;
  sdpa_mask_t dmask;
  if (tensor_mask) {
    dmask = *static_cast<const sdpa_mask_t*>(mask_ptr);
    if (!h2d(om, dmask.data, nmask)) return SDPA_ERR_CUDA;
  }

  // Pipeline over slabs of (batch, head): slab i's inputs go up on one copy
  // stream while slab i-1 computes on the caller's stream and slab i-2's
  // output comes down on the other, so the copies overlap the kernels (and
  // each other, on separate copy engines).  A slab is whole batches when
  // there are at least kHostChunks of them, else a run of query heads of one
  // batch that covers whole GQA groups.
  const int group = Hq / Hkv;
  struct Slab { int b0, nb, h0, nh; };
  Slab slabs[kHostChunks];
  int ns = 0;
  if (B >= kHostChunks || Hq / group <= 1) {
    const int per = (B + kHostChunks - 1) / kHostChunks;
    for (int b0 = 0; b0 < B && ns < kHostChunks; b0 += per) slabs[ns++] = {b0, std::min(per, B - b0), 0, Hq};
  } else {
    const int groups = Hkv;                                   // kv heads per batch
    const int per_b = std::max(1, kHostChunks / B);            // slabs per batch
    const int gpc = (groups + per_b - 1) / per_b;              // kv groups per slab
    for (int b = 0; b < B; ++b)
      for (int g0 = 0; g0 < groups && ns < kHostChunks; g0 += gpc)
        slabs[ns++] = {b, 1, g0 * group, std::min(gpc, groups - g0) * group};
  }
  const size_t qrow = (size_t)Tq * d * esz, krow = (size_t)Tkv * d * esz;  // bytes per (b, h)
  const size_t mesz = mask_kind == SDPA_MASK_BOOL ? 1 : esz;
  for (int i = 0; i < ns; ++i) {
    const Slab& c = slabs[i];
    const size_t zq0 = (size_t)c.b0 * Hq + c.h0, nzq = (size_t)c.nb * c.nh;        // (b, h) rows of q / out
    const size_t zk0 = (size_t)c.b0 * Hkv + c.h0 / group, nzk = nzq / group;       // rows of k / v
    const char* qh = static_cast<const char*>(q) + zq0 * qrow;
    if (!h2d(oq + zq0 * qrow, qh, nzq * qrow)) return SDPA_ERR_CUDA;
    if (Tkv > 0) {
      if (!h2d(ok + zk0 * krow, static_cast<const char*>(k) + zk0 * krow, nzk * krow) ||
          !h2d(ov + zk0 * krow, static_cast<const char*>(v) + zk0 * krow, nzk * krow))
        return SDPA_ERR_CUDA;
    }
    if (cudaEventRecord(st.landed[i], st.up) != cudaSuccess || cudaStreamWaitEvent(stream, st.landed[i], 0) != cudaSuccess)
      return SDPA_ERR_CUDA;
    sdpa_mask_t cm;
    const void* mptr = mask_ptr;
    if (tensor_mask) {
      cm = dmask;
      cm.data = nmask ? base + om + ((long long)c.b0 * dmask.stride_b + (long long)c.h0 * dmask.stride_h) * mesz
                      : nullptr;
      mptr = &cm;
    }
    Problem dpr;
    rc = build_problem(base + oq + zq0 * qrow, Tkv ? base + ok + zk0 * krow : nullptr,
                       Tkv ? base + ov + zk0 * krow : nullptr, base + oo + zq0 * qrow, dtype, c.nb, c.nh,
                       c.nh / group, Tq, Tkv, d, scale, mask_kind, mptr, nrh ? base + orh : nullptr,
                       nrw ? base + orw : nullptr, q_hw, k_hw, nullptr, &dpr);
    if (rc != SDPA_OK) return rc;
    rc = run(dpr, path, stream);
    if (rc != SDPA_OK) return rc;
    if (cudaEventRecord(st.computed[i], stream) != cudaSuccess ||
        cudaStreamWaitEvent(st.down, st.computed[i], 0) != cudaSuccess ||
        cudaMemcpyAsync(static_cast<char*>(out) + zq0 * qrow, base + oo + zq0 * qrow, nzq * qrow,
                        cudaMemcpyDeviceToHost, st.down) != cudaSuccess)
      return SDPA_ERR_CUDA;
  }
  if (cudaStreamSynchronize(st.down) != cudaSuccess || cudaStreamSynchronize(stream) != cudaSuccess)
    return SDPA_ERR_CUDA;
  return SDPA_OK;
}

extern "C" int sdpa_fwd_split_kv_static(const void* q, const void* k, const void* v, void* out,
                                        sdpa_dtype_t dtype, int B, int Hq, int Hkv, int Tq, int Tkv, int d,
                                        float scale, int mask_kind, const void* mask_ptr, float* lse,
                                        cudaStream_t stream) {
  Problem pr;
  int rc = build_problem(q, k, v, out, dtype, B, Hq, Hkv, Tq, Tkv, d, scale, mask_kind, mask_ptr, nullptr,
                         nullptr, nullptr, nullptr, lse, &pr);
  if (rc != SDPA_OK) return rc;
  if (pr.empty_out) return SDPA_OK;
  Params p = pr.p;
  p.err = error_word_ptr();
  if (p.err == nullptr) return SDPA_ERR_CUDA;
  return split_kv_static(p, pr.dtype, stream);
}

extern "C" int sdpa_selftest_wait_timeout(unsigned long long limit_ns, cudaStream_t stream) {
  // the wait must end well inside any watchdog: at most the kernels' own 2 s
  if (limit_ns == 0 || limit_ns > 2000000000ull) return SDPA_ERR_INVALID_ARG;
  int* err = error_word_ptr();
  if (err == nullptr) return SDPA_ERR_CUDA;
  return selftest_wait_timeout(limit_ns, err, stream);
}

extern "C" int sdpa_selftest_index_check(long long index, long long extent, cudaStream_t stream) {
  if (extent < 0) return SDPA_ERR_INVALID_ARG;
  int* err = error_word_ptr();
  if (err == nullptr) return SDPA_ERR_CUDA;
  return selftest_index_check(index, extent, err, stream);
}

extern "C" int sdpa_debug_checks(void) {
#ifdef SDPA_DEBUG
  return 1;
#else
  return 0;
#endif
}

extern "C" int sdpa_last_device_error(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return SDPA_ERR_CUDA;
  int* w = error_word_ptr();
  if (w == nullptr) return SDPA_ERR_CUDA;
  int host = 0;
  if (cudaMemcpy(&host, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SDPA_ERR_CUDA;
  if (host != 0) {
    const int zero = 0;
    if (cudaMemcpy(w, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return SDPA_ERR_CUDA;
    mark_workspace_dirty();  // an abandoned split may have left its counters behind
    return (host & ERR_INDEX) ? SDPA_ERR_DEVICE_INDEX : SDPA_ERR_TIMEOUT;
  }
  return SDPA_OK;
}

extern "C" const char* sdpa_strerror(int status) {
  switch (status) {
    case SDPA_OK: return "ok";
    case SDPA_ERR_INVALID_ARG: return "invalid argument";
    case SDPA_ERR_UNSUPPORTED: return "unsupported by this build";
    case SDPA_ERR_MISALIGNED: return "misaligned pointer or stride";
    case SDPA_ERR_CUDA: return "CUDA error";
    case SDPA_ERR_TIMEOUT: return "device-side wait timed out";
    case SDPA_ERR_CAPACITY: return "request exceeds a fixed-size buffer";
    case SDPA_ERR_DEVICE_INDEX: return "device-side index check failed (debug build)";
  }
  return "unknown status";
}

extern "C" int sdpa_version(void) { return 100; }
