// sdpa_fwd_split_kv_static: the split-KV forward on library scratch that lives
// in a fixed-size device array instead of memory the library allocates.
//
// Who needs it: callers that must not allocate device memory during a call --
// code that runs under a memory pool it does not control, or whose startup
// already reserved every byte it may use.  The regular split-KV path asks
// the CUDA allocator for its scratch on first use (and again when a larger
// problem needs more); this entry point never does.
//
// The scratch is one file-scope __device__ array of kStaticScratchBytes.
// Every device that loads the library holds it until the process exits.
// Every call on a device shares it, and each call leaves its contents behind,
// so two calls whose kernels overlap on the GPU (different streams, or no
// ordering between them) race on it; calls on one stream are fine.
#include <mutex>

#include "common.cuh"

namespace sdpa {
namespace {

// 4 MiB: 64 KiB of tickets (one int per (batch, head), at most 16384 of them)
// followed by the partial results of the split.
constexpr size_t kStaticScratchBytes = 4u << 20;
constexpr size_t kStaticTicketBytes = 64u << 10;

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDev = 64;

// The array's device address, looked up once per device (under a lock, so
// that two host threads making their first call on one device at once do not
// race on the cache).  Host code must not use the symbol itself: on the host
// it names a host-side stand-in, and a kernel given that address would fault
// (or quietly read the wrong memory).
int static_scratch(void** ptr) {
  static void* addr[kMaxDev] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return SDPA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return SDPA_ERR_CUDA;
    addr[dev] = p;
  }
  *ptr = addr[dev];
  return SDPA_OK;
}

}  // namespace

int split_kv_static(const Params& p, sdpa_dtype_t dtype, cudaStream_t stream) {
  const int rc = split_kv_check(p, dtype);
  if (rc != SDPA_OK) return rc;
  size_t cnt_bytes = 0, data_bytes = 0;
  split_kv_workspace_bytes(p, &cnt_bytes, &data_bytes);
  if (cnt_bytes > kStaticTicketBytes || data_bytes > kStaticScratchBytes - kStaticTicketBytes)
    return SDPA_ERR_CAPACITY;
  void* base = nullptr;
  const int sc = static_scratch(&base);
  if (sc != SDPA_OK) return sc;
  char* b = static_cast<char*>(base);
  // the tickets must start at zero; the previous call on this array may have
  // been abandoned part-way, so clear them on the stream (no allocation)
  if (cudaMemsetAsync(b, 0, cnt_bytes, stream) != cudaSuccess) return SDPA_ERR_CUDA;
  const cudaError_t e = launch_split_kv_ws(p, reinterpret_cast<int*>(b), b + kStaticTicketBytes, stream);
  return e == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

}  // namespace sdpa
