// sdpa_selftest_wait_timeout: exercises the failure-detection path of the
// tensor-core kernels without any fault.  Every mbarrier wait of those kernels
// is bounded by a %globaltimer limit; when it runs out the kernel sets the
// device error word and unwinds, and sdpa_last_device_error() reports
// SDPA_ERR_TIMEOUT.  This kernel makes one such wait run out on purpose: a
// single thread waits, with the caller's short limit, on an mbarrier that
// nothing ever arrives on, then returns.  The wait always ends (the limit is
// checked on the host to be at most 2 s), no memory is touched except the
// error word, and the CUDA context stays usable.
//
// sdpa_selftest_index_check: runs one device-side index check (the checks a
// build with SDPA_DEBUG compiles into the kernels) on an index and an extent
// the caller gives.  Nothing is read or written at the index: the kernel only
// evaluates the check, which in a debug build sets the error word when the
// index is outside [0, n), and in a release build is the constant true.
#include "common.cuh"
#include "sm100.cuh"

namespace sdpa {
namespace {

using namespace sm100;

__global__ void wait_timeout_kernel(int* err, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    // phase 0 never completes: no thread arrives and no copy is in flight
    (void)mbar_wait_for(&bar, 0, nullptr, err, limit_ns);
  }
}

__global__ void index_check_kernel(int* err, long long i, long long n) {
  if (threadIdx.x == 0) (void)dcheck_idx(err, i, n);
}

}  // namespace

int selftest_index_check(long long i, long long n, int* err, cudaStream_t stream) {
  index_check_kernel<<<1, 32, 0, stream>>>(err, i, n);
  return cudaGetLastError() == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

int selftest_wait_timeout(unsigned long long limit_ns, int* err, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(err, limit_ns);
  return cudaGetLastError() == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

}  // namespace sdpa
