// Self-test of the device-side failure detection: the bounded mbarrier waits
// every kernel of the library uses (mbar_wait_for / mbar_wait_cluster_for in
// common.cuh) give up after their limit, raise DEVERR_TIMEOUT in the error
// word and return, so a stuck pipeline ends as an error status instead of a
// hung GPU.  This kernel makes such a wait run out on purpose, on barriers
// that nothing arrives on and with nothing else in flight: no copy, no
// tensor-memory allocation, no peer CTA, so returning early leaves nothing
// behind.  The host then reads the status as DSA_ERR_TIMEOUT.
#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

// One CTA of 32 threads: thread 0 waits on a local barrier of count 2 that
// receives one arrival (its phase never completes), then on the same barrier
// with the cluster-scope poll; each gives up after limit_ns and raises
// DEVERR_TIMEOUT in err[0].
__global__ void __launch_bounds__(32) bounded_wait_selftest_kernel(uint32_t* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 2);
    mbar_fence_init();
    mbar_arrive(&bar);                      // one of the two arrivals; the other never comes
    mbar_wait_for(&bar, 0, err, limit_ns);
    mbar_wait_cluster_for(&bar, 0, err, limit_ns);
  }
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" dsa_status dsa_selftest_bounded_wait(int limit_us, void* ws, size_t ws_bytes,
                                                void* stream) {
  if (!ws || ws_bytes < 256) return DSA_ERR_INVALID_ARG;
  if (limit_us < 1 || limit_us > 2000000) return DSA_ERR_INVALID_ARG;   // at most the library's 2 s
  bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint32_t*>(ws), static_cast<uint64_t>(limit_us) * 1000u);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}
