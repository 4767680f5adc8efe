// selftest.cu — runs the kernels' bounded-wait path to its timeout on
// purpose, so that a test can check the failure report end to end.
//
// One thread initialises an mbarrier that nothing will ever arrive on and
// waits on it with the same bounded wait the pipelines use (mbar_wait), but
// with a caller-given limit: the wait gives up, DA_ERR_DEVICE_TIMEOUT lands
// in the caller's status word, and the kernel returns normally, leaving the
// context usable.  Nothing faults, traps or waits without a bound.
#include <cuda_runtime.h>

#include <cstdint>

#include "diffattn.h"
#include "ptx.cuh"

namespace da {
namespace {

__global__ void wait_timeout_kernel(int* dev_status, unsigned long long limit_ns,
                                    unsigned long long* waited_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // expects one arrival that never comes
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    bool failed = false;
    const uint64_t t0 = global_ns();
    const bool done = mbar_wait(&bar, 0, dev_status, &failed, limit_ns);
    if (waited_ns) *waited_ns = global_ns() - t0;
    if (done) report(dev_status, DA_ERR_INVALID_ARG);  // cannot happen: nothing arrives
  }
}

}  // namespace
}  // namespace da

extern "C" int diffattn_selftest_wait_timeout(unsigned int timeout_us, int* dev_status,
                                              unsigned long long* waited_ns, void* stream) {
  if (!dev_status || timeout_us == 0 || timeout_us > 1000000u) return DA_ERR_INVALID_ARG;
  da::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      dev_status, 1000ull * timeout_us, waited_ns);
  return cudaGetLastError() == cudaSuccess ? DA_OK : DA_ERR_CUDA;
}
