// Self-test of the failure path of the library's bounded device waits.  One
// small CTA waits on an mbarrier that nothing ever arrives at, with the same
// bounded wait the tensor-core kernels use (mbar_wait: a globaltimer limit),
// gives up, records KDA_ERR_DEVICE_TIMEOUT in the status word, runs the error
// exit's drain on the barrier (which runs out too) and returns.  Nothing faults
// or traps, so the context stays usable; the host reads the status word.
#include "kda_common.cuh"
#include "kda_tcgen05.cuh"

namespace kda {
namespace {
using namespace tc;

__global__ void __launch_bounds__(32) wait_timeout_kernel(uint64_t limit_ns, int *status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  const bool ok = mbar_wait(&bar, 0u, limit_ns);  // phase 0 never completes
  if (!ok && threadIdx.x == 0) {
    report(status, KDA_ERR_DEVICE_TIMEOUT);
    drain(&bar, limit_ns);
  }
  __syncwarp();
}

}  // namespace

cudaError_t launch_wait_timeout(unsigned limit_us, int *status, cudaStream_t s) {
  wait_timeout_kernel<<<1, 32, 0, s>>>((uint64_t)limit_us * 1000ull, status);
  return cudaGetLastError();
}

}  // namespace kda
