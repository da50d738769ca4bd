// Self-tests of the library's failure detection.
//
// Bounded waits: one
// small CTA waits on an mbarrier that nothing ever arrives at, with the same
// bounded wait the tensor-core kernels use (mbar_wait: a globaltimer limit),
// gives up, records KDA_ERR_DEVICE_TIMEOUT in the status word, runs the error
// exit's drain on the barrier (which runs out too) and returns.  Nothing faults
// or traps, so the context stays usable; the host reads the status word.
//
// Debug-build index checks: one thread writes a four-slot probe array at a
// caller-chosen index through the same check the kernels use (in_range).  In a
// debug build an index outside [0, 4) records KDA_ERR_DEVICE_BOUNDS and the
// write is skipped.  Release builds compile the check out, so the host entry
// refuses to launch there.
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

__device__ int g_bounds_probe[4];

__global__ void __launch_bounds__(32) bounds_probe_kernel(int index, int *status) {
  if (threadIdx.x == 0 && in_range(status, index, 4)) g_bounds_probe[index] = 1;
}

}  // namespace

cudaError_t launch_bounds_probe(int index, int *status, cudaStream_t s) {
  if (!kDebugChecks) return cudaErrorNotSupported;
  bounds_probe_kernel<<<1, 32, 0, s>>>(index, status);
  return cudaGetLastError();
}

cudaError_t launch_wait_timeout(unsigned limit_us, int *status, cudaStream_t s) {
  wait_timeout_kernel<<<1, 32, 0, s>>>((uint64_t)limit_us * 1000ull, status);
  return cudaGetLastError();
}

}  // namespace kda
