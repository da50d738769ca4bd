// Scratch of kda_chunk_fwd_static: a file-scope __device__ array, one per
// device, that no call allocates or frees.  It lives in a file of its own so
// that its device module (and with it the array's memory) is loaded only when
// kda_chunk_fwd_static first looks it up under lazy module loading, not by the
// other entry points; under eager loading every context holds it.  It is held
// until the context is destroyed.
#include <cuda_runtime.h>

#include <mutex>

#include "kda_common.cuh"

namespace kda {
namespace {

__device__ __align__(256) uint8_t g_static_scratch[KDA_CHUNK_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_addr[kMaxDevices] = {nullptr};

}  // namespace

// Device address of the array on the current device, looked up once per device
// with that device current.  A host-side reference to g_static_scratch names a
// host stand-in, not device memory: a kernel given it would fault or, where the
// GPU can reach host memory, silently use the wrong memory.
cudaError_t static_scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace kda
