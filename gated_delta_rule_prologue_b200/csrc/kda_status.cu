// The per-device status word of libkda: one int in a file-scope __device__
// variable, so that no entry point ever allocates it.  It starts at zero when
// this file's device module loads; kernels record faults they detect there
// (KDA_ERR_DEVICE_*), and kda_get_device_status reads and clears it.
//
// This file holds nothing else, so loading its module (at the first library
// call on a device under lazy module loading) reserves only the word itself.
#include <cuda_runtime.h>

#include <mutex>

#include "kda_common.cuh"

namespace kda {
namespace {

__device__ int g_status_word;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int *g_addr[kMaxDevices] = {nullptr};

}  // namespace

// Device address of the status word of the current device, looked up once per
// device with that device current (a host-side reference to g_status_word is
// only a stand-in, never a device address).
cudaError_t status_word_address(int **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_status_word);
    if (e != cudaSuccess) return e;
    g_addr[dev] = static_cast<int *>(p);
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace kda
