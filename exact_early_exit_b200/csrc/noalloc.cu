// nv_philox4x32_10_noalloc: the Philox test hook without any allocation.
//
// nv_philox4x32_10 stages its counters and results through a device buffer it
// cudaMalloc's and cudaFree's on every call.  Some callers cannot do that: a
// host framework whose caching allocator already holds the device's memory
// (a fresh cudaMalloc fails or fragments it), or a latency-critical loop that
// cannot afford the device-wide synchronisation cudaMalloc / cudaFree may
// imply.  This variant stages through a fixed array in device global memory,
// declared below, and runs the same kernel.
#include <mutex>

#include "kernels.cuh"

// Staging array: counters in the first half, results in the second.  Every
// GPU that loads the library holds it (1 MiB) until the process exits.
static __device__ __align__(256) unsigned char nv_philox_noalloc_scratch[2 * NV_PHILOX_NOALLOC_MAX * 16];

namespace {
// Device address of the array for each device.  In host code the array's name
// stands for a host-side shadow, not a device address, so it is looked up
// once per device with that device current.
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};
}  // namespace

extern "C" nv_status nv_philox4x32_10_noalloc(uint64_t seed, const uint32_t* ctr, int n, uint32_t* out,
                                              void* stream) {
  if (!ctr || !out) {
    nv::set_error("null argument");
    return NV_ERR_INVALID_ARG;
  }
  if (n < 1 || n > NV_PHILOX_NOALLOC_MAX) {
    nv::set_error("nv_philox4x32_10_noalloc: n must be in [1, NV_PHILOX_NOALLOC_MAX = " +
                  std::to_string(NV_PHILOX_NOALLOC_MAX) + "], got " + std::to_string(n));
    return NV_ERR_INVALID_ARG;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    nv::set_error(std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    return NV_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    nv::set_error("device index beyond the supported range");
    return NV_ERR_UNSUPPORTED;
  }
  unsigned char* base = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, nv_philox_noalloc_scratch);
      if (e != cudaSuccess || !p) {
        nv::set_error(std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
        return NV_ERR_CUDA;
      }
      g_addr[dev] = p;
    }
    base = (unsigned char*)g_addr[dev];
  }
  unsigned char* din = base;
  unsigned char* dout = base + (size_t)NV_PHILOX_NOALLOC_MAX * 16;
  cudaStream_t st = (cudaStream_t)stream;
  // nothing needs clearing: the n counters are copied in and the n results
  // are fully written before they are copied out
  e = cudaMemcpyAsync(din, ctr, (size_t)n * 16, cudaMemcpyDefault, st);
  if (e == cudaSuccess) {
    nv::launch_philox(seed, din, n, dout, st);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaMemcpyAsync(out, dout, (size_t)n * 16, cudaMemcpyDefault, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) {
    nv::set_error(std::string("nv_philox4x32_10_noalloc: ") + cudaGetErrorString(e));
    return NV_ERR_CUDA;
  }
  return NV_OK;
}
