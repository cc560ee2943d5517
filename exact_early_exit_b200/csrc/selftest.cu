// nv_selftest_bounded_wait: exercises the bounded-wait rule every kernel of
// the library follows (an mbarrier or flag wait gives up after a time limit,
// records DEV_ERR_TIMEOUT and returns, so the context stays usable) on a
// barrier that nothing ever completes.  The decode path has no wait that can
// be made to run out on purpose without breaking its inputs, so this entry
// point is how that rule is tested on a GPU.
#include "kernels.cuh"

namespace nv {
namespace {

__global__ void k_selftest_wait(unsigned long long limit_ns, int* result) {
  pdl_wait();
  pdl_launch();
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(&bar);
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(a) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  unsigned long long t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  int code = 0;
  for (uint32_t i = 0;; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(a)
        : "memory");
    if (ok) break;  // never: no thread arrives
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    if (t - t0 > limit_ns) {
      code = DEV_ERR_TIMEOUT;
      break;
    }
  }
  *result = code;
}

}  // namespace
}  // namespace nv

extern "C" nv_status nv_selftest_bounded_wait(int limit_us, int* expired_out, void* stream) {
  if (!expired_out) {
    nv::set_error("null argument");
    return NV_ERR_INVALID_ARG;
  }
  if (limit_us < 1 || limit_us > 1000000) {
    nv::set_error("limit_us must be in [1, 1000000]");
    return NV_ERR_INVALID_ARG;
  }
  cudaStream_t st = (cudaStream_t)stream;
  int* d = nullptr;
  cudaError_t e = cudaMallocAsync((void**)&d, sizeof(int), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(d, 0xff, sizeof(int), st);
  if (e == cudaSuccess) e = nv::launch_k(nv::k_selftest_wait, 1, 32, 0, st, (unsigned long long)limit_us * 1000ull, d);
  int h = -1;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&h, d, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (d) cudaFreeAsync(d, st);
  if (e != cudaSuccess) {
    nv::set_error(std::string("nv_selftest_bounded_wait: ") + cudaGetErrorString(e));
    cudaGetLastError();
    return NV_ERR_CUDA;
  }
  *expired_out = h == nv::DEV_ERR_TIMEOUT ? 1 : 0;
  return NV_OK;
}
