// Internal definitions shared by libnvium's kernels and host code.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstddef>
#include <string>
#include <utility>

#include "../../include/nvium.h"

namespace nv {

// ---------------------------------------------------------------------------
// error plumbing
// ---------------------------------------------------------------------------
void set_error(const std::string& msg);

#define NV_CUDA_TRY(expr)                                                        \
  do {                                                                           \
    cudaError_t _e = (expr);                                                     \
    if (_e != cudaSuccess) {                                                     \
      ::nv::set_error(std::string(#expr) + ": " + cudaGetErrorString(_e));       \
      return NV_ERR_CUDA;                                                        \
    }                                                                            \
  } while (0)

#define NV_TRY(expr)                 \
  do {                               \
    nv_status _s = (expr);           \
    if (_s != NV_OK) return _s;      \
  } while (0)

// Device status word values (first error wins).
enum DevErr : int {
  DEV_OK = 0,
  DEV_ERR_ROWS = 1,     // a work list exceeded its capacity
  DEV_ERR_KV = 2,       // a KV position beyond the page table
  DEV_ERR_TIMEOUT = 3,  // a bounded wait ran out
};

__device__ __forceinline__ void dev_fail(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------------------
// element access: float or bf16 storage, fp32 arithmetic
// ---------------------------------------------------------------------------
template <typename T> __device__ __forceinline__ float ld(const T* p);
template <> __device__ __forceinline__ float ld<float>(const float* p) { return *p; }
template <> __device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename T> __device__ __forceinline__ T cvt(float x);
template <> __device__ __forceinline__ float cvt<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 cvt<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);  // round to nearest even
}
// value after the storage type's rounding (identity for float)
template <typename T> __device__ __forceinline__ float rnd(float x);
template <> __device__ __forceinline__ float rnd<float>(float x) { return x; }
template <> __device__ __forceinline__ float rnd<__nv_bfloat16>(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}

// ---------------------------------------------------------------------------
// per-element arithmetic shared by every kernel that performs the step, so
// that two kernels doing the same step round identically
// ---------------------------------------------------------------------------
// (each written with explicit rounding intrinsics, so the compiler cannot
// contract or reorder it differently in different kernels)
// rotate-half RoPE of the pair (y0, y1) by (cos, sin)
__device__ __forceinline__ float2 rope_pair(float y0, float y1, float2 cs) {
  return make_float2(__fmaf_rn(y0, cs.x, -__fmul_rn(y1, cs.y)), __fmaf_rn(y1, cs.x, __fmul_rn(y0, cs.y)));
}
// SwiGLU: silu(g) * u = g / (1 + 2^(-g log2 e)) * u, with the hardware's
// base-2 exponential and reciprocal (PTX ex2.approx / rcp.approx, relative
// errors near 2^-22; the product is rounded to bf16 afterwards)
__device__ __forceinline__ float swiglu(float g, float u) {
  float e, r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(__fmul_rn(g, -1.4426950408889634f)));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(__fadd_rn(1.0f, e)));
  return __fmul_rn(__fmul_rn(g, r), u);
}
// sum of squares of four values (one float4 of an RMSNorm row)
__device__ __forceinline__ float sumsq4(float4 x) {
  return __fmaf_rn(x.w, x.w, __fmaf_rn(x.z, x.z, __fmaf_rn(x.y, x.y, __fmul_rn(x.x, x.x))));
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
// Easy as 1, 2, 3", SC'11, section 3.2): ten rounds; each multiplies counter
// words 0 and 2 by fixed odd constants, swaps in the high halves XORed with
// words 1/3 and the round key, and the key is bumped by the Weyl constants
// between rounds.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}
// 32 random bits -> U in (0,1): ((x >> 9) + 1/2) * 2^-23, exact in fp32.
__device__ __forceinline__ float uniform01(uint32_t x) {
  return ((float)(x >> 9) + 0.5f) * 1.1920928955078125e-07f;
}
__device__ __forceinline__ uint32_t lane_of(uint4 v, int lane) {
  return lane == 0 ? v.x : lane == 1 ? v.y : lane == 2 ? v.z : v.w;
}
constexpr uint32_t STREAM_EXIT = 0;
constexpr uint32_t STREAM_GUMBEL = 1;

// ---------------------------------------------------------------------------
// device-side views
// ---------------------------------------------------------------------------
struct LayerDev {
  const void* attn_norm;
  const void* w_qkv;  // [3*H*hd, d]: q rows, then k rows, then v rows
  const void* w_o;    // [d, H*hd]
  const void* mlp_norm;
  const void* w_gu;   // [2F, d], gate/up interleaved in blocks of gu_block rows
  const void* w_d;    // [d, F]
};
struct ExitDev {
  const void* norm;
  const void* head;      // [V, d]
  const void* router_w;  // [d] (unused for the last exit)
  float router_b;
  const void* router_w1;    // router MLP [r, d] (model dtype), or null
  const float* router_b1;   // [r]
  const float* router_w2;   // [r]
  const void* adapter_w1;   // exit adapter [a, d] (model dtype), or null
  const void* adapter_w2;   // [d, a]
};

// Rows processed together at one layer.  Rows of a sequence are contiguous and
// in ascending position order; seq_start[b]..seq_start[b+1] are b's rows.
struct RowSet {
  const int* nrows;      // device scalar: rows in this set
  const int* row_b;      // [max_rows]
  const int* row_pos;    // [max_rows]
  const int* row_hrow;   // [max_rows] row of h holding this row's residual
  const int* seq_start;  // [B+1]
  float* h;              // residual stream, [*, d] fp32
  int max_rows;
  int B;
};

// Paged KV cache.  A page holds page_size positions of one sequence for one
// layer: [2 (K,V)][H][page_size][hd].  Layer m's pages start at
// base + m * layer_stride elements.
struct KVView {
  void* base;
  size_t layer_stride;
  const int* page_table;  // [B][pages_per_seq] physical page ids
  int pages_per_seq;
  int page_size;
  int H, hd;
  __host__ __device__ __forceinline__ size_t offset(int layer, int b, int pos, int head, int kv) const {
    const int page = page_table[(size_t)b * pages_per_seq + pos / page_size];
    return (size_t)layer * layer_stride +
           (((size_t)page * 2 + kv) * H + head) * (size_t)page_size * hd + (size_t)(pos % page_size) * hd;
  }
};

// ---------------------------------------------------------------------------
// Programmatic dependent launch: every kernel of the path is launched with
// programmatic stream serialisation, so its launch and prologue overlap the
// previous kernel; each kernel waits (griddepcontrol.wait) before it reads
// anything a predecessor wrote, on every path, and then lets its own
// dependents launch.  NVIUM_PDL=0 launches them plainly.
// ---------------------------------------------------------------------------
bool pdl_enabled();
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                            Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Which part of a fused weight a GEMM output column belongs to.
// EPI_LSE: scoring head; per row and 128-token tile the max and the sum of
// exp(logit - max), and the target token's logit (the logits never reach
// global memory)
enum EpiMode : int { EPI_QKV = 0, EPI_RESID = 1, EPI_SWIGLU = 2, EPI_STORE = 3, EPI_HEAD = 4, EPI_LSE = 5 };

}  // namespace nv
