// tcgen05 GEMM for bf16 models (sm_100a): Y[r][n] = sum_k X[r][k] W[n][k].
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace nv {

struct TcPlanCache;
TcPlanCache* tc_plans_create();
void tc_plans_destroy(TcPlanCache* c);
nv_status tc_prepare();
int* tc_status_ptr(TcPlanCache* c);
size_t tc_workspace_elems(size_t N);
struct EpiArgs;
nv_status tc_gemm_run(TcPlanCache* c, const void* X, int ldx, const void* W, int N, int K, const int* nrows,
                      int max_rows, float* Y, bool allow_split, const EpiArgs* epi, int* tile_counters,
                      const void* prefetch, size_t prefetch_bytes, cudaStream_t st, int* grid_out = nullptr,
                      const int* skip_if_zero = nullptr);
// 2-D tensor map over rows of 64 bf16 (128 bytes) with 128-byte swizzle and
// boxes of box_rows rows (decode attention's view of the KV pool)
nv_status encode_rows128_map(const void* base, uint64_t rows, uint32_t box_rows, CUtensorMap* out);
// elements between split-K slices of an N-column output
size_t tc_split_stride(size_t N);
// Cached 2-D bf16 tensor map over [outer][inner] (row stride ld_elems), boxes
// of 64 x box_rows, 128-byte swizzle (the GEMM operand layout).
nv_status tc_map(TcPlanCache* c, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld_elems,
                 uint32_t box_rows, CUtensorMap* out);
// SMs of the current device (the persistent grids' size)
int tc_sm_count();
}  // namespace nv
