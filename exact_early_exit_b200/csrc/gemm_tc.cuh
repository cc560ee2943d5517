// tcgen05 GEMM for bf16 models (sm_100a): Y[r][n] = sum_k X[r][k] W[n][k].
#pragma once

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
// elements between split-K slices of an N-column output
size_t tc_split_stride(size_t N);
}  // namespace nv
