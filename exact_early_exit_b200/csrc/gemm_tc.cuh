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
nv_status tc_gemm_run(TcPlanCache* c, const void* X, int ldx, const void* W, int N, int K, const int* nrows,
                      int max_rows, float* Y, bool allow_split, int* split_grid, size_t* split_stride,
                      cudaStream_t st);

}  // namespace nv
