// GEMM dispatch (see gemm.cuh).
#include <cstdlib>
#include <cstring>

#include "gemm.cuh"
#include "gemm_tc.cuh"
#include "kernels.cuh"

namespace nv {

struct GemmPlanCache {
  TcPlanCache* tc = nullptr;
};

GemmPlanCache* gemm_plans_create() {
  GemmPlanCache* c = new GemmPlanCache();
  c->tc = tc_plans_create();
  return c;
}
void gemm_plans_destroy(GemmPlanCache* c) {
  if (!c) return;
  tc_plans_destroy(c->tc);
  delete c;
}

TcPlanCache* gemm_tc_plans(GemmPlanCache* c) { return c ? c->tc : nullptr; }

int* gemm_status_ptr(GemmPlanCache* c) { return c ? tc_status_ptr(c->tc) : nullptr; }

int gemm_default_kind() {
  const char* e = std::getenv("NVIUM_GEMM");
  if (e && std::strcmp(e, "simt") == 0) return GEMM_SIMT;
  return GEMM_TC;
}

nv_status gemm_prepare(int kind, bool bf16) {
  if (kind == GEMM_TC && bf16) return tc_prepare();
  return NV_OK;
}

size_t gemm_workspace_elems(int kind, size_t rows, size_t N) {
  size_t e = rows * N;
  if (kind == GEMM_TC) {
    const size_t t = tc_workspace_elems(N);
    if (t > e) e = t;
  }
  return e;
}

int gemm_launch_count(int kind, bool bf16, bool allow_split, const EpiArgs* epi) {
  const int epilogue = (epi && epi->mode != EPI_STORE) ? 1 : 0;
  if (kind == GEMM_TC && bf16) return allow_split ? 1 + epilogue : 1;
  return 1 + epilogue;
}

nv_status gemm_run(GemmPlanCache* plans, int kind, bool bf16, const void* X, int ldx, const void* W, int N, int K,
                   const int* nrows, int max_rows, float* Y, bool allow_split, const EpiArgs* epi, int* tile_counters,
                   int epi_grid, const void* prefetch, size_t prefetch_bytes, cudaStream_t st,
                   int* split_grid_out) {
  if (kind == GEMM_TC && bf16) {
    if (!allow_split)  // one slice: the epilogue runs inside the GEMM kernel
      return tc_gemm_run(plans->tc, X, ldx, W, N, K, nrows, max_rows, Y, false, epi, tile_counters, prefetch,
                         prefetch_bytes, st);
    // split-K slices: the GEMM writes fp32 partials, the epilogue kernel sums them
    int grid = 0;
    NV_TRY(tc_gemm_run(plans->tc, X, ldx, W, N, K, nrows, max_rows, Y, true, nullptr, nullptr, prefetch,
                       prefetch_bytes, st, &grid));
    if (split_grid_out) *split_grid_out = grid;
    if (epi && epi->mode != EPI_STORE) {
      EpiArgs e = *epi;
      e.Y = Y;
      e.split_grid = grid;
      e.split_K = K;
      e.split_stride = tc_split_stride(N);
      e.N = N;
      launch_epilogue(true, e, epi_grid, st);
    }
    return NV_OK;
  }
  launch_gemm_simt(bf16, X, ldx, W, N, K, nrows, max_rows, Y, st);
  if (split_grid_out) *split_grid_out = 0;
  if (epi && epi->mode != EPI_STORE) {
    EpiArgs e = *epi;
    e.Y = Y;
    e.split_grid = 0;
    e.split_stride = 0;
    e.N = N;
    launch_epilogue(bf16, e, epi_grid, st);
  }
  return NV_OK;
}

}  // namespace nv
