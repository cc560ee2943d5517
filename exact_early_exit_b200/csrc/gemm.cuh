// GEMM dispatch: Y = X W^T for the packed layer weights.
//
// Two engines: a SIMT fp32-accumulate kernel (the fp32 model; tf32 tensor
// cores would break its 1e-4 bound) and a tcgen05 kernel for bf16 models
// (operands staged in shared memory by TMA, fp32 accumulators in TMEM).
// Both write fp32 Y[nsplit][rows][N]; the epilogue kernels sum the split
// partials in a fixed order.
#pragma once

#include "common.cuh"

namespace nv {

enum GemmKind : int { GEMM_SIMT = 0, GEMM_TC = 1 };

struct GemmPlanCache;  // tensor maps keyed by (pointer, shape)
struct TcPlanCache;
TcPlanCache* gemm_tc_plans(GemmPlanCache* c);
GemmPlanCache* gemm_plans_create();
void gemm_plans_destroy(GemmPlanCache* c);

// Device status word of the GEMM engine (0 = fine), or null.
int* gemm_status_ptr(GemmPlanCache* c);
// Engine used for bf16 models: tcgen05 unless NVIUM_GEMM=simt.
int gemm_default_kind();
// One-time kernel attributes (shared memory opt-in); call outside capture.
nv_status gemm_prepare(int kind, bool bf16);
// fp32 elements of workspace for `rows` x N outputs, split partials included.
size_t gemm_workspace_elems(int kind, size_t rows, size_t N);

// Split-K policy of the tcgen05 engine, shared by the GEMM and the epilogues
// so that both derive the same count from the device-side row count R: when
// all rows fit one 256-row tile and the 128-feature tiles alone cannot fill
// the `grid` persistent CTAs, the K range is split (at most max_split ways).
constexpr int TC_MAX_SPLIT = 16;
__host__ __device__ __forceinline__ int tc_split_count(int R, int N, int K, int grid, int max_split) {
  if (grid <= 0 || R <= 0) return 1;
  const int ntn = N / 128, nrt = (R + 255) / 256, kblocks = K / 64;
  const int base = ntn * nrt;
  if (nrt != 1 || base >= grid) return 1;
  int s = grid / base;
  if (s > kblocks) s = kblocks;
  if (s > max_split) s = max_split;
  return s < 1 ? 1 : s;
}

struct EpiArgs;
// Kernels one gemm_run call with these arguments launches (1 or 2).
int gemm_launch_count(int kind, bool bf16, bool allow_split, const EpiArgs* epi);
// Launch Y = X W^T followed by the layer epilogue `epi` (mode EPI_QKV,
// EPI_RESID or EPI_SWIGLU; null or EPI_STORE: write fp32 Y).  X: [rows][ldx]
// (rows <= max_rows, count in *nrows on the device), W: [N][K] row-major.
// The tcgen05 engine applies the epilogue inside the GEMM kernel when the K
// range is not split; with allow_split it may split K (tc_split_count), store
// fp32 slices in Y and run the epilogue kernel after it, which sums the slices
// in a fixed order.  The SIMT engine always runs the epilogue kernel after it.
// `prefetch` / `prefetch_bytes`: the next GEMM's weights, pulled into L2 by
// the tcgen05 engine while it runs (a hint; may be null).
nv_status gemm_run(GemmPlanCache* plans, int kind, bool bf16, const void* X, int ldx, const void* W, int N, int K,
                   const int* nrows, int max_rows, float* Y, bool allow_split, const EpiArgs* epi, int* tile_counters,
                   int epi_grid, const void* prefetch, size_t prefetch_bytes, cudaStream_t st,
                   int* split_grid_out = nullptr);

}  // namespace nv
