// tcgen05 GEMM (sm_100a): Y[r][n] = sum_k X[r][k] W[n][k], bf16 in, fp32 out.
//
// The packed-row GEMM of every backbone layer: the new tokens' rows and the
// deferred rows of one layer form X (section 2 "Inferenz: Piggybacking" of
// the N-vium summary: deferred rows ride in the same batched pass), W is the
// layer's packed weight.  Orientation: the weight is the MMA's A operand (128
// output features per tile, TMEM lanes) and the rows are its N dimension (up
// to 256 per tile, TMEM columns), so a decode step with a handful of rows
// still issues full 128-row MMAs and streams each weight tile once.
//
// Persistent, warp-specialised CTAs (one per SM):
//   warp 4, one lane: TMA producer, 4-stage ring of (W tile 128x64, X tile
//                     <=256x64), 128-byte swizzle, mbarrier complete_tx;
//   warp 5, one lane: issues tcgen05.mma (kind::f16, M=128, N=32..256,
//                     K=16) into one of two TMEM accumulators, commits to the
//                     stage's "empty" barrier and to "accumulator full";
//   warps 0-3:        epilogue, tcgen05.ld 32 columns at a time and coalesced
//                     fp32 stores (each warp owns 32 features = TMEM lanes).
// When all rows fit one tile and the feature tiles cannot fill the GPU, the K
// range is split (tc_split_count); the partial slices are summed in a fixed
// order by the epilogue kernels.  Every mbarrier wait is bounded: on expiry
// the CTA flags DEV_ERR_TIMEOUT, stops issuing work, frees its TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <map>
#include <mutex>
#include <tuple>

#include "gemm.cuh"
#include "gemm_tc.cuh"

namespace nv {
namespace {

constexpr int BM = 128;      // features per tile (MMA M, TMEM lanes)
constexpr int BK = 64;       // K per stage: one 128-byte swizzle row of bf16
constexpr int BNMAX = 256;   // rows per tile (MMA N, TMEM columns)
constexpr int BOXN = 32;     // rows per X TMA box
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BNMAX * BK * 2;
constexpr int BOX_BYTES = BOXN * BK * 2;
constexpr int SMEM_TILES = STAGES * (A_BYTES + B_BYTES);
constexpr int SMEM_BYTES = SMEM_TILES + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t TMEM_COLS = 512;  // two 256-column fp32 accumulators
constexpr int THREADS = 192;
constexpr unsigned long long WAIT_NS = 2000000000ull;  // 2 s bound on any single wait

struct TcArgs {
  const int* nrows;
  float* Y;
  int N, K;
  int max_split;
  size_t split_stride;
  int* status;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait; false when `limit_ns` ran out (the CTA then aborts) or
// another role aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag,
                                          unsigned long long limit_ns = WAIT_NS) {
  if (mbar_try_wait(b, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(b, parity)) return true;
    if ((i & 63u) == 0u) {
      if (*abort_flag) return false;
      if (global_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        return false;
      }
    }
  }
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), descriptor version 1 (sm_100).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major.
__device__ __forceinline__ uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}
__device__ __forceinline__ void umma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

struct Item {
  int n0, r0, rows, nbox, kb0, kb1, split;
};
__device__ __forceinline__ Item decode_item(int it, int ntn, int splits, int R, int kblocks) {
  Item t;
  t.split = it % splits;
  const int tile = it / splits;
  t.n0 = (tile % ntn) * BM;
  t.r0 = (tile / ntn) * BNMAX;
  t.rows = min(BNMAX, R - t.r0);
  t.nbox = (t.rows + BOXN - 1) / BOXN;
  t.kb0 = (int)((long long)t.split * kblocks / splits);
  t.kb1 = (int)((long long)(t.split + 1) * kblocks / splits);
  return t;
}

__global__ void __launch_bounds__(THREADS, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tw, const __grid_constant__ CUtensorMap tx, TcArgs a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  const int R = *a.nrows;
  if (R <= 0) return;
  const int ntn = a.N / BM, nrt = (R + BNMAX - 1) / BNMAX, kblocks = a.K / BK;
  const int splits = tc_split_count(R, a.N, a.K, gridDim.x, a.max_split);
  const int items = ntn * nrt * splits;
  if ((int)blockIdx.x >= items) return;

  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  unsigned char* sA = smem;
  unsigned char* sB = smem + STAGES * A_BYTES;
  uint64_t* full = (uint64_t*)(smem + SMEM_TILES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(tfull + s, 1);
      mbar_init(tempty + s, 128);
    }
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;

  if (warp == 4) {
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tw)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tx)) : "memory");
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int issued[STAGES];  // parity of the last load issued into each stage, -1 if none
#pragma unroll
      for (int s = 0; s < STAGES; ++s) issued[s] = -1;
      for (int it = blockIdx.x; it < items && ok; it += gridDim.x) {
        const Item t = decode_item(it, ntn, splits, R, kblocks);
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          if (!mbar_wait(empty + stage, phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          issued[stage] = (int)phase;
          mbar_expect_tx(full + stage, (uint32_t)(A_BYTES + t.nbox * BOX_BYTES));
          tma_load_2d(sA + stage * A_BYTES, &tw, full + stage, kb * BK, t.n0);
          for (int j = 0; j < t.nbox; ++j)
            tma_load_2d(sB + stage * B_BYTES + j * BOX_BYTES, &tx, full + stage, kb * BK, t.r0 + j * BOXN);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {
        // let the copies already issued land before the CTA leaves (bounded)
        volatile int never = 0;
        for (int s = 0; s < STAGES; ++s)
          if (issued[s] >= 0) mbar_wait(full + s, (uint32_t)issued[s], &never, WAIT_NS / 4);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, aphase = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < items && ok; it += gridDim.x) {
        const Item t = decode_item(it, ntn, splits, R, kblocks);
        const uint32_t idesc = idesc_bf16(t.nbox * BOXN);
        if (!mbar_wait(tempty + acc, aphase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * BNMAX);
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          if (!mbar_wait(full + stage, phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_desc(smem_u32(sA + stage * A_BYTES));
          const uint64_t bd = sw128_desc(smem_u32(sB + stage * B_BYTES));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma(d, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc, (kb > t.kb0 || kk > 0) ? 1u : 0u);
          umma_commit(empty + stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(tfull + acc);
        acc ^= 1;
        if (acc == 0) aphase ^= 1u;
      }
    }
  } else {
    // epilogue warps 0..3: TMEM lanes 32*warp .. 32*warp+31
    int acc = 0;
    uint32_t aphase = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x) {
      const Item t = decode_item(it, ntn, splits, R, kblocks);
      if (!mbar_wait(tfull + acc, aphase, abort_flag)) break;
      __syncwarp();
      tc_fence_after();
      const int n = t.n0 + warp * 32 + lane;
      float* Ys = a.Y + (size_t)t.split * a.split_stride;
      const uint32_t tbase = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(acc * BNMAX);
      for (int c0 = 0; c0 < t.nbox * BOXN; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tbase + (uint32_t)c0, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int r = t.r0 + c0 + j;
          if (r < R) Ys[(size_t)r * a.N + n] = __uint_as_float(v[j]);
        }
      }
      tc_fence_before();
      mbar_arrive(tempty + acc);
      acc ^= 1;
      if (acc == 0) aphase ^= 1u;
    }
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
  if (threadIdx.x == 0 && s_abort) dev_fail(a.status, DEV_ERR_TIMEOUT);
}

// ---------------------------------------------------------------------------
// host side: tensor maps (cached per buffer and shape), launch
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
  });
  return fn;
}

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  }
  return n;
}

}  // namespace

struct TcPlanCache {
  std::mutex mu;
  std::map<std::tuple<uintptr_t, uint64_t, uint64_t, uint64_t, uint32_t>, CUtensorMap> maps;
  int* status = nullptr;
};

TcPlanCache* tc_plans_create() {
  TcPlanCache* c = new TcPlanCache();
  if (cudaMalloc((void**)&c->status, sizeof(int)) == cudaSuccess) cudaMemset(c->status, 0, sizeof(int));
  else c->status = nullptr;
  return c;
}
void tc_plans_destroy(TcPlanCache* c) {
  if (!c) return;
  if (c->status) cudaFree(c->status);
  delete c;
}

int* tc_status_ptr(TcPlanCache* c) { return c ? c->status : nullptr; }

nv_status tc_prepare() {
  cudaError_t e = cudaFuncSetAttribute(k_gemm_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) {
    set_error(std::string("tcgen05 GEMM shared memory: ") + cudaGetErrorString(e));
    return NV_ERR_UNSUPPORTED;
  }
  if (!get_encode()) {
    set_error("cuTensorMapEncodeTiled is unavailable");
    return NV_ERR_UNSUPPORTED;
  }
  return NV_OK;
}

size_t tc_workspace_elems(size_t N) { return (size_t)TC_MAX_SPLIT * BNMAX * N; }

static nv_status make_map(TcPlanCache* c, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld_elems,
                          uint32_t box_rows, CUtensorMap* out) {
  const auto key = std::make_tuple((uintptr_t)ptr, inner, outer, ld_elems, box_rows);
  std::lock_guard<std::mutex> g(c->mu);
  auto it = c->maps.find(key);
  if (it != c->maps.end()) {
    *out = it->second;
    return NV_OK;
  }
  auto enc = get_encode();
  if (!enc) {
    set_error("cuTensorMapEncodeTiled is unavailable");
    return NV_ERR_UNSUPPORTED;
  }
  if (((uintptr_t)ptr & 15) || (ld_elems * 2) % 16) {
    set_error("tcgen05 GEMM operand not 16-byte aligned");
    return NV_ERR_INVALID_ARG;
  }
  CUtensorMap m;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld_elems * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed with code " + std::to_string((int)r));
    return NV_ERR_CUDA;
  }
  c->maps[key] = m;
  *out = m;
  return NV_OK;
}

nv_status tc_gemm_run(TcPlanCache* c, const void* X, int ldx, const void* W, int N, int K, const int* nrows,
                      int max_rows, float* Y, bool allow_split, int* split_grid, size_t* split_stride,
                      cudaStream_t st) {
  if (N % BM || K % BK || K > ldx) {
    set_error("tcgen05 GEMM needs N % 128 == 0 and K % 64 == 0 (N=" + std::to_string(N) + ", K=" +
              std::to_string(K) + ")");
    return NV_ERR_UNSUPPORTED;
  }
  CUtensorMap tw, tx;
  NV_TRY(make_map(c, W, (uint64_t)K, (uint64_t)N, (uint64_t)K, BM, &tw));
  NV_TRY(make_map(c, X, (uint64_t)K, (uint64_t)max_rows, (uint64_t)ldx, BOXN, &tx));
  // persistent grid: never more CTAs than there can be work items
  const int ntn = N / BM;
  const int nrt_max = (max_rows + BNMAX - 1) / BNMAX;
  long long most = (long long)ntn * nrt_max * (allow_split ? TC_MAX_SPLIT : 1);
  int grid = sm_count();
  if (most < grid) grid = (int)most;
  TcArgs a;
  a.nrows = nrows;
  a.Y = Y;
  a.N = N;
  a.K = K;
  a.max_split = allow_split ? TC_MAX_SPLIT : 1;
  a.split_stride = (size_t)BNMAX * N;
  a.status = c->status;
  k_gemm_tc<<<grid, THREADS, SMEM_BYTES, st>>>(tw, tx, a);
  *split_grid = allow_split ? grid : 0;
  *split_stride = a.split_stride;
  return NV_OK;
}

}  // namespace nv
