// Persistent decode-layer kernel (sm_100a, bf16 models).
//
// One launch runs everything of a backbone layer that follows its attention,
// for the packed rows of a decode step or a flush (the new tokens still
// active at this depth and the deferred rows of their sequences: section 2
// "Inferenz: Piggybacking" of the N-vium summary, arXiv 2605.13190; LLaMA-2
// backbone, section 4):
//
//   O      h += o W_o^T               split-K slices of fp32 partial sums
//   N1     h += sum of the slices; act = RMSNorm(h) * g_mlp
//   GU     u = silu(act W_g^T) * (act W_u^T)   (SwiGLU in the epilogue)
//   D      slices of u W_d^T
//   N2     h += sum of the slices, then either act = RMSNorm(h) * g (the next
//          layer's attention norm, when that layer runs the same rows) or
//          nothing more (the last layer before an exit)
//   QKV    slices of act W_qkv^T for the next layer (or, in a launch that
//          runs only this part, for this layer after the planner's norm)
//   E      q, k, v = sum of the slices; RoPE on q and k; q -> q buffer, k and
//          v -> the paged KV cache
//
// One CTA per SM for the whole launch.  Warp roles:
//   warp 4 (one lane)   streams weight tiles (128 features x 64 K, TMA,
//                       128-byte swizzle) through a ring of stages from the
//                       first instruction on; weights never depend on the
//                       rows, so the ring keeps filling across every
//                       dependency wait below;
//   warp 6 (one lane)   loads the activation tile of each stage (TMA) once the
//                       producing part is complete;
//   warp 5 (one lane)   issues tcgen05.mma (M = 128 features, N = rows, K =
//                       16) into two TMEM accumulators;
//   warps 0-3           epilogues (slices, SwiGLU), the row norms and E.
// Dependencies between CTAs are counters and per-tile flags in global
// memory (release increments, acquire polls), never a whole-grid barrier:
// N1 waits for every O item, GU's activation loads for every N1 row, each D
// item only for the gate/up tiles that produce its K range, N2 for every D
// item, QKV's loads for every N2 row, E for every QKV item.  Every wait is
// bounded (2 s): on expiry the CTA records DEV_ERR_TIMEOUT, raises a global
// abort flag that ends the other CTAs' waits, lets its own copies land and
// frees its TMEM.  The last CTA to finish zeroes the counters.
//
// The split counts, slice layouts, reduction orders and per-element
// arithmetic are those of the per-kernel path (k_gemm_tc + k_resid_norm +
// k_epilogue), so the two paths give bit-identical results.
#include <cuda.h>

#include "gemm.cuh"
#include "kernels.cuh"
#include "layer_tc.cuh"
#include "tc_prims.cuh"

namespace nv {
namespace {
using namespace tc;

constexpr int LT_THREADS = 224;
constexpr int W_WARP = 4, MMA_WARP = 5, X_WARP = 6;
// Separate rings for weight tiles (16 KB each) and activation tiles (the
// row tile's boxes): the activations come from L2 right after their producer
// finishes, so three stages hide them, and the rest of the shared memory goes
// to the weight ring, which keeps streaming while a part waits for its input.
constexpr int SMEM_TILES = 4 * (A_BYTES + BNMAX * BK * 2);  // 192 KB for both rings
constexpr int XST = 3;      // activation stages
constexpr int MAXST = 16;   // weight stages at most (used for small row tiles)
constexpr int EPI_BYTES = 32 * BM * 4;  // fp32 staging tile [32 rows][128 features]
constexpr int BAR_BYTES = 512;
constexpr int SMEM_BYTES = SMEM_TILES + BAR_BYTES + EPI_BYTES + 1024;
constexpr uint32_t TMEM_COLS = 512;
constexpr int NORM_SLOTS = 4;  // float4 slots per thread in a row norm (d <= 2048)

// global sync words of one launch site
enum : int { SY_O = 0, SY_N1 = 1, SY_D = 2, SY_N2 = 3, SY_QKV = 4, SY_FINISH = 5, SY_ABORT = 6, SY_GU = 16 };
enum : int { PH_O = 0, PH_GU = 1, PH_D = 2, PH_QKV = 3, NPH = 4 };

struct LtArgs {
  RowSet rs;
  KVView kv;
  const float2* rope;
  const __nv_bfloat16* mlp_norm;
  const __nv_bfloat16* norm2;
  __nv_bfloat16* act;
  __nv_bfloat16* u;
  __nv_bfloat16* q;
  float* Y;
  float* Ygu;  // gate/up split slices [split][256][2F] (separate: D writes Y while gate/up tiles are reduced)
  int* sync;
  int* status;
  int d, HQ, H, hd, F, kv_layer, flags;
  float eps;
  int sgrid[NPH];  // grid whose split count a phase reproduces (the per-kernel path's GEMM grid)
};

struct Ph {
  int on, N, K, ntn, kblocks, nrt, splits, items, lo, cnt;
};

struct Item {
  int n0, r0, rows, nbox, kb0, kb1, split, rt, tn;
};
__device__ __forceinline__ Item item_of(const Ph& p, int it, int R) {
  Item t;
  t.split = it % p.splits;
  const int tile = it / p.splits;
  t.tn = tile % p.ntn;
  t.rt = tile / p.ntn;
  t.n0 = t.tn * BM;
  t.r0 = t.rt * BNMAX;
  t.rows = min(BNMAX, R - t.r0);
  t.nbox = (t.rows + BOXN - 1) / BOXN;
  t.kb0 = (int)((long long)t.split * p.kblocks / p.splits);
  t.kb1 = (int)((long long)(t.split + 1) * p.kblocks / p.splits);
  return t;
}

// The four GEMM parts of this launch: every part is spread over all CTAs,
// K split as the per-kernel path splits it (tc_split_count), so that each
// CTA's share of a part's weights is a few tiles that its ring can hold
// before the part's activations are ready.
__device__ __forceinline__ void make_phases(const LtArgs& a, int R, int G, Ph* ph, int flags) {
  const int NK[NPH][2] = {{a.d, a.HQ}, {2 * a.F, a.d}, {a.d, a.F}, {3 * a.HQ, a.d}};
  const bool mlp = flags & LT_MLP, qkv = flags & LT_QKV;
  const bool on[NPH] = {mlp, mlp, mlp, qkv};
  for (int p = 0; p < NPH; ++p) {
    Ph& q = ph[p];
    q.on = on[p];
    q.N = NK[p][0];
    q.K = NK[p][1];
    q.ntn = q.N / BM;
    q.kblocks = q.K / BK;
    q.nrt = (R + BNMAX - 1) / BNMAX;
    q.splits = tc_split_count(R, q.N, q.K, a.sgrid[p], TC_MAX_SPLIT);
    q.items = q.ntn * q.nrt * q.splits;
    q.lo = 0;
    q.cnt = G;
  }
}
__device__ __forceinline__ bool mine(const Ph& p, int c) { return p.on && c >= p.lo && c < p.lo + p.cnt; }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ void store4_bf16(__nv_bfloat16* p, float a, float b, float c, float d) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
  uint2 v;
  v.x = *reinterpret_cast<uint32_t*>(&lo);
  v.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(p) = v;
}
__device__ __forceinline__ float4 add4(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

// k_epilogue's sum of the split slices adds all TC_MAX_SPLIT terms from 0,
// the ones past the split count being +0; adding +0 once after the real
// terms gives the same value (it only turns a -0 into +0).
__device__ __forceinline__ float pad_zero(float y, int ns) { return ns < TC_MAX_SPLIT ? y + 0.f : y; }

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// generic-proxy writes of this thread (or acquired from others) ordered
// before its later async-proxy (TMA) accesses of global memory
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Bounded poll until *p >= target.  False when the CTA or another CTA gave
// up, or when 2 s passed (then this CTA gives up and raises the global flag).
__device__ __noinline__ bool wait_geq(const int* p, int target, int* gabort, volatile int* sabort) {
  const unsigned long long t0 = global_ns();
  for (uint32_t i = 0;; ++i) {
    if (ld_acquire(p) >= target) return true;
    if (*sabort) return false;
    if ((i & 15u) == 15u) {
      if (ld_acquire(gabort)) {
        *sabort = 1;
        return false;
      }
      if (global_ns() - t0 > WAIT_NS) {
        *sabort = 1;
        atomicExch(gabort, 1);
        return false;
      }
    }
    if (i >= 512) __nanosleep(64);  // a tight poll first: most waits end within a few microseconds
  }
}

// ---------------------------------------------------------------------------
// row phases (epilogue warps, 128 threads)
// ---------------------------------------------------------------------------
// Residual from split slices, then RMSNorm into act: the reduction order of
// k_resid_norm (one float4 slot per thread of a CTA of ceil(d/4 / 32) warps)
// reproduced with 128 threads: thread t holds slots t + 128 c, whose warp
// there is t/32 + 4c; each such warp's sum is the same xor butterfly, and the
// warps' sums are added by one warp in warp order.
__device__ void rows_norm(const LtArgs& a, int R, int ns, int K, const __nv_bfloat16* g, float* s_red) {
  (void)K;
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  const int d = a.d, nv = d >> 2, nwarps = (nv + 31) / 32;
  const size_t sstride4 = (size_t)BNMAX * d / 4;
  for (int r = blockIdx.x; r < R; r += gridDim.x) {
    float4* hp = reinterpret_cast<float4*>(a.rs.h + (size_t)a.rs.row_hrow[r] * d);
    const float4* yp = reinterpret_cast<const float4*>(a.Y + (size_t)r * d);
    // the row's residual and the slices of four splits for every slot are
    // loaded together, then added in split order
    float4 x[NORM_SLOTS], ys[NORM_SLOTS], hv[NORM_SLOTS];
#pragma unroll
    for (int c = 0; c < NORM_SLOTS; ++c) {
      const int j = t + 128 * c;
      ys[c] = make_float4(0.f, 0.f, 0.f, 0.f);
      hv[c] = j < nv ? __ldcg(hp + j) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int s0 = 0; s0 < ns; s0 += 4) {
      float4 v[4][NORM_SLOTS];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int c = 0; c < NORM_SLOTS; ++c) {
          const int j = t + 128 * c;
          v[q][c] = (s0 + q < ns && j < nv) ? __ldcg(yp + (s0 + q) * sstride4 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (s0 + q < ns) {
#pragma unroll
          for (int c = 0; c < NORM_SLOTS; ++c) ys[c] = add4(ys[c], v[q][c]);
        }
    }
#pragma unroll
    for (int c = 0; c < NORM_SLOTS; ++c) {
      const int j = t + 128 * c;
      x[c] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j < nv) {
        const float4 y4 = make_float4(pad_zero(ys[c].x, ns), pad_zero(ys[c].y, ns), pad_zero(ys[c].z, ns),
                                      pad_zero(ys[c].w, ns));
        x[c] = add4(hv[c], y4);
        hp[j] = x[c];
      }
      const float ss = warp_sum(sumsq4(x[c]));
      if (lane == 0 && w + 4 * c < 16) s_red[w + 4 * c] = ss;
    }
    epi_bar();
    if (w == 0) {
      float tt = lane < nwarps ? s_red[lane] : 0.f;
      tt = warp_sum(tt);
      if (lane == 0) s_red[16] = tt;
    }
    epi_bar();
    const float inv = 1.0f / sqrtf(s_red[16] / (float)d + a.eps);
    epi_bar();
#pragma unroll
    for (int c = 0; c < NORM_SLOTS; ++c) {
      const int j = t + 128 * c;
      if (j < nv) {
        const __nv_bfloat16* gp = g + 4 * j;
        store4_bf16(a.act + (size_t)r * d + 4 * j, x[c].x * inv * __bfloat162float(gp[0]),
                    x[c].y * inv * __bfloat162float(gp[1]), x[c].z * inv * __bfloat162float(gp[2]),
                    x[c].w * inv * __bfloat162float(gp[3]));
      }
    }
  }
}


// h += slices (the last layer before an exit: no norm follows here).  Each
// thread takes four elements at a time and issues their slice loads together.
__device__ void rows_resid(const LtArgs& a, int R, int ns) {
  const long long stride = (long long)gridDim.x * 128;
  const size_t sstride = (size_t)BNMAX * a.d;
  const long long n_el = (long long)R * a.d;
  for (long long i0 = blockIdx.x * 128LL + threadIdx.x; i0 < n_el; i0 += 4 * stride) {
    float y[4] = {0.f, 0.f, 0.f, 0.f};
    const float* src[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const long long idx = i0 + e * stride;
      src[e] = idx < n_el ? a.Y + idx : nullptr;  // Y[0][r][n] with N = d: element idx
    }
    for (int s0 = 0; s0 < ns; s0 += 8) {
      float v[8][4];
#pragma unroll
      for (int q = 0; q < 8; ++q)
#pragma unroll
        for (int e = 0; e < 4; ++e) v[q][e] = (s0 + q < ns && src[e]) ? __ldcg(src[e] + (s0 + q) * sstride) : 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (s0 + q < ns) {
#pragma unroll
          for (int e = 0; e < 4; ++e) y[e] += v[q][e];
        }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (!src[e]) continue;
      const long long idx = i0 + e * stride;
      const int r = (int)(idx / a.d), n = (int)(idx % a.d);
      float* hp = a.rs.h + (size_t)a.rs.row_hrow[r] * a.d + n;
      *hp = __ldcg(hp) + pad_zero(y[e], ns);
    }
  }
}

// E: q, k, v from the slices, RoPE, stores (k_epilogue's EPI_QKV per
// element).  A thread takes four consecutive rotation pairs of one head (16
// bytes of each half), two such quads at a time: every slice load and the
// row indices are issued first, the RoPE table (which needs the position)
// second.
__device__ __forceinline__ void store_bf16x4(__nv_bfloat16* p, float a, float b, float c, float d) {
  store4_bf16(p, a, b, c, d);
}
__device__ void qkv_epilogue(const LtArgs& a, int R, int ns) {
  const int half = a.hd / 2, N = 3 * a.HQ, qph = half / 4;  // quads per head
  const int per_row = 3 * a.H * qph;
  const long long stride = (long long)gridDim.x * 128;
  const size_t sstride4 = (size_t)BNMAX * N / 4;
  const long long n_q = (long long)R * per_row;
  const float4* Y4 = reinterpret_cast<const float4*>(a.Y);
  for (long long q0 = blockIdx.x * 128LL + threadIdx.x; q0 < n_q; q0 += 2 * stride) {
    int r[2], c0[2], h3[2];
    bool on[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const long long qd = q0 + e * stride;
      on[e] = qd < n_q;
      const long long id = on[e] ? qd : q0;
      r[e] = (int)(id / per_row);
      const int rem = (int)(id % per_row);
      h3[e] = rem / qph;
      c0[e] = h3[e] * a.hd + (rem % qph) * 4;
    }
    int pos[2], rb[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      pos[e] = a.rs.row_pos[r[e]];
      rb[e] = a.rs.row_b[r[e]];
    }
    float4 y0[2], y1[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) y0[e] = y1[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < ns; s0 += 4) {
      float4 v[4][4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float4* p = Y4 + (s0 + q) * sstride4 + ((size_t)r[e] * N + c0[e]) / 4;
          const bool ld = s0 + q < ns && on[e];
          v[q][2 * e] = ld ? __ldcg(p) : make_float4(0.f, 0.f, 0.f, 0.f);
          v[q][2 * e + 1] = ld ? __ldcg(p + half / 4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (s0 + q < ns) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            y0[e] = add4(y0[e], v[q][2 * e]);
            y1[e] = add4(y1[e], v[q][2 * e + 1]);
          }
        }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      if (!on[e]) continue;
      const int part = h3[e] / a.H, head = h3[e] % a.H, i = c0[e] % a.hd;
      float z0[4] = {pad_zero(y0[e].x, ns), pad_zero(y0[e].y, ns), pad_zero(y0[e].z, ns), pad_zero(y0[e].w, ns)};
      float z1[4] = {pad_zero(y1[e].x, ns), pad_zero(y1[e].y, ns), pad_zero(y1[e].z, ns), pad_zero(y1[e].w, ns)};
      if (part < 2) {
        const float4* cs4 = reinterpret_cast<const float4*>(a.rope + (size_t)pos[e] * half + i);
        const float4 ca = cs4[0], cb = cs4[1];
        const float2 cs[4] = {make_float2(ca.x, ca.y), make_float2(ca.z, ca.w), make_float2(cb.x, cb.y),
                              make_float2(cb.z, cb.w)};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 u = rope_pair(z0[k], z1[k], cs[k]);
          z0[k] = u.x;
          z1[k] = u.y;
        }
      }
      __nv_bfloat16* dst;
      if (part == 0) dst = a.q + (size_t)r[e] * a.HQ + head * a.hd;
      else dst = (__nv_bfloat16*)a.kv.base + a.kv.offset(a.kv_layer, rb[e], pos[e], head, part - 1);
      store_bf16x4(dst + i, z0[0], z0[1], z0[2], z0[3]);
      store_bf16x4(dst + i + half, z1[0], z1[1], z1[2], z1[3]);
    }
  }
}

__global__ void __launch_bounds__(LT_THREADS, 1)
    k_layer_tc(const __grid_constant__ CUtensorMap m_wo, const __grid_constant__ CUtensorMap m_wgu,
               const __grid_constant__ CUtensorMap m_wd, const __grid_constant__ CUtensorMap m_wqkv,
               const __grid_constant__ CUtensorMap m_xo, const __grid_constant__ CUtensorMap m_xact,
               const __grid_constant__ CUtensorMap m_xu, LtArgs a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort, s_go, s_last;
  __shared__ float s_red[20];
  const CUtensorMap* wmap[NPH] = {&m_wo, &m_wgu, &m_wd, &m_wqkv};
  const CUtensorMap* xmap[NPH] = {&m_xo, &m_xact, &m_xu, &m_xact};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, c = blockIdx.x;

  // Before waiting for the previous kernel (nothing here reads what it
  // writes): pull this CTA's first weight tiles into L2, for the schedule
  // of a launch whose rows fit one tile (every decode step in practice).
  if (threadIdx.x == W_WARP * 32) {
    for (int i = 0; i < NPH; ++i) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(wmap[i])) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(xmap[i])) : "memory");
    }
    Ph ph[NPH];
    make_phases(a, 1, G, ph, a.flags);
    int n = 0;
    for (int p = 0; p < NPH && n < MAXST; ++p) {
      if (!mine(ph[p], c)) continue;
      for (int it = c - ph[p].lo; it < ph[p].items && n < MAXST; it += ph[p].cnt) {
        const Item t = item_of(ph[p], it, 1);
        for (int kb = t.kb0; kb < t.kb1 && n < MAXST; ++kb, ++n) tma_prefetch_l2_2d(wmap[p], kb * BK, t.n0);
      }
    }
  }
  pdl_wait();
  pdl_launch();
  const int R = *a.rs.nrows;
  if (R <= 0) return;
  Ph ph[NPH];
  make_phases(a, R, G, ph, a.flags);
  int* sync = a.sync;
  int* gabort = sync + SY_ABORT;

  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int nbmax = (min(R, BNMAX) + BOXN - 1) / BOXN;
  const int xstage_bytes = nbmax * BOX_BYTES;
  const int nwst = min(MAXST, (SMEM_TILES - XST * xstage_bytes) / A_BYTES);
  unsigned char* xring = smem + nwst * A_BYTES;
  uint64_t* fullw = (uint64_t*)(smem + SMEM_TILES);
  uint64_t* emptyw = fullw + MAXST;
  uint64_t* fullx = emptyw + MAXST;
  uint64_t* emptyx = fullx + XST;
  uint64_t* tfull = emptyx + XST;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  float* stile = (float*)(smem + SMEM_TILES + BAR_BYTES);

  if (threadIdx.x == 0) {
    for (int s = 0; s < nwst; ++s) {
      mbar_init(fullw + s, 1);
      mbar_init(emptyw + s, 1);
    }
    for (int s = 0; s < XST; ++s) {
      mbar_init(fullx + s, 1);
      mbar_init(emptyx + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(tfull + s, 1);
      mbar_init(tempty + s, 128);
    }
    mbar_init(drain, 1);
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

  if (warp == W_WARP || warp == X_WARP) {
    // producers: the same walk over (part, item, K block); warp 4 fills the
    // weight ring, warp 6 the activation ring
    if (lane == 0) {
      const bool isw = warp == W_WARP;
      uint64_t* full = isw ? fullw : fullx;
      uint64_t* empty = isw ? emptyw : emptyx;
      const int nst = isw ? nwst : XST;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int issued[MAXST];
#pragma unroll
      for (int s = 0; s < MAXST; ++s) issued[s] = -1;
      for (int p = 0; p < NPH && ok; ++p) {
        if (!mine(ph[p], c)) continue;
        bool dep_done = isw || p == PH_O || (p == PH_QKV && !(a.flags & LT_MLP));
        for (int it = c - ph[p].lo; it < ph[p].items && ok; it += ph[p].cnt) {
          const Item t = item_of(ph[p], it, R);
          if (!isw) {
            // the activations this item reads must be complete
            if (p == PH_D) {
              const int* f = sync + SY_GU + t.rt * ph[PH_GU].ntn;
              for (int j = t.kb0; j < t.kb1 && ok; ++j) ok = wait_geq(f + j, 1, gabort, abort_flag);
            } else if (!dep_done) {
              ok = wait_geq(sync + (p == PH_GU ? SY_N1 : SY_N2), R, gabort, abort_flag);
              dep_done = true;
            }
            if (!ok) break;
            fence_proxy_async_global();
          }
          for (int kb = t.kb0; kb < t.kb1; ++kb) {
            if (!mbar_wait(empty + stage, phase ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            issued[stage] = (int)phase;
            if (isw) {
              mbar_expect_tx(full + stage, (uint32_t)A_BYTES);
              tma_load_2d(smem + stage * A_BYTES, wmap[p], full + stage, kb * BK, t.n0);
            } else {
              unsigned char* sx = xring + stage * xstage_bytes;
              mbar_expect_tx(full + stage, (uint32_t)(t.nbox * BOX_BYTES));
              for (int j = 0; j < t.nbox; ++j)
                tma_load_2d(sx + j * BOX_BYTES, xmap[p], full + stage, kb * BK, t.r0 + j * BOXN);
            }
            if (++stage == nst) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
      if (*abort_flag) {
        // let the copies already issued land before the CTA leaves (bounded)
        volatile int never = 0;
        for (int s = 0; s < nst; ++s)
          if (issued[s] >= 0) mbar_wait(full + s, (uint32_t)issued[s], &never, WAIT_NS / 4);
      }
    }
  } else if (warp == MMA_WARP) {
    if (lane == 0) {
      int ws = 0, xs = 0, acc = 0;
      uint32_t wphase = 0, xphase = 0, aphase = 0;
      bool ok = true, issued_any = false;
      for (int p = 0; p < NPH && ok; ++p) {
        if (!mine(ph[p], c)) continue;
        for (int it = c - ph[p].lo; it < ph[p].items && ok; it += ph[p].cnt) {
          const Item t = item_of(ph[p], it, R);
          const uint32_t idesc = idesc_bf16(t.nbox * BOXN);
          if (!mbar_wait(tempty + acc, aphase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t dt = tmem + (uint32_t)(acc * BNMAX);
          for (int kb = t.kb0; kb < t.kb1; ++kb) {
            if (!mbar_wait(fullw + ws, wphase, abort_flag) || !mbar_wait(fullx + xs, xphase, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t ad = sw128_desc(smem_u32(smem + ws * A_BYTES));
            const uint64_t bd = sw128_desc(smem_u32(xring + xs * xstage_bytes));
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma(dt, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc, (kb > t.kb0 || kk > 0) ? 1u : 0u);
            issued_any = true;
            umma_commit(emptyw + ws);
            umma_commit(emptyx + xs);
            if (++ws == nwst) {
              ws = 0;
              wphase ^= 1u;
            }
            if (++xs == XST) {
              xs = 0;
              xphase ^= 1u;
            }
          }
          if (!ok) break;
          umma_commit(tfull + acc);
          acc ^= 1;
          if (acc == 0) aphase ^= 1u;
        }
      }
      if (!ok && issued_any) {
        // the MMAs already issued finish before the accumulators are freed
        umma_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, &never, WAIT_NS / 4);
      }
    }
  } else {
    // epilogue warps 0..3: TMEM lanes 32*warp .. 32*warp+31
    int acc = 0;
    uint32_t aphase = 0;
    bool ok = true;
    for (int p = 0; p < NPH && ok; ++p) {
      if (!ph[p].on) continue;
      if (mine(ph[p], c)) {
        for (int it = c - ph[p].lo; it < ph[p].items; it += ph[p].cnt) {
          const Item t = item_of(ph[p], it, R);
          if (threadIdx.x == 0) s_go = mbar_wait(tfull + acc, aphase, abort_flag) ? 1 : 0;
          epi_bar();
          if (!s_go) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t tbase = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(acc * BNMAX);
          bool publish = true;
          if (p == PH_GU) {
            // SwiGLU over the tile's 64 gate and 64 matching up features, from
            // the sum of its K splits: every split but the last to finish
            // leaves its partial sums in memory; the last one adds them in
            // split order to its own (still in TMEM), as k_epilogue does
            const int ns = ph[p].splits, gn = 2 * a.F;
            const int col = t.n0 + warp * 32 + lane;
            const int tile_idx = t.rt * ph[PH_GU].ntn + t.tn;
            const size_t gstride = (size_t)BNMAX * gn;
            if (ns > 1) {
              float* Ys = a.Ygu + (size_t)t.split * gstride;
              for (int c0 = 0; c0 < t.nbox * BOXN; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tbase + (uint32_t)c0, v);
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                  const int r = t.r0 + c0 + j;
                  if (r < R) Ys[(size_t)r * gn + col] = __uint_as_float(v[j]);
                }
              }
              __threadfence();
              epi_bar();
              if (threadIdx.x == 0)
                s_go = atomicAdd(sync + SY_GU + ph[PH_GU].nrt * ph[PH_GU].ntn + tile_idx, 1) == ns - 1 ? 1 : 0;
              epi_bar();
              publish = s_go != 0;
              // every thread has read the decision before thread 0 reuses s_go
              epi_bar();
              if (publish) __threadfence();
            }
            if (publish) {
              for (int c0 = 0; c0 < t.nbox * BOXN; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tbase + (uint32_t)c0, v);
                // y = 0 + slice 0 + slice 1 + ..., each other split's 32 rows
                // loaded together; v (this split, from TMEM) enters at its turn
                float y[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) y[j] = 0.f;
                for (int sp = 0; sp < ns; ++sp) {
                  if (sp == t.split) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) y[j] += __uint_as_float(v[j]);
                  } else {
                    const float* src = a.Ygu + sp * gstride + (size_t)(t.r0 + c0) * gn + col;
#pragma unroll
                    for (int j = 0; j < 32; ++j) y[j] += t.r0 + c0 + j < R ? __ldcg(src + (size_t)j * gn) : 0.f;
                  }
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) stile[j * BM + warp * 32 + lane] = pad_zero(y[j], ns);
                epi_bar();
                const int nrows = min(32, R - (t.r0 + c0));
#pragma unroll 4
                for (int idx = threadIdx.x; idx < nrows * (BM / 2); idx += 128) {
                  const int j = idx / (BM / 2), jj = idx % (BM / 2);
                  const float gv = stile[j * BM + jj], uv = stile[j * BM + BM / 2 + jj];
                  a.u[(size_t)(t.r0 + c0 + j) * a.F + (t.n0 / BM) * (BM / 2) + jj] =
                      __float2bfloat16_rn(swiglu(gv, uv));
                }
                epi_bar();
              }
            }
          } else {
            const int n = t.n0 + warp * 32 + lane;
            float* Ys = a.Y + (size_t)t.split * ((size_t)BNMAX * ph[p].N);
            for (int c0 = 0; c0 < t.nbox * BOXN; c0 += 32) {
              uint32_t v[32];
              tmem_ld32(tbase + (uint32_t)c0, v);
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int r = t.r0 + c0 + j;
                if (r < R) Ys[(size_t)r * ph[p].N + n] = __uint_as_float(v[j]);
              }
            }
          }
          tc_fence_before();
          mbar_arrive(tempty + acc);
          acc ^= 1;
          if (acc == 0) aphase ^= 1u;
          // publish: this item's outputs, then its counter or (the split that
          // finished a gate/up tile) the tile's ready flag
          if (publish) {
            // the barrier orders every thread's stores before thread 0's
            // release; TMA (the async proxy) reads the gate/up output
            if (p == PH_GU) fence_proxy_async_global();
            epi_bar();
            if (threadIdx.x == 0) {
              if (p == PH_GU) red_release_add(sync + SY_GU + t.rt * ph[PH_GU].ntn + t.tn, 1);
              else red_release_add(sync + (p == PH_O ? SY_O : p == PH_D ? SY_D : SY_QKV), 1);
            }
          }
        }
        if (!ok) break;
      }
      // the row parts that follow a GEMM part (every CTA takes part)
      if (p == PH_O || p == PH_D || p == PH_QKV) {
        const int ctr = p == PH_O ? SY_O : p == PH_D ? SY_D : SY_QKV;
        if (threadIdx.x == 0) s_go = wait_geq(sync + ctr, ph[p].items, gabort, abort_flag) ? 1 : 0;
        epi_bar();
        if (!s_go) {
          ok = false;
          break;
        }
        if (p == PH_QKV) {
          qkv_epilogue(a, R, ph[p].splits);
        } else if (p == PH_D && !(a.flags & LT_NORM2)) {
          rows_resid(a, R, ph[p].splits);
        } else {
          const __nv_bfloat16* g = p == PH_O ? a.mlp_norm : a.norm2;
          rows_norm(a, R, ph[p].splits, ph[p].K, g, s_red);
          // publish the normed rows (TMA reads them in other CTAs)
          fence_proxy_async_global();
          epi_bar();
          int mine_rows = 0;
          for (int r = blockIdx.x; r < R; r += gridDim.x) ++mine_rows;
          if (threadIdx.x == 0 && mine_rows) red_release_add(sync + (p == PH_O ? SY_N1 : SY_N2), mine_rows);
        }
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
  if (threadIdx.x == 0) {
    if (s_abort) {
      dev_fail(a.status, DEV_ERR_TIMEOUT);
      atomicExch(gabort, 1);
    }
    __threadfence();
    s_last = atomicAdd(sync + SY_FINISH, 1) == G - 1;
  }
  __syncthreads();
  if (s_last) {
    // every CTA is past its last use of the sync words: zero them for the next launch
    __threadfence();
    // gate/up ready flags, then the gate/up split arrival counters
    const int nflags = ph[PH_GU].nrt * ph[PH_GU].ntn;
    for (int i = threadIdx.x; i < SY_GU + 2 * nflags; i += blockDim.x) sync[i] = 0;
  }
}

}  // namespace

size_t layer_tc_sync_ints(int max_rows, int F) {
  const size_t nrt = ((size_t)max_rows + BNMAX - 1) / BNMAX;
  return SY_GU + 2 * nrt * (size_t)(2 * F / BM);
}

size_t layer_tc_gu_floats(int F) { return (size_t)TC_MAX_SPLIT * BNMAX * 2 * F; }

bool layer_tc_supported(int d, int HQ, int hd, int F, bool bf16) {
  return bf16 && hd == 64 && d % BM == 0 && HQ % BM == 0 && F % 64 == 0 && (2 * F) % BM == 0 && d <= 2048 &&
         d / 4 <= 128 * NORM_SLOTS;
}

nv_status layer_tc_prepare() {
  cudaError_t e = cudaFuncSetAttribute(k_layer_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) {
    set_error(std::string("decode-layer kernel shared memory: ") + cudaGetErrorString(e));
    return NV_ERR_UNSUPPORTED;
  }
  return NV_OK;
}

nv_status layer_tc_launch(TcPlanCache* plans, const LayerTcRun& r, cudaStream_t st) {
  const int d = r.d, HQ = r.HQ, F = r.F;
  const int max_rows = r.rs.max_rows;
  const bool mlp = r.flags & LT_MLP, qkv = r.flags & LT_QKV;
  if (!mlp && !qkv) return NV_OK;
  CUtensorMap m[7];
  // maps of unused parts repeat a used one (never read)
  const void* wo = mlp ? r.w_o : r.w_qkv;
  const void* wgu = mlp ? r.w_gu : r.w_qkv;
  const void* wd = mlp ? r.w_d : r.w_qkv;
  const void* wq = qkv ? r.w_qkv : r.w_o;
  if (mlp) {
    NV_TRY(tc_map(plans, wo, (uint64_t)HQ, (uint64_t)d, (uint64_t)HQ, BM, &m[0]));
    NV_TRY(tc_map(plans, wgu, (uint64_t)d, (uint64_t)(2 * F), (uint64_t)d, BM, &m[1]));
    NV_TRY(tc_map(plans, wd, (uint64_t)F, (uint64_t)d, (uint64_t)F, BM, &m[2]));
    NV_TRY(tc_map(plans, r.o, (uint64_t)HQ, (uint64_t)max_rows, (uint64_t)HQ, BOXN, &m[4]));
    NV_TRY(tc_map(plans, r.u, (uint64_t)F, (uint64_t)max_rows, (uint64_t)F, BOXN, &m[6]));
  }
  if (qkv) NV_TRY(tc_map(plans, wq, (uint64_t)d, (uint64_t)(3 * HQ), (uint64_t)d, BM, &m[3]));
  NV_TRY(tc_map(plans, r.act, (uint64_t)d, (uint64_t)max_rows, (uint64_t)d, BOXN, &m[5]));
  if (!mlp) m[0] = m[1] = m[2] = m[3], m[4] = m[6] = m[5];
  if (!qkv) m[3] = m[0];

  const int G = tc_sm_count();
  LtArgs a{};
  a.rs = r.rs;
  a.kv = r.kv;
  a.rope = r.rope;
  a.mlp_norm = (const __nv_bfloat16*)r.mlp_norm;
  a.norm2 = (const __nv_bfloat16*)r.norm2;
  a.act = (__nv_bfloat16*)r.act;
  a.u = (__nv_bfloat16*)r.u;
  a.q = (__nv_bfloat16*)r.q;
  a.Y = r.Y;
  a.Ygu = r.Ygu;
  a.sync = r.sync;
  a.status = r.status;
  a.d = d;
  a.HQ = HQ;
  a.H = r.H;
  a.hd = r.hd;
  a.F = F;
  a.kv_layer = r.kv_layer;
  a.flags = r.flags;
  a.eps = r.eps;
  // the split counts of the per-kernel path: its GEMM grid is the SM count,
  // capped by the work items it could have (feature tiles x row tiles x 16)
  const int nrt_max = (max_rows + BNMAX - 1) / BNMAX;
  const int NN[NPH] = {d, 2 * F, d, 3 * HQ};
  for (int p = 0; p < NPH; ++p) {
    const long long most = (long long)(NN[p] / BM) * nrt_max * TC_MAX_SPLIT;
    a.sgrid[p] = most < G ? (int)most : G;
  }
  cudaError_t e = launch_k(k_layer_tc, dim3(G), dim3(LT_THREADS), SMEM_BYTES, st, m[0], m[1], m[2], m[3], m[4], m[5],
                           m[6], a);
  if (e != cudaSuccess) {
    set_error(std::string("decode-layer kernel launch: ") + cudaGetErrorString(e));
    return NV_ERR_CUDA;
  }
  return NV_OK;
}

}  // namespace nv
