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
//   warp 4, one lane: TMA producer, ring of (W tile 128x64, X tile
//                     <=256x64) stages, 128-byte swizzle, mbarrier
//                     complete_tx; the stage count follows the row tile (4
//                     stages at 256 rows, up to 12 for a handful of rows);
//   warp 5, one lane: issues tcgen05.mma (kind::f16, M=128, N=32..256,
//                     K=16) into one of two TMEM accumulators, commits to the
//                     stage's "empty" barrier and to "accumulator full";
//   warps 0-3:        epilogue, tcgen05.ld 32 columns at a time and coalesced
//                     fp32 stores (each warp owns 32 features = TMEM lanes).
// When all rows fit one tile and the feature tiles cannot fill the GPU, the K
// range is split (tc_split_count); the partial slices are summed in a fixed
// order by the epilogue kernel that follows.  Without a split, the layer
// epilogue (RoPE + KV write, residual, SwiGLU) runs in the epilogue warps
// from a staged tile (or, for the exit heads, the Gumbel-max sampler and
// log-sum-exp of each 128-token tile).  Before griddepcontrol.wait a CTA pulls
// its own first weight tiles and the next GEMM's weights into L2.  Every
// mbarrier wait is bounded: on expiry the CTA flags DEV_ERR_TIMEOUT, stops
// issuing work, frees its TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include "gemm.cuh"
#include "gemm_tc.cuh"
#include "kernels.cuh"
#include "tc_prims.cuh"

namespace nv {
namespace {
using namespace tc;

constexpr int STAGES = 4;        // stages at the largest row tile (256 rows)
constexpr int MAXST = 12;        // stages when the row tile is small
constexpr int B_BYTES = BNMAX * BK * 2;
constexpr int SMEM_TILES = STAGES * (A_BYTES + B_BYTES);
// Epilogue: one or two groups of four warps (warp w reads TMEM lanes
// 32*(w%4)..+31); with two, group g takes the 16-column accumulator chunks
// 2k+g of a tile, so two chunks are in flight at once.  Launches that may
// split K (decode: a few rows, fp32 slices) run one group; the others two.
// The TMA and MMA warps follow the epilogue warps.
constexpr int EPI_WARPS = 8;  // at most
constexpr int EPI_THREADS = EPI_WARPS * 32;
constexpr int WARP_TMA = EPI_WARPS, WARP_MMA = EPI_WARPS + 1;  // with two groups
constexpr int EPI_ROWS = 16;                        // rows per staged chunk (one 32x32b.x16 TMEM load)
constexpr int EPI_BYTES = 2 * EPI_ROWS * BM * 4;    // fp32 staging tile [16 rows][128 features] per group
// per-row data of the fused epilogue, two tiles deep: [2][BNMAX] offsets + [2][BNMAX] ints
constexpr int META_BYTES = 2 * BNMAX * (8 + 4);
constexpr int SMEM_BYTES = SMEM_TILES + 512 /*barriers*/ + EPI_BYTES + META_BYTES + 1024 /*align*/;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory of one CTA");
constexpr uint32_t TMEM_COLS = 512;  // two 256-column fp32 accumulators
constexpr int THREADS = EPI_THREADS + 64;  // + the TMA warp and the MMA warp (two groups)
constexpr int THREADS_1G = 128 + 64;        // one epilogue group
// row tiles per band of the tile order: within a band the row tile changes
// fastest, so each weight tile is read once per band and the band's rows
// (16 x 256 rows) stay in L2 while the feature tiles sweep past
constexpr int RBAND = 16;

struct TcArgs {
  const int* nrows;
  float* Y;
  int N, K;
  int max_split;
  size_t split_stride;
  int* status;
  int fused;             // apply `epi` in-kernel (one K slice only; else store fp32 Y)
  const int* skip_if_zero;      // when set and *skip_if_zero == 0 the launch does nothing
  const unsigned char* pf_ptr;  // bytes to pull into L2 for the next GEMM (may be null)
  unsigned long long pf_bytes;
  EpiArgs epi;
};

struct Item {
  int n0, r0, rows, nbox, kb0, kb1, split;
};
// fw: features per tile (128, or 256 for a CTA pair)
__device__ __forceinline__ Item decode_item(int it, int ntn, int splits, int R, int kblocks, int fw = BM) {
  Item t;
  t.split = it % splits;
  const int tile = it / splits;
  const int nrt = (R + BNMAX - 1) / BNMAX;
  const int band = tile / (ntn * RBAND), rt0 = band * RBAND, gb = min(RBAND, nrt - rt0);
  const int local = tile - band * ntn * RBAND;
  t.n0 = (local / gb) * fw;
  t.r0 = (rt0 + local % gb) * BNMAX;
  t.rows = min(BNMAX, R - t.r0);
  t.nbox = (t.rows + BOXN - 1) / BOXN;
  t.kb0 = (int)((long long)t.split * kblocks / splits);
  t.kb1 = (int)((long long)(t.split + 1) * kblocks / splits);
  return t;
}

// all epilogue warps (ng groups); the four warps of group g
__device__ __forceinline__ void epi_bar(int ng) { asm volatile("bar.sync 1, %0;" ::"r"(ng * 128) : "memory"); }
__device__ __forceinline__ void grp_bar(int g) { asm volatile("bar.sync %0, 128;" ::"r"(2 + g) : "memory"); }

// Per-row data of a fused epilogue, gathered into shared memory by the
// epilogue threads before they wait for the tile's accumulator, so these
// loads overlap the tile's MMAs instead of sitting inside the per-element
// loops.  off[j] / iv[j] for row r0 + j of the tile:
//   EPI_QKV:   iv = position; off = element offset of the row in q (part q),
//              or of its slot in the KV page with head 0 and the K half
//              (parts k, v: the head and half add (half*H + head)*page*hd)
//   EPI_RESID: off = element offset of the row's residual in h
//   EPI_HEAD:  iv = the token position t[b] when sequence b stopped here, else -1
//   EPI_LSE:   iv = the row's target token
__device__ __forceinline__ void load_row_meta(const EpiArgs& e, int n0, int r0, int rows, long long* off, int* iv,
                                              int nthreads) {
  for (int j = threadIdx.x; j < rows; j += nthreads) {
    const int r = r0 + j;
    if (e.mode == EPI_QKV) {
      const int pos = e.rs.row_pos[r];
      iv[j] = pos;
      off[j] = n0 < e.H * e.hd ? (long long)r * (e.H * e.hd)
                               : (long long)e.kv.offset(e.layer, e.rs.row_b[r], pos, 0, 0);
    } else if (e.mode == EPI_RESID) {
      off[j] = (long long)e.rs.row_hrow[r] * e.d;
      // the tile's 128 residual values of the row (512 bytes) into L2
      const float* hp = e.rs.h + off[j] + n0;
#pragma unroll
      for (int q = 0; q < 4; ++q) asm volatile("prefetch.global.L2 [%0];" ::"l"(hp + 32 * q));
    } else if (e.mode == EPI_HEAD) {
      iv[j] = e.stop[r] ? e.t[r] : -1;
    } else if (e.mode == EPI_LSE) {
      iv[j] = e.lse_target[r];
    }
  }
}

__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// EPI_QKV in two steps around the staging barrier.  Thread gt of a group
// (0..127) takes rotary pair p = gt % 64 of the tile's 128 features (feature
// f0 of its head half and f0 + hd/2) in rows gt / 64, gt / 64 + 2, ... of the
// group's staged chunk: first it loads the
// (cos, sin) entries of its rows, all independent loads, then (tile staged)
// it rotates q and k, and writes q rows or the paged K / V cache.
constexpr int QKV_RPT = EPI_ROWS / 2;  // rows per thread of a staged chunk
__device__ __forceinline__ void qkv_load_rope(const EpiArgs& e, int n0, int nrows, const int* iv, int gt,
                                              float2 (&cs)[QKV_RPT]) {
  const int half = e.hd / 2, pr = gt & 63, j0 = gt >> 6, i = pr % half;
  const bool rot = n0 < 2 * e.H * e.hd;  // q or k
#pragma unroll
  for (int k = 0; k < QKV_RPT; ++k) {
    const int j = j0 + 2 * k;
    cs[k] = rot && j < nrows ? __ldg(e.rope + (size_t)iv[j] * half + i) : make_float2(1.f, 0.f);
  }
}
__device__ __forceinline__ void qkv_store(const EpiArgs& e, const float* S, int n0, int nrows, const long long* off,
                                          int gt, const float2 (&cs)[QKV_RPT]) {
  const int half = e.hd / 2, HQ = e.H * e.hd, part = n0 / HQ;
  const int pr = gt & 63, j0 = gt >> 6;
  const int f0 = (pr / half) * e.hd + pr % half;
  const int nl = n0 % HQ + f0;  // feature within q, k or v
  const int head = nl / e.hd, i = nl % e.hd;
  const size_t fo = part == 0 ? (size_t)head * e.hd + i
                              : (size_t)((part - 1) * e.H + head) * e.kv.page_size * e.hd + i;
  __nv_bfloat16* base = part == 0 ? (__nv_bfloat16*)e.q_out : (__nv_bfloat16*)e.kv.base;
#pragma unroll
  for (int k = 0; k < QKV_RPT; ++k) {
    const int j = j0 + 2 * k;
    if (j < nrows) {
      float y0 = S[j * BM + f0], y1 = S[j * BM + f0 + half];
      if (part < 2) {
        const float2 u = rope_pair(y0, y1, cs[k]);
        y0 = u.x;
        y1 = u.y;
      }
      __nv_bfloat16* dst = base + off[j] + fo;
      dst[0] = __float2bfloat16_rn(y0);
      dst[half] = __float2bfloat16_rn(y1);
    }
  }
}

// Apply the layer epilogue to a staged tile: S[j][f] = y for row r0 + j and
// feature n0 + f (f < 128); off / iv are the rows' entries of load_row_meta.
// Run by the 128 threads of epilogue group g (gt = 0..127).
//   EPI_SWIGLU: the tile holds 64 gate rows then the 64 matching up rows.
//   EPI_HEAD / EPI_LSE: per-row reductions over the tile's 128 tokens.
// (EPI_RESID runs from the accumulator registers, without staging; EPI_QKV
// is qkv_load_rope / qkv_store above.)
__device__ __forceinline__ void tile_epilogue(const EpiArgs& e, const float* S, int n0, int r0, int nrows,
                                              const long long* off, const int* iv, int gt, int g) {
  const int tid = gt;
  if (e.mode == EPI_HEAD) {
    // exact sampling at this exit: score_v = logit_v + Gumbel(U_v), U_v from
    // Philox counter (b, t, 1, v/4) lane v%4; argmax with ties to the lowest
    // v, and the log-sum-exp of the logits, over this tile's 128 v.  A warp
    // takes whole rows (rows w, w+4, ...), a lane the 4 tokens of one Philox
    // block (v = n0 + 4 lane + i), then a butterfly over the warp.
    const unsigned long long seed = *e.seed;
    const int lane = tid & 31, w = tid >> 5;
    for (int j = w; j < nrows; j += 4) {
      const int b = r0 + j, tb = iv[j];
      if (tb < 0) continue;  // same row for the whole warp: uniform
      const int v0 = n0 + 4 * lane;
      const uint4 rb = philox4x32_10(make_uint4((uint32_t)b, (uint32_t)tb, STREAM_GUMBEL, (uint32_t)(v0 >> 2)),
                                     (uint32_t)seed, (uint32_t)(seed >> 32));
      const float* row = S + j * BM + 4 * lane;
      float bs = -INFINITY, bl = 0.f, M = -INFINITY;
      int bv = v0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float logit = row[i];
        const float sc = logit - logf(-logf(uniform01(lane_of(rb, i))));
        if (sc > bs) {  // ascending v: ties keep the lowest
          bs = sc;
          bv = v0 + i;
          bl = logit;
        }
        M = fmaxf(M, logit);
      }
      float Ssum = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) Ssum += expf(row[i] - M);
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        const float s2 = __shfl_xor_sync(0xffffffffu, bs, o);
        const int v2 = __shfl_xor_sync(0xffffffffu, bv, o);
        const float l2 = __shfl_xor_sync(0xffffffffu, bl, o);
        const float M2 = __shfl_xor_sync(0xffffffffu, M, o);
        const float S2 = __shfl_xor_sync(0xffffffffu, Ssum, o);
        if (s2 > bs || (s2 == bs && v2 < bv)) {
          bs = s2;
          bv = v2;
          bl = l2;
        }
        const float Mn = fmaxf(M, M2);
        Ssum = Ssum * expf(M - Mn) + S2 * expf(M2 - Mn);
        M = Mn;
      }
      if (lane == 0) {
        float* out = e.head_part + ((size_t)b * e.nblk + n0 / BM) * HEAD_PART;
        out[0] = bs;
        out[1] = __int_as_float(bv);
        out[2] = bl;
        out[3] = M;
        out[4] = Ssum;
      }
    }
  } else if (e.mode == EPI_LSE) {
    // scoring head: for each row of the tile, the max of this tile's 128
    // logits (lanes take 4 tokens each, then a butterfly), then the sum of
    // exp(logit - max) as 2^((logit - max) log2 e) with the hardware's
    // base-2 exponential (relative error near 2^-22 per term), and the
    // target token's logit when the target falls in this tile
    const int lane = tid & 31, w = tid >> 5;
    constexpr float LOG2E = 1.4426950408889634f;
    // a warp takes rows w, w+4, w+8, w+12 of the staged chunk together, so
    // the four rows' butterflies interleave instead of running one by one
    constexpr int RPW = EPI_ROWS / 4;
    float x[RPW][4], M[RPW], Ssum[RPW];
#pragma unroll
    for (int k = 0; k < RPW; ++k) {
      const int j = w + 4 * k;
#pragma unroll
      for (int i = 0; i < 4; ++i) x[k][i] = j < nrows ? S[j * BM + lane + 32 * i] : 0.f;
      M[k] = fmaxf(fmaxf(x[k][0], x[k][1]), fmaxf(x[k][2], x[k][3]));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
#pragma unroll
      for (int k = 0; k < RPW; ++k) M[k] = fmaxf(M[k], __shfl_xor_sync(0xffffffffu, M[k], o));
#pragma unroll
    for (int k = 0; k < RPW; ++k) {
      Ssum[k] = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) Ssum[k] += exp2_approx(__fmul_rn(x[k][i] - M[k], LOG2E));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
#pragma unroll
      for (int k = 0; k < RPW; ++k) Ssum[k] += __shfl_xor_sync(0xffffffffu, Ssum[k], o);
#pragma unroll
    for (int k = 0; k < RPW; ++k) {
      const int j = w + 4 * k;
      if (j >= nrows) break;
      const int r = r0 + j;
      if (lane == 0) e.lse_part[(size_t)r * e.nblk + n0 / BM] = make_float2(M[k], Ssum[k]);
      const int tg = iv[j] - n0;
      if (tg >= 0 && tg < BM && (tg & 31) == lane) e.lse_tgt[r] = S[j * BM + tg];
    }
  } else if (e.mode == EPI_SWIGLU) {
#pragma unroll 4
    for (int idx = tid; idx < nrows * (BM / 2); idx += 128) {
      const int j = idx / (BM / 2), jj = idx % (BM / 2);
      const float g = S[j * BM + jj], u = S[j * BM + BM / 2 + jj];
      ((__nv_bfloat16*)e.u_out)[(size_t)(r0 + j) * e.F + (n0 / BM) * (BM / 2) + jj] =
          __float2bfloat16_rn(swiglu(g, u));
    }
  }
}

// Epilogue warps 0..7 of both GEMM kernels: warp w reads TMEM lanes
// 32*(w%4) .. +31 (features n0 + 32*(w%4) ..), group w/4 takes the tile's
// 16-column chunks 2k + w/4.  PAIR: this CTA holds rows 128*rank .. of a CTA
// pair's M = 256 accumulator (features n0 + 128*rank ..), and each warp
// signals the end of a tile on the leader CTA's barrier.
struct EpiCtx {
  float* stile;
  long long* meta_off;
  int* meta_iv;
  int* s_go;
  uint64_t* tfull;
  uint64_t* tempty;      // one CTA: this CTA's tile-empty barriers
  uint32_t tempty_lead;  // pair: cluster address of the leader's tile-empty barriers
  uint32_t tmem;
  volatile int* abort_flag;
};
template <bool PAIR>
__device__ __forceinline__ void epilogue_warps(const TcArgs& a, const EpiCtx& c, int ntn, int splits, int R,
                                               int kblocks, int items, int first, int stride, uint32_t rank,
                                               int ng) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = warp >> 2, qw = warp & 3, gt = threadIdx.x & 127;
  float* sg = c.stile + g * EPI_ROWS * BM;
  int acc = 0, ipar = 0;
  uint32_t aphase = 0;
  const bool direct = a.fused != 0;  // fused launches never split
  for (int it = first; it < items; it += stride, ipar ^= 1) {
    const Item t = decode_item(it, ntn, splits, R, kblocks, PAIR ? 2 * BM : BM);
    const int n0 = t.n0 + (int)rank * BM;  // this CTA's 128 features
    long long* moff = c.meta_off + ipar * BNMAX;
    int* miv = c.meta_iv + ipar * BNMAX;
    // the tile's per-row data first (the previous tile's copy is the other
    // buffer: every thread passed this tile's predecessor's barrier, so
    // none still reads the buffer written here)
    if (direct) load_row_meta(a.epi, n0, t.r0, t.rows, moff, miv, ng * 128);
    // one thread waits, the named barrier releases all epilogue warps
    // together, so an expired wait makes them all leave at the same point
    if (threadIdx.x == 0) c.s_go[ipar] = mbar_wait(c.tfull + acc, aphase, c.abort_flag) ? 1 : 0;
    epi_bar(ng);
    if (!c.s_go[ipar]) break;
    tc_fence_after();
    const int n = n0 + qw * 32 + lane;
    const uint32_t tbase = c.tmem + ((uint32_t)(qw * 32) << 16) + (uint32_t)(acc * BNMAX);
    float* Ys = a.Y + (size_t)t.split * a.split_stride;
    for (int c0 = g * EPI_ROWS; c0 < t.nbox * BOXN; c0 += ng * EPI_ROWS) {
      uint32_t v[EPI_ROWS];
      tmem_ld16(tbase + (uint32_t)c0, v);
      const int nr = min(EPI_ROWS, R - (t.r0 + c0));  // may be <= 0 in a ragged last chunk
      if (direct && a.epi.mode == EPI_RESID) {
        // h[row][n] += y straight from the accumulator: for each row the
        // warp's 32 features are 128 contiguous bytes; all loads first
        float hv[EPI_ROWS];
#pragma unroll
        for (int j = 0; j < EPI_ROWS; ++j) hv[j] = j < nr ? a.epi.rs.h[moff[c0 + j] + n] : 0.f;
#pragma unroll
        for (int j = 0; j < EPI_ROWS; ++j)
          if (j < nr) a.epi.rs.h[moff[c0 + j] + n] = hv[j] + __uint_as_float(v[j]);
      } else if (direct && a.epi.mode == EPI_QKV) {
        // the rotary table loads go out before the staging barrier
        float2 cs[QKV_RPT];
        qkv_load_rope(a.epi, n0, nr, miv + c0, gt, cs);
#pragma unroll
        for (int j = 0; j < EPI_ROWS; ++j) sg[j * BM + qw * 32 + lane] = __uint_as_float(v[j]);
        grp_bar(g);
        qkv_store(a.epi, sg, n0, nr, moff + c0, gt, cs);
        grp_bar(g);
      } else if (direct) {
        // stage [16 rows][128 features], then the layer epilogue
#pragma unroll
        for (int j = 0; j < EPI_ROWS; ++j) sg[j * BM + qw * 32 + lane] = __uint_as_float(v[j]);
        grp_bar(g);
        tile_epilogue(a.epi, sg, n0, t.r0 + c0, nr, moff + c0, miv + c0, gt, g);
        grp_bar(g);
      } else {
#pragma unroll
        for (int j = 0; j < EPI_ROWS; ++j) {
          const int r = t.r0 + c0 + j;
          if (r < R) Ys[(size_t)r * a.N + n] = __uint_as_float(v[j]);
        }
      }
    }
    tc_fence_before();
    if (PAIR) {
      // one arrival per warp on the leader CTA's barrier
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(c.tempty_lead + 8u * (uint32_t)acc);
    } else {
      mbar_arrive(c.tempty + acc);
    }
    acc ^= 1;
    if (acc == 0) aphase ^= 1u;
  }
}

__global__ void __launch_bounds__(THREADS, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tw, const __grid_constant__ CUtensorMap tx, TcArgs a) {
  const int ng = ((int)blockDim.x - 64) >> 7;  // epilogue groups: 1 or 2
  const int warp_tma = 4 * ng, warp_mma = 4 * ng + 1;
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_go[2];
  const int ntn = a.N / BM, kblocks = a.K / BK;
  // Before waiting for the previous kernel: nothing here reads what it
  // writes.  Pull the weight tiles this CTA will stream when all rows fit
  // one tile (the decode case), and the next GEMM's share, into L2.
  if (threadIdx.x == warp_mma * 32) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tw)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tx)) : "memory");
    const int s1 = tc_split_count(1, a.N, a.K, gridDim.x, a.max_split);
    if ((int)blockIdx.x < ntn * s1) {
      const Item t = decode_item(blockIdx.x, ntn, s1, 1, kblocks);
      for (int kb = t.kb0; kb < t.kb1; ++kb)
        asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                         reinterpret_cast<uint64_t>(&tw)),
                     "r"(kb * BK), "r"(t.n0)
                     : "memory");
    }
    if (a.pf_ptr && a.pf_bytes) {
      const unsigned long long share = ((a.pf_bytes / gridDim.x) + 15ull) & ~15ull;
      const unsigned long long beg = share * blockIdx.x;
      for (unsigned long long o = beg; o < beg + share && o < a.pf_bytes; o += 65536ull) {
        unsigned long long n = beg + share - o;
        if (n > 65536ull) n = 65536ull;
        if (o + n > a.pf_bytes) n = a.pf_bytes - o;
        n &= ~15ull;
        if (n)
          asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.pf_ptr + o), "r"((uint32_t)n) : "memory");
      }
    }
  }
  pdl_wait();
  pdl_launch();
  const int R = *a.nrows;
  if (R <= 0 || (a.skip_if_zero && *a.skip_if_zero == 0)) return;
  const int nrt = (R + BNMAX - 1) / BNMAX;
  const int splits = tc_split_count(R, a.N, a.K, gridDim.x, a.max_split);
  const int items = ntn * nrt * splits;
  if ((int)blockIdx.x >= items) return;

  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  // Stage ring sized to the row tile this launch needs: a stage is one W tile
  // (16 KB) plus nbmax X boxes (4 KB each); small row counts (decode) get up
  // to MAXST stages in flight.
  const int nbmax = (min(R, BNMAX) + BOXN - 1) / BOXN;
  const int stage_bytes = A_BYTES + nbmax * BOX_BYTES;
  const int nst = min(MAXST, SMEM_TILES / stage_bytes);
  uint64_t* full = (uint64_t*)(smem + SMEM_TILES);
  uint64_t* empty = full + MAXST;
  uint64_t* tfull = empty + MAXST;
  uint64_t* tempty = tfull + 2;
  float* stile = (float*)(smem + SMEM_TILES + 512);  // epilogue staging [2 groups][EPI_ROWS][BM]
  long long* meta_off = (long long*)(smem + SMEM_TILES + 512 + EPI_BYTES);  // [2][BNMAX]
  int* meta_iv = (int*)(meta_off + 2 * BNMAX);                              // [2][BNMAX]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < nst; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(tfull + s, 1);
      mbar_init(tempty + s, ng * 128);
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

  if (warp == warp_tma) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int issued[MAXST];  // parity of the last load issued into each stage, -1 if none
#pragma unroll
      for (int s = 0; s < MAXST; ++s) issued[s] = -1;
      for (int it = blockIdx.x; it < items && ok; it += gridDim.x) {
        const Item t = decode_item(it, ntn, splits, R, kblocks);
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          if (!mbar_wait(empty + stage, phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          issued[stage] = (int)phase;
          unsigned char* sa = smem + stage * stage_bytes;
          mbar_expect_tx(full + stage, (uint32_t)(A_BYTES + t.nbox * BOX_BYTES));
          tma_load_2d(sa, &tw, full + stage, kb * BK, t.n0);
          for (int j = 0; j < t.nbox; ++j)
            tma_load_2d(sa + A_BYTES + j * BOX_BYTES, &tx, full + stage, kb * BK, t.r0 + j * BOXN);
          if (++stage == nst) {
            stage = 0;
            phase ^= 1u;
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
  } else if (warp == warp_mma) {
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
          const uint64_t ad = sw128_desc(smem_u32(smem + stage * stage_bytes));
          const uint64_t bd = sw128_desc(smem_u32(smem + stage * stage_bytes + A_BYTES));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma(d, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc, (kb > t.kb0 || kk > 0) ? 1u : 0u);
          umma_commit(empty + stage);
          if (++stage == nst) {
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
    EpiCtx c{stile, meta_off, meta_iv, s_go, tfull, tempty, 0u, tmem, abort_flag};
    epilogue_warps<false>(a, c, ntn, splits, R, kblocks, items, blockIdx.x, gridDim.x, 0u, ng);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
  if (threadIdx.x == 0 && s_abort) dev_fail(a.status, DEV_ERR_TIMEOUT);
}

// ---------------------------------------------------------------------------
// CTA-pair GEMM (prefill and scoring: many rows, one K slice).  A cluster of
// two CTAs computes a 256-feature x 256-row tile with tcgen05.mma
// cta_group::2 (M = 256): each CTA stages its own 128 weight rows and 128 of
// the tile's X rows, so a CTA moves 32 KB of operands per 64-deep K step
// instead of 48 KB, and holds its 128 features x 256 rows of the accumulator
// in its own TMEM.  The leader CTA (rank 0) issues the MMAs; both CTAs' TMA
// loads count on the leader's stage barrier, and the leader's commits
// arrive on the stage and tile barriers of both CTAs.  Epilogue as in the
// one-CTA kernel, on this CTA's 128 features.
// ---------------------------------------------------------------------------
constexpr int PAIR_ROWS = BNMAX / 2;  // X rows a CTA stages per tile
constexpr int PAIR_STAGE = A_BYTES + (PAIR_ROWS / BOXN) * BOX_BYTES;
constexpr int PAIR_NST = SMEM_TILES / PAIR_STAGE;
static_assert(PAIR_NST <= MAXST, "pair stages fit the barrier array");

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    k_gemm_tc2(const __grid_constant__ CUtensorMap tw, const __grid_constant__ CUtensorMap tx, TcArgs a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_go[2];
  const int ntn2 = a.N / (2 * BM), kblocks = a.K / BK;
  const uint32_t rank = cluster_ctarank();
  if (threadIdx.x == WARP_MMA * 32) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tw)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tx)) : "memory");
  }
  pdl_wait();
  pdl_launch();
  // both CTAs of a pair read the same values, so they leave together
  const int R = *a.nrows;
  if (R <= 0 || (a.skip_if_zero && *a.skip_if_zero == 0)) return;
  const int items = ntn2 * ((R + BNMAX - 1) / BNMAX);
  const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);
  if (pair >= items) return;

  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(smem + SMEM_TILES);
  uint64_t* empty = full + MAXST;
  uint64_t* tfull = empty + MAXST;
  uint64_t* tempty = tfull + 2;
  float* stile = (float*)(smem + SMEM_TILES + 512);
  long long* meta_off = (long long*)(smem + SMEM_TILES + 512 + EPI_BYTES);
  int* meta_iv = (int*)(meta_off + 2 * BNMAX);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < PAIR_NST; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(tfull + s, 1);
      mbar_init(tempty + s, 2 * EPI_WARPS);  // the leader's: one arrival per epilogue warp of both CTAs
    }
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers are initialised before either uses the other's
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;

  if (warp == WARP_TMA) {
    if (lane == 0) {
      const uint32_t full_lead = mapa_shared(smem_u32(full), 0);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int issued[MAXST];  // leader: parity of the last phase it armed in each stage, -1 if none
#pragma unroll
      for (int s = 0; s < MAXST; ++s) issued[s] = -1;
      for (int it = pair; it < items && ok; it += npairs) {
        const Item t = decode_item(it, ntn2, 1, R, kblocks, 2 * BM);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(empty + stage, phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          unsigned char* sa = smem + stage * PAIR_STAGE;
          if (rank == 0) {
            issued[stage] = (int)phase;
            mbar_expect_tx(full + stage, (uint32_t)(2 * PAIR_STAGE));  // both CTAs' bytes
          }
          const uint32_t fb = full_lead + 8u * (uint32_t)stage;
          tma_load_2d_pair(sa, &tw, fb, kb * BK, t.n0 + (int)rank * BM);
          for (int j = 0; j < PAIR_ROWS / BOXN; ++j)
            tma_load_2d_pair(sa + A_BYTES + j * BOX_BYTES, &tx, fb, kb * BK, t.r0 + (int)rank * PAIR_ROWS + j * BOXN);
          if (++stage == PAIR_NST) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag && rank == 0) {
        // let the copies already issued land before the pair leaves (bounded;
        // the leader's stage barriers count both CTAs' bytes)
        volatile int never = 0;
        for (int s = 0; s < PAIR_NST; ++s)
          if (issued[s] >= 0) mbar_wait(full + s, (uint32_t)issued[s], &never, WAIT_NS / 4);
      }
    }
  } else if (warp == WARP_MMA) {
    if (lane == 0 && rank == 0) {
      const uint32_t empty_own = mapa_shared(smem_u32(empty), 0), empty_peer = mapa_shared(smem_u32(empty), 1);
      const uint32_t tfull_own = mapa_shared(smem_u32(tfull), 0), tfull_peer = mapa_shared(smem_u32(tfull), 1);
      const uint32_t idesc = idesc_bf16_m256(BNMAX);
      int stage = 0, acc = 0;
      uint32_t phase = 0, aphase = 0;
      bool ok = true;
      for (int it = pair; it < items && ok; it += npairs) {
        if (!mbar_wait(tempty + acc, aphase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * BNMAX);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(full + stage, phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_desc(smem_u32(smem + stage * PAIR_STAGE));
          const uint64_t bd = sw128_desc(smem_u32(smem + stage * PAIR_STAGE + A_BYTES));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_pair(d, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit_pair(empty_own + 8u * (uint32_t)stage);
          umma_commit_pair(empty_peer + 8u * (uint32_t)stage);
          if (++stage == PAIR_NST) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(tfull_own + 8u * (uint32_t)acc);
        umma_commit_pair(tfull_peer + 8u * (uint32_t)acc);
        acc ^= 1;
        if (acc == 0) aphase ^= 1u;
      }
    }
  } else {
    EpiCtx c{stile, meta_off, meta_iv, s_go, tfull, tempty, mapa_shared(smem_u32(tempty), 0), tmem, abort_flag};
    epilogue_warps<true>(a, c, ntn2, 1, R, kblocks, items, pair, npairs, rank, 2);
  }
  __syncthreads();
  tc_fence_before();
  cluster_sync();  // neither CTA leaves while the other may still signal its barriers or read its tiles
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
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

// CTA-pair kernel for launches with many rows and one K slice, unless
// NVIUM_GEMM_PAIR=0 keeps every launch on the one-CTA kernel
static bool pair_gemm_enabled() {
  static const bool on = [] {
    const char* ev = std::getenv("NVIUM_GEMM_PAIR");
    return !(ev && ev[0] == '0');
  }();
  return on;
}
constexpr int PAIR_MIN_ROWS = 1024;

nv_status tc_prepare() {
  cudaError_t e = cudaFuncSetAttribute(k_gemm_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_gemm_tc2, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
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

nv_status encode_rows128_map(const void* base, uint64_t rows, uint32_t box_rows, CUtensorMap* out) {
  auto enc = get_encode();
  if (!enc) {
    set_error("cuTensorMapEncodeTiled is unavailable");
    return NV_ERR_UNSUPPORTED;
  }
  if (((uintptr_t)base & 15) || rows == 0 || box_rows == 0 || box_rows > 256) {
    set_error("row tensor map: bad base or box");
    return NV_ERR_INVALID_ARG;
  }
  cuuint64_t dims[2] = {64, rows};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled (rows of 128 bytes) failed with code " + std::to_string((int)r));
    return NV_ERR_CUDA;
  }
  return NV_OK;
}

size_t tc_split_stride(size_t N) { return (size_t)BNMAX * N; }

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

nv_status tc_map(TcPlanCache* c, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld_elems,
                 uint32_t box_rows, CUtensorMap* out) {
  return make_map(c, ptr, inner, outer, ld_elems, box_rows, out);
}

int tc_sm_count() { return sm_count(); }

nv_status tc_gemm_run(TcPlanCache* c, const void* X, int ldx, const void* W, int N, int K, const int* nrows,
                      int max_rows, float* Y, bool allow_split, const EpiArgs* epi, int* tile_counters,
                      const void* prefetch, size_t prefetch_bytes, cudaStream_t st, int* grid_out,
                      const int* skip_if_zero) {
  if (N % BM || K % BK || K > ldx) {
    set_error("tcgen05 GEMM needs N % 128 == 0 and K % 64 == 0 (N=" + std::to_string(N) + ", K=" +
              std::to_string(K) + ")");
    return NV_ERR_UNSUPPORTED;
  }
  if (epi && epi->mode != EPI_STORE) {
    if (allow_split) {
      set_error("fused tcgen05 epilogue needs one K slice");
      return NV_ERR_UNSUPPORTED;
    }
    const bool ok = epi->mode == EPI_RESID || epi->mode == EPI_HEAD || epi->mode == EPI_LSE ||
                    (epi->mode == EPI_QKV && BM % epi->hd == 0 && (epi->H * epi->hd) % BM == 0) ||
                    (epi->mode == EPI_SWIGLU && epi->G == BM / 2);
    if (!ok) {
      set_error("fused tcgen05 epilogue: unsupported tile layout");
      return NV_ERR_UNSUPPORTED;
    }
  }
  CUtensorMap tw, tx;
  NV_TRY(make_map(c, W, (uint64_t)K, (uint64_t)N, (uint64_t)K, BM, &tw));
  NV_TRY(make_map(c, X, (uint64_t)K, (uint64_t)max_rows, (uint64_t)ldx, BOXN, &tx));
  if (!allow_split && N % (2 * BM) == 0 && max_rows >= PAIR_MIN_ROWS && pair_gemm_enabled() &&
      !(epi && epi->mode == EPI_HEAD)) {
    // CTA pairs: an even grid of at most one pair per 256 x 256 tile
    const long long tiles = (long long)(N / (2 * BM)) * ((max_rows + BNMAX - 1) / BNMAX);
    int grid = sm_count() & ~1;
    if (2 * tiles < grid) grid = (int)(2 * tiles);
    TcArgs a;
    a.nrows = nrows;
    a.Y = Y;
    a.N = N;
    a.K = K;
    a.max_split = 1;
    a.split_stride = (size_t)BNMAX * N;
    a.status = c->status;
    a.fused = (epi && epi->mode != EPI_STORE) ? 1 : 0;
    a.skip_if_zero = skip_if_zero;
    a.pf_ptr = nullptr;
    a.pf_bytes = 0;
    if (epi) a.epi = *epi;
    else std::memset(&a.epi, 0, sizeof(a.epi));
    cudaError_t le = launch_k(k_gemm_tc2, dim3(grid), dim3(THREADS), SMEM_BYTES, st, tw, tx, a);
    if (le != cudaSuccess) {
      set_error(std::string("tcgen05 pair GEMM launch: ") + cudaGetErrorString(le));
      return NV_ERR_CUDA;
    }
    if (grid_out) *grid_out = grid;
    return NV_OK;
  }
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
  a.fused = (epi && epi->mode != EPI_STORE) ? 1 : 0;
  a.skip_if_zero = skip_if_zero;
  a.pf_ptr = (const unsigned char*)prefetch;
  a.pf_bytes = ((uintptr_t)prefetch & 15) ? 0ull : (unsigned long long)prefetch_bytes;
  if (epi) a.epi = *epi;
  else std::memset(&a.epi, 0, sizeof(a.epi));
  cudaError_t le = launch_k(k_gemm_tc, dim3(grid), dim3(allow_split ? THREADS_1G : THREADS), SMEM_BYTES, st, tw, tx, a);
  if (le != cudaSuccess) {
    set_error(std::string("tcgen05 GEMM launch: ") + cudaGetErrorString(le));
    return NV_ERR_CUDA;
  }
  if (grid_out) *grid_out = grid;
  return NV_OK;
}

}  // namespace nv
