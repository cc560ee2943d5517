// Causal attention for prefill and scoring on the 5th-generation tensor
// cores (tcgen05, accumulators in TMEM), bf16 caches with head_dim 64.
//
// What it computes is the causal softmax attention of the LLaMA-2 backbone
// ("N-vium: Mixture-of-Exits Transformer for Accelerated Exact Generation",
// section 4): a row at position p gets o = sum_j softmax_j(q . k_j / sqrt(hd))
// v_j over the keys j <= p of its sequence.
//
// CTA (128-row query tile, head, sequence); two CTAs per SM.  Roles:
//   warps 0-3  one query row per thread (= its TMEM lane): read the row's
//              64 scores of a key tile from TMEM, causal mask, online softmax
//              (running max and sum), write P to shared memory as a bf16
//              pair hi + lo (hi = bf16(P), lo = bf16(P - hi), ~16 significant
//              bits), and fold each tile's P V into a register accumulator
//              with the softmax correction factor;
//   warp 4     TMA: the query tile once, then 64-key tiles of K and V
//              through a 3-stage ring (128-byte swizzle);
//   warp 5     issues the MMAs: S = Q K^T (M 128, N 64, K 16 x 4) into one
//              of two TMEM score buffers, one tile ahead of the softmax, and
//              O_tile = P_hi V + P_lo V (V read in place as an MN-major
//              operand) into one of two TMEM output buffers.
// The softmax of tile j+1 overlaps the P V product of tile j.  Every wait is
// bounded (2 s); on expiry the CTA records DEV_ERR_TIMEOUT, lets its copies
// and MMAs land and frees its TMEM.
#include <math_constants.h>

#include "kernels.cuh"
#include "tc_prims.cuh"

namespace nv {
namespace {
using namespace tc;

constexpr int HD = 64;
constexpr int TQ = 128;   // query rows per CTA (MMA M, TMEM lanes)
constexpr int TK = 64;    // keys per tile (MMA N of S, K of P V)
constexpr int KST = 3;    // K/V ring stages
constexpr int FT_THREADS = 192;
constexpr uint32_t FT_TMEM_COLS = 256;  // S[2] at columns 0 and 64, O at 128
constexpr int TILE_BYTES = TK * HD * 2;  // 8 KB

struct FtSmem {
  __nv_bfloat16 Q[TQ * HD];        // 16 KB, 1024-byte aligned (128-byte swizzle atoms)
  __nv_bfloat16 K[KST][TK * HD];   // 8 KB each
  __nv_bfloat16 V[KST][TK * HD];
  __nv_bfloat16 Phi[TQ * TK];      // 16 KB
  __nv_bfloat16 Plo[TQ * TK];
  uint64_t q_full, kv_full[KST], kv_empty[KST], s_full[2], s_empty[2], p_full, o_full, drain;
  uint32_t tmem;
  int abort;
};
constexpr size_t FT_SMEM_BYTES = sizeof(FtSmem) + 1024;

__device__ __forceinline__ void tma_row_box(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int row) {
  tma_load_2d(dst, map, bar, x, row);
}
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}
// 2^x by the hardware approximation (PTX ex2.approx.ftz.f32, relative error
// about 2^-22): the softmax runs in base 2 with the scores pre-scaled by
// log2(e), so exp(s - m) = 2^(s log2 e - m log2 e)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
// packed pairs of fp32 (sm_100 f32x2 instructions: each lane of the pair is
// an ordinary IEEE fp32 operation, rounded to nearest)
__device__ __forceinline__ uint64_t as_u64(float2 v) { return *reinterpret_cast<const uint64_t*>(&v); }
__device__ __forceinline__ float2 as_f2(uint64_t v) { return *reinterpret_cast<const float2*>(&v); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(as_u64(a)), "l"(as_u64(b)), "l"(as_u64(c)));
  return as_f2(r);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(as_u64(a)), "l"(as_u64(b)));
  return as_f2(r);
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(as_u64(a)), "l"(as_u64(b)));
  return as_f2(r);
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// Each softmax warp waits on its own: lane 0 polls (bounded), the warp
// follows.  No barrier across the four warps, so a warp starts on a tile as
// soon as the tile is ready, not when the slowest warp has finished the last.
__device__ __forceinline__ bool sm_wait(FtSmem& S, uint64_t* bar, uint32_t parity) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, &S.abort) ? 1 : 0;
  __syncwarp();
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__global__ void __launch_bounds__(FT_THREADS, 2)
    k_attn_fa_tc(const __grid_constant__ CUtensorMap kvmap, const __grid_constant__ CUtensorMap qmap, AttnArgs a) {
  pdl_wait();
  pdl_launch();
  extern __shared__ unsigned char smem_raw[];
  FtSmem& S = *reinterpret_cast<FtSmem*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  if (*a.rs.nrows == 0) return;
  // grid (row tile, head, sequence), the latest row tiles (the most keys) first
  const int b = blockIdx.z, head = blockIdx.y;
  const int s0 = a.rs.seq_start[b], s1 = a.rs.seq_start[b + 1];
  const int nrt = (s1 - s0 + TQ - 1) / TQ;
  const int rt = nrt - 1 - (int)blockIdx.x;
  if (rt < 0) return;
  const int g0 = s0 + rt * TQ, g1 = min(s1, g0 + TQ), nr = g1 - g0;
  const int pos_last = a.rs.row_pos[g1 - 1];
  const int ntk = pos_last / TK + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&S.q_full, 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(&S.kv_full[s], 1);
      mbar_init(&S.kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&S.s_full[s], 1);
      mbar_init(&S.s_empty[s], 128);
    }
    mbar_init(&S.o_full, 1);
    mbar_init(&S.p_full, 128);
    mbar_init(&S.drain, 1);
    S.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&S.tmem)),
                 "r"(FT_TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem;
  volatile int* abort_flag = &S.abort;

  if (warp == 4) {
    // the whole warp walks the key tiles: lanes hold the page ids of the next
    // 32 pages (loaded ahead, off the per-tile path), lane 0 waits and issues
    const int ps = a.kv.page_size;
    const size_t hstride = (size_t)ps * HD, lbase = (size_t)a.layer * a.kv.layer_stride;
    const int* pt = a.kv.page_table + (size_t)b * a.kv.pages_per_seq;
    const int plast = pos_last / ps;
    int chunk = -1, pg = 0;
    bool ok = true;
    int issued[KST];
    for (int s = 0; s < KST; ++s) issued[s] = -1;
    if (lane == 0) {
      mbar_expect_tx(&S.q_full, (uint32_t)(TQ * HD * 2));
      tma_row_box(S.Q, &qmap, &S.q_full, head * HD, g0);
    }
    for (int j = 0; j < ntk && ok; ++j) {
      const int st = j % KST;
      const uint32_t ph = (uint32_t)((j / KST) & 1);
      const int pos = j * TK, pi = pos / ps;
      if (pi >= chunk + 32 || chunk < 0) {
        chunk = pi;
        pg = chunk + lane <= plast ? pt[chunk + lane] : 0;
      }
      const int page = __shfl_sync(0xffffffffu, pg, pi - chunk);
      int go = 1;
      if (lane == 0) {
        if (!mbar_wait(&S.kv_empty[st], ph ^ 1u, abort_flag)) {
          go = 0;
        } else {
          issued[st] = (int)ph;
          mbar_expect_tx(&S.kv_full[st], (uint32_t)(2 * TILE_BYTES));
          const size_t off = lbase + ((size_t)page * 2 * a.H + head) * hstride + (size_t)(pos % ps) * HD;
          tma_row_box(S.K[st], &kvmap, &S.kv_full[st], 0, (int)(off / HD));
          tma_row_box(S.V[st], &kvmap, &S.kv_full[st], 0, (int)((off + (size_t)a.H * hstride) / HD));
        }
      }
      ok = __shfl_sync(0xffffffffu, go, 0) != 0;
    }
    if (lane == 0) {
      if (*abort_flag) {
        volatile int never = 0;
        mbar_wait(&S.q_full, 0, &never, WAIT_NS / 4);
        for (int s = 0; s < KST; ++s)
          if (issued[s] >= 0) mbar_wait(&S.kv_full[s], (uint32_t)issued[s], &never, WAIT_NS / 4);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      bool ok = mbar_wait(&S.q_full, 0, abort_flag), issued_any = false;
      const uint32_t idesc_s = idesc_bf16(TK);                  // M 128, N 64, K-major A and B
      const uint32_t idesc_o = idesc_bf16(HD) | (1u << 16);     // B (V) MN-major
      const uint64_t qd = sw128_desc(smem_u32(S.Q));
      auto issue_s = [&](int j) -> bool {
        const int st = j % KST;
        if (!mbar_wait(&S.kv_full[st], (uint32_t)((j / KST) & 1), abort_flag)) return false;
        if (!mbar_wait(&S.s_empty[j & 1], (uint32_t)(((j >> 1) & 1) ^ 1), abort_flag)) return false;
        tc_fence_after();
        const uint64_t kd = sw128_desc(smem_u32(S.K[st]));
        const uint32_t d = tmem + (uint32_t)((j & 1) * TK);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) umma(d, qd + (uint64_t)(2 * kk), kd + (uint64_t)(2 * kk), idesc_s, kk > 0);
        issued_any = true;
        umma_commit(&S.s_full[j & 1]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < ntk && ok; ++j) {
        if (j + 1 < ntk && !issue_s(j + 1)) {
          ok = false;
          break;
        }
        // P of tile j is in shared memory and O has been rescaled for it
        if (!mbar_wait(&S.p_full, (uint32_t)(j & 1), abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int st = j % KST;
        const uint64_t ph = sw128_desc(smem_u32(S.Phi)), pl = sw128_desc(smem_u32(S.Plo));
        const uint64_t vd = sw128_desc(smem_u32(S.V[st]));
        const uint32_t d = tmem + (uint32_t)(2 * TK);
#pragma unroll
        for (int kk = 0; kk < TK / 16; ++kk) {
          // K step of 16 keys: 32 bytes along a P row, 16 rows (2048 bytes) of V
          umma(d, ph + (uint64_t)(2 * kk), vd + (uint64_t)(128 * kk), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
          umma(d, pl + (uint64_t)(2 * kk), vd + (uint64_t)(128 * kk), idesc_o, 1u);
        }
        umma_commit(&S.o_full);
        umma_commit(&S.kv_empty[st]);
      }
      if (!ok && issued_any) {
        umma_commit(&S.drain);
        volatile int never = 0;
        mbar_wait(&S.drain, 0, &never, WAIT_NS / 4);
      }
    }
  } else {
    // softmax warps: thread t owns query row t of the tile (TMEM lane t)
    const int t = threadIdx.x;
    const int pos = t < nr ? a.rs.row_pos[g0 + t] : -1;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    float mref = -CUDART_INF_F, l = 0.f;
    const float scale2 = a.scale * 1.4426950408889634f;  // log2(e) / sqrt(hd)
    unsigned char* prow_hi = reinterpret_cast<unsigned char*>(S.Phi) + t * 128;
    unsigned char* prow_lo = reinterpret_cast<unsigned char*>(S.Plo) + t * 128;
    const uint32_t o_addr = lane_base + (uint32_t)(2 * TK);
    bool ok = true;
    for (int j = 0; j < ntk; ++j) {
      if (!sm_wait(S, &S.s_full[j & 1], (uint32_t)((j >> 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // the row's 64 scores of this key tile, turned into P in place
      uint32_t r[TK];
      const uint32_t sa = lane_base + (uint32_t)((j & 1) * TK);
      tmem_ld32_nowait(sa, *reinterpret_cast<uint32_t(*)[32]>(r));
      tmem_ld32_nowait(sa + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&S.s_empty[j & 1]);
      const int k0 = j * TK;
      // raw scores; keys past the row's position (only in the tiles that
      // reach the diagonal) get -inf
      if (k0 + TK - 1 > pos) {
#pragma unroll
        for (int i = 0; i < TK; ++i)
          if (k0 + i > pos) r[i] = __float_as_uint(-CUDART_INF_F);
      }
      // the row max as eight independent chains, then a tree (a single
      // 64-long dependent chain would leave the pipe waiting on itself)
      float pm[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) pm[c] = __uint_as_float(r[c]);
#pragma unroll
      for (int i = 8; i < TK; ++i) pm[i & 7] = fmaxf(pm[i & 7], __uint_as_float(r[i]));
      const float tmax = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                               fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
      // Softmax in base 2 against a reference max mref (scores scaled by
      // log2(e) / sqrt(hd)): P = 2^(s scale2 - mref).  mref moves only when a
      // score exceeds it by more than 8, so P <= 256 and O is rescaled in TMEM
      // only then, not at every growth of the running max; numerator and
      // denominator share the reference, so O / l is unchanged.
      const float tm2 = tmax * scale2;
      float cj = 1.f;
      bool resc = false;
      if (tm2 > mref + 8.f) {
        if (mref != -CUDART_INF_F) {
          cj = ex2(mref - tm2);
          resc = true;
        }
        mref = tm2;
      }
      float rs = 0.f;
      if (mref == -CUDART_INF_F) {
#pragma unroll
        for (int i = 0; i < TK; ++i) r[i] = 0u;
      } else {
        // the row sum as eight partial sums (element i into sum i % 8, as
        // pairs) added in a fixed tree
        const float2 sc2 = make_float2(scale2, scale2), nm2 = make_float2(-mref, -mref);
        float2 ps[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) ps[c] = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < TK / 2; ++e) {
          const float2 y = fma2(make_float2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1])), sc2, nm2);
          const float2 p = make_float2(ex2(y.x), ex2(y.y));
          r[2 * e] = __float_as_uint(p.x);
          r[2 * e + 1] = __float_as_uint(p.y);
          ps[e & 3] = add2(ps[e & 3], p);
        }
        rs = ((ps[0].x + ps[0].y) + (ps[1].x + ps[1].y)) + ((ps[2].x + ps[2].y) + (ps[3].x + ps[3].y));
      }
      l = l * cj + rs;
      // P as bf16 pairs, hi = bf16(P) and lo = bf16(P - hi), packed
      // (pk[0..31]: hi, pk[32..63]: lo) before waiting for the previous P V
      uint32_t pk[TK];
#pragma unroll
      for (int e = 0; e < TK / 2; ++e) {
        const float x0 = __uint_as_float(r[2 * e]), x1 = __uint_as_float(r[2 * e + 1]);
        const __nv_bfloat162 hb = __floats2bfloat162_rn(x0, x1);
        pk[e] = *reinterpret_cast<const uint32_t*>(&hb);
        const float2 lo = sub2(make_float2(x0, x1), make_float2(__low2float(hb), __high2float(hb)));
        pk[TK / 2 + e] = pack2(lo.x, lo.y);
      }
      // the previous tile's P V must be done with P (and with O) first
      if (j > 0 && !sm_wait(S, &S.o_full, (uint32_t)((j - 1) & 1))) {
        ok = false;
        break;
      }
      if (j == ntk - 1 && pos_last + 1 - k0 < TK) {
        // V rows past the last key may hold stale values (P is 0 there, and
        // 0 * NaN would poison the sums): zero them before the P V product
        const int nk = pos_last + 1 - k0;
        unsigned char* vb = reinterpret_cast<unsigned char*>(S.V[j % KST]);
        for (int i = nk * 8 + t; i < TK * 8; i += 128)
          *reinterpret_cast<uint4*>(vb + (i >> 3) * 128 + (i & 7) * 16) = make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int off = ((c ^ (t & 7)) << 4);
        *reinterpret_cast<uint4*>(prow_hi + off) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(prow_lo + off) =
            make_uint4(pk[TK / 2 + 4 * c], pk[TK / 2 + 4 * c + 1], pk[TK / 2 + 4 * c + 2], pk[TK / 2 + 4 * c + 3]);
      }
      // a row whose reference moved: O (the sum over the earlier tiles) is
      // rescaled in TMEM by 2^(mref_old - mref_new) before this tile's P V
      // adds to it.  The TMEM loads and stores are warp-collective: a warp
      // with any such row rescales all its rows, the others by exactly 1.
      if (__any_sync(0xffffffffu, resc)) {
        const float f = resc ? cj : 1.0f;
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t v[32];
          tmem_ld32_nowait(o_addr + 32 * h, v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * f);
          tmem_st32(o_addr + 32 * h, v);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      mbar_arrive(&S.p_full);
    }
    if (ok && !sm_wait(S, &S.o_full, (uint32_t)((ntk - 1) & 1))) ok = false;
    if (ok) {
      tc_fence_after();
      const float inv = 1.0f / l;
      uint4* orow = reinterpret_cast<uint4*>((__nv_bfloat16*)a.o + (size_t)(g0 + t) * a.H * HD + head * HD);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t v[32];
        tmem_ld32_nowait(o_addr + 32 * h, v);
        tmem_wait_ld();
        if (t < nr) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float* o = reinterpret_cast<const float*>(v) + 8 * c;
            orow[4 * h + c] = make_uint4(pack2(o[0] * inv, o[1] * inv), pack2(o[2] * inv, o[3] * inv),
                                         pack2(o[4] * inv, o[5] * inv), pack2(o[6] * inv, o[7] * inv));
          }
        }
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(FT_TMEM_COLS) : "memory");
  }
  if (threadIdx.x == 0) {
    if (S.abort) dev_fail(a.status, DEV_ERR_TIMEOUT);
    else if (a.lens && head == 0 && g1 == s1) a.lens[b * a.L + a.layer] = pos_last + 1;
  }
}

}  // namespace

cudaError_t attn_tc_prepare() {
  return cudaFuncSetAttribute(k_attn_fa_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FT_SMEM_BYTES);
}

void launch_attn_fa_tc(const CUtensorMap* kvmap, const CUtensorMap* qmap, const AttnArgs& a, cudaStream_t st) {
  dim3 grid((a.row_groups * ATTN_RPC + TQ - 1) / TQ, a.H, a.rs.B);
  launch_k(k_attn_fa_tc, grid, FT_THREADS, FT_SMEM_BYTES, st, *kvmap, *qmap, a);
}

}  // namespace nv
