// Attention for bf16 caches with head_dim 64 on warp-level bf16 tensor-core
// MMAs (mma.sync m16n8k16, fp32 accumulation): k_attn_dec_mma for decode and
// flush (few rows per sequence; a CTA streams a sequence's keys for one head,
// or a range of them when splits are needed to fill the GPU) and
// k_attn_fa_mma for prefill and scoring (64-row query tiles streaming 64-key
// tiles with an online softmax, flash-attention style).
//
// What it computes is the causal softmax attention of the LLaMA-2 backbone
// ("N-vium: Mixture-of-Exits Transformer for Accelerated Exact Generation",
// section 4): for a row at position p, o = sum_j softmax_j(q . k_j /
// sqrt(hd)) v_j over keys j <= p.  Rows are the new token of each sequence
// plus the deferred rows that run this layer in the same step (section 2
// "Inferenz: Piggybacking": the layers above an exit run later, batched with
// the next token that reaches them).
//
// Data movement: K and V arrive in 64-position boxes by TMA through a 2-D
// tensor map over the whole KV pool (rows of 64 bf16 = 128 bytes, 128-byte
// swizzle), so the ldmatrix reads of 8 consecutive keys hit 8 different bank
// groups.  Barrier waits are done by one lane (or thread) while the others
// wait at a warp or CTA barrier, spending no issue slots.
//
// Numerics: q and the cache are bf16 (the bf16 contract of the model), S =
// q k^T accumulates in fp32; the softmax weights P are fp32 and enter the PV
// product as a bf16 pair hi + lo (hi = bf16(P), lo = bf16(P - hi)), which
// keeps ~16 significant bits of P; V is exact in bf16.  So the result matches
// an fp32 SIMT evaluation to ~1e-5 relative, far inside the path's tolerance.
#include <math_constants.h>

#include "common.cuh"
#include "kernels.cuh"
#include "mma_prims.cuh"

namespace nv {
namespace {

constexpr int HD = 64;           // head dim (128-byte rows)
constexpr int RG = 16;           // rows per MMA pass
constexpr int QLD = HD + 8;      // padded Q row: 144 bytes, conflict-free ldmatrix
constexpr int OLD = HD + 2;      // per-warp partial row: HD sums, max, weight sum
constexpr int BOX = 64;          // positions per TMA box (a page holds 64 or 128)
constexpr int BOX_BYTES = BOX * HD * 2;

using namespace mp;

constexpr int FQ = 64;   // query rows per CTA
constexpr int FK = 64;   // keys per tile (one box)
constexpr int FST = 3;   // ring stages

struct FaSmem {
  __nv_bfloat16 K[FST][FK * HD];  // 8 KB per stage, 1024-byte aligned
  __nv_bfloat16 V[FST][FK * HD];
  __nv_bfloat16 Q[FQ * QLD];
  uint64_t full[FST];
  int abort;
};
constexpr size_t FA_SMEM_BYTES = sizeof(FaSmem) + 1024;

__device__ __forceinline__ void fa_issue(FaSmem& S, const CUtensorMap* map, const AttnArgs& a, int b, int head,
                                         int tile, int stage) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(&S.full[stage])),
               "r"((uint32_t)(2 * BOX_BYTES))
               : "memory");
  const int pos = tile * FK;
  tma_box(S.K[stage], map, &S.full[stage], (int)(a.kv.offset(a.layer, b, pos, head, 0) / HD));
  tma_box(S.V[stage], map, &S.full[stage], (int)(a.kv.offset(a.layer, b, pos, head, 1) / HD));
}

// bounded wait on a ring stage by every thread; false once 2 s have passed
__device__ __forceinline__ bool fa_wait(uint64_t* bar, uint32_t parity) {
  unsigned long long t0 = 0;
  for (uint32_t i = 0;; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, "
        "p;\n\t}"
        : "=r"(ok)
        : "r"(saddr(bar)), "r"(parity)
        : "memory");
    if (ok) return true;
    if ((i & 63u) == 0u) {
      unsigned long long t;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
      if (i == 0) t0 = t;
      else if (t - t0 > 2000000000ull) return false;
    }
  }
}

// ---------------------------------------------------------------------------
// Decode / flush: CTA (sequence, head, split).  The split owns a contiguous
// range of the sequence's 64-key tiles (all of them when there is one
// split).  Warp 4 streams the range through a DS-stage TMA ring; consumer
// warp w takes tiles w, w+4, ... for the sequence's rows (16 per pass) with
// an online softmax, and the four warps merge once per pass.  One split: the
// CTA writes the normalised output rows; several: unnormalised partials
// (sum, max, weight sum) per (row, head, split), and the last split CTA of
// the (sequence, head) to finish (a per-pair arrival counter) merges them in
// split order, so the result does not depend on which CTA came last.
// ---------------------------------------------------------------------------
constexpr int DS = 4;
constexpr int DEC_THREADS = 160;
struct DecSmem {
  __nv_bfloat16 K[DS][BOX * HD];  // 8 KB per stage, 1024-byte aligned
  __nv_bfloat16 V[DS][BOX * HD];
  __nv_bfloat16 Q[RG * QLD];
  uint64_t full[DS], empty[DS];
  int abort;
};
// the per-pass merge buffer [4 warps][16 rows][HD + 2] reuses the idle ring
static_assert(4 * RG * OLD * 4 <= 2 * DS * BOX * HD * 2, "merge buffer fits in the ring");
constexpr size_t DEC_SMEM_BYTES = sizeof(DecSmem) + 1024;

// lane 0 waits (bounded), the warp follows
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = fa_wait(bar, parity) ? 1 : 0;
  __syncwarp();
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Called by every split CTA of (b, head) after its partials are written; the
// last to arrive merges the splits of each row of b in split order (the same
// order for any arrival order) and writes the normalised output.
__device__ __forceinline__ void dec_merge_splits(const AttnArgs& a, int b, int head, int s0, int s1) {
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    int* c = a.dec_ctr + b * a.H + head;
    const int last = atomicAdd(c, 1) == (int)gridDim.z - 1;
    if (last) *c = 0;  // every split has arrived: ready for the next launch
    s_last = last;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int H = a.H, nsp = gridDim.z, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int r = s0 + (int)(threadIdx.x >> 5); r < s1; r += nw) {
    const float* pp = a.part + ((size_t)r * H + head) * a.kv_splits * OLD;
    float M = -CUDART_INF_F;
    for (int q = 0; q < nsp; ++q) M = fmaxf(M, __ldcg(pp + q * OLD + HD));
    float L = 0.f, acc0 = 0.f, acc1 = 0.f;
    for (int q = 0; q < nsp; ++q) {
      const float mq = __ldcg(pp + q * OLD + HD);
      if (mq == -CUDART_INF_F) continue;
      const float e = expf(mq - M);
      L += __ldcg(pp + q * OLD + HD + 1) * e;
      const float2 v = __ldcg(reinterpret_cast<const float2*>(pp + q * OLD + 2 * lane));
      acc0 += v.x * e;
      acc1 += v.y * e;
    }
    const float inv = 1.0f / L;
    *reinterpret_cast<__nv_bfloat162*>((__nv_bfloat16*)a.o + (size_t)r * H * HD + head * HD + 2 * lane) =
        __floats2bfloat162_rn(acc0 * inv, acc1 * inv);
  }
}

__global__ void __launch_bounds__(DEC_THREADS, 3) k_attn_dec_mma(const __grid_constant__ CUtensorMap kvmap, AttnArgs a) {
  pdl_wait();
  pdl_launch();
  extern __shared__ unsigned char smem_raw[];
  DecSmem& S = *reinterpret_cast<DecSmem*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  if (*a.rs.nrows == 0) return;
  const int b = blockIdx.x, head = blockIdx.y, sp = blockIdx.z, nsp = gridDim.z;
  const int s0 = a.rs.seq_start[b], s1 = a.rs.seq_start[b + 1];
  if (s0 >= s1) return;
  const int pos_last = a.rs.row_pos[s1 - 1];
  const int ntk = pos_last / BOX + 1;
  const int tps = (ntk + nsp - 1) / nsp;
  const int t_beg = min(ntk, sp * tps), t_end = min(ntk, t_beg + tps);
  const int nt = t_end - t_beg;
  const int npass = (s1 - s0 + RG - 1) / RG;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31, g = lane >> 2, tq = lane & 3;
  if (tid == 0) {
    S.abort = 0;
    for (int st = 0; st < DS; ++st) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(saddr(&S.full[st])) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(saddr(&S.empty[st])) : "memory");
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const int H = a.H;
  const __nv_bfloat16* qg = (const __nv_bfloat16*)a.q;
  float(*Ob)[RG][OLD] = reinterpret_cast<float(*)[RG][OLD]>(&S.K[0][0]);
  int q_base = 0;  // ring uses before this pass
  for (int pass = 0; pass < npass; ++pass) {
    const int g0 = s0 + pass * RG, ng = min(RG, s1 - g0);
    float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F, l0 = 0.f, l1 = 0.f;
    float oc[8][4];
#pragma unroll
    for (int nt8 = 0; nt8 < 8; ++nt8)
#pragma unroll
      for (int e = 0; e < 4; ++e) oc[nt8][e] = 0.f;
    if (w == 4) {
      // the whole warp walks the tiles: lanes hold the page ids of the next
      // 32 pages (loaded ahead, off the per-tile path), lane 0 waits and issues
      const int ps = a.kv.page_size;
      const size_t hstride = (size_t)ps * HD, lbase = (size_t)a.layer * a.kv.layer_stride;
      const int* pt = a.kv.page_table + (size_t)b * a.kv.pages_per_seq;
      const int plast = pos_last / ps;
      int chunk = -1, pg = 0;
      for (int i = 0; i < nt; ++i) {
        const int q = q_base + i, st = q % DS;
        const int pos = (t_beg + i) * BOX, pi = pos / ps;
        if (pi >= chunk + 32 || chunk < 0) {
          chunk = pi;
          pg = chunk + lane <= plast ? pt[chunk + lane] : 0;
        }
        const int page = __shfl_sync(0xffffffffu, pg, pi - chunk);
        int ok = 1;
        if (lane == 0) {
          if (q >= DS && !fa_wait(&S.empty[st], (uint32_t)((q / DS - 1) & 1))) {
            S.abort = 1;
            ok = 0;
          } else {
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(&S.full[st])),
                         "r"((uint32_t)(2 * BOX_BYTES))
                         : "memory");
            const size_t off = lbase + ((size_t)page * 2 * a.H + head) * hstride + (size_t)(pos % ps) * HD;
            tma_box(S.K[st], &kvmap, &S.full[st], (int)(off / HD));
            tma_box(S.V[st], &kvmap, &S.full[st], (int)((off + (size_t)a.H * hstride) / HD));
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      }
    } else {
      {  // this pass's query rows (16 rows x 8 chunks: one chunk per consumer thread)
        const int r = tid >> 3, c = tid & 7;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < ng) v = *reinterpret_cast<const uint4*>(qg + (size_t)(g0 + r) * H * HD + head * HD + c * 8);
        *reinterpret_cast<uint4*>(S.Q + r * QLD + c * 8) = v;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      uint32_t qa[4][4];
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        ldsm_x4(qa[ks], saddr(S.Q + ((lane & 7) + 8 * ((lane >> 3) & 1)) * QLD + (2 * ks + (lane >> 4)) * 8));
      const int p0 = g < ng ? a.rs.row_pos[g0 + g] : -1;
      const int p1 = g + 8 < ng ? a.rs.row_pos[g0 + g + 8] : -1;
      for (int i = w; i < nt; i += 4) {
        const int q = q_base + i, st = q % DS;
        if (!warp_wait(&S.full[st], (uint32_t)((q / DS) & 1))) {
          S.abort = 1;
          break;
        }
        const int k0 = (t_beg + i) * BOX;
        if (k0 + BOX > pos_last + 1) {
          // V rows past the last key may be stale or never written: zero them
          // (P is 0 there, and 0 * NaN would poison the sums)
          for (int e = (pos_last + 1 - k0) * 8 + lane; e < BOX * 8; e += 32)
            *reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(S.V[st]) + (e >> 3) * 128 + (e & 7) * 16) =
                make_uint4(0, 0, 0, 0);
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
        }
        const uint32_t kb_ = saddr(S.K[st]), vb_ = saddr(S.V[st]);
        float sc[8][4];
#pragma unroll
        for (int n8 = 0; n8 < 8; ++n8) {
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[n8][e] = 0.f;
          const int r = 8 * n8 + (lane & 7);
#pragma unroll
          for (int kp = 0; kp < 2; ++kp) {
            uint32_t kb[4];
            ldsm_x4(kb, kb_ + swz(r, 4 * kp + (lane >> 3)));
            mma_bf16(sc[n8], qa[2 * kp], kb[0], kb[1]);
            mma_bf16(sc[n8], qa[2 * kp + 1], kb[2], kb[3]);
          }
        }
        float t0 = -CUDART_INF_F, t1 = -CUDART_INF_F;
#pragma unroll
        for (int n8 = 0; n8 < 8; ++n8)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int kk = k0 + 8 * n8 + 2 * tq + (e & 1);
            const bool hi = e >= 2;
            const float v = kk <= (hi ? p1 : p0) ? sc[n8][e] * a.scale : -CUDART_INF_F;
            sc[n8][e] = v;
            if (hi) t1 = fmaxf(t1, v); else t0 = fmaxf(t0, v);
          }
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
          t0 = fmaxf(t0, __shfl_xor_sync(0xffffffffu, t0, o));
          t1 = fmaxf(t1, __shfl_xor_sync(0xffffffffu, t1, o));
        }
        const float n0 = fmaxf(m0, t0), n1 = fmaxf(m1, t1);
        const float c0 = n0 == -CUDART_INF_F ? 1.f : expf(m0 - n0);
        const float c1 = n1 == -CUDART_INF_F ? 1.f : expf(m1 - n1);
        m0 = n0;
        m1 = n1;
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int n8 = 0; n8 < 8; ++n8)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const bool hi = e >= 2;
            const float m = hi ? n1 : n0;
            const float pr = m == -CUDART_INF_F ? 0.f : expf(sc[n8][e] - m);
            sc[n8][e] = pr;
            if (hi) a1 += pr; else a0 += pr;
          }
        l0 = l0 * c0 + a0;  // this thread's columns; the quad is summed at the merge
        l1 = l1 * c1 + a1;
#pragma unroll
        for (int n8 = 0; n8 < 8; ++n8) {
          oc[n8][0] *= c0;
          oc[n8][1] *= c0;
          oc[n8][2] *= c1;
          oc[n8][3] *= c1;
        }
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) {
          uint32_t ph[4], pl[4];
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
              const float x0 = sc[2 * kq + h][2 * rr], x1 = sc[2 * kq + h][2 * rr + 1];
              const __nv_bfloat16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
              ph[2 * h + rr] = pack_bf16(__bfloat162float(h0), __bfloat162float(h1));
              pl[2 * h + rr] = pack_bf16(x0 - __bfloat162float(h0), x1 - __bfloat162float(h1));
            }
          const int r = 16 * kq + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
          for (int np = 0; np < 4; ++np) {
            uint32_t vb[4];
            ldsm_x4_t(vb, vb_ + swz(r, 2 * np + (lane >> 4)));
            mma_bf16(oc[2 * np], ph, vb[0], vb[1]);
            mma_bf16(oc[2 * np], pl, vb[0], vb[1]);
            mma_bf16(oc[2 * np + 1], ph, vb[2], vb[3]);
            mma_bf16(oc[2 * np + 1], pl, vb[2], vb[3]);
          }
        }
        __syncwarp();
        if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(&S.empty[st])) : "memory");
      }
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, o);
        l1 += __shfl_xor_sync(0xffffffffu, l1, o);
      }
    }
    __syncthreads();  // pass end: every issued tile has been consumed, the ring is idle
    if (S.abort) {
      if (tid == 0) {
        dev_fail(a.status, DEV_ERR_TIMEOUT);
        // keep the pair's arrival count consistent for later launches
        if (nsp > 1 && atomicAdd(a.dec_ctr + b * a.H + head, 1) == nsp - 1) a.dec_ctr[b * a.H + head] = 0;
      }
      if (tid == 128) {
        // let this pass's copies land before the CTA leaves (each wait bounded)
        for (int i = 0; i < nt; ++i) {
          const int q = q_base + i;
          if (!fa_wait(&S.full[q % DS], (uint32_t)((q / DS) & 1))) break;
        }
      }
      return;
    }
    if (w < 4) {
#pragma unroll
      for (int n8 = 0; n8 < 8; ++n8) {
        *reinterpret_cast<float2*>(&Ob[w][g][8 * n8 + 2 * tq]) = make_float2(oc[n8][0], oc[n8][1]);
        *reinterpret_cast<float2*>(&Ob[w][g + 8][8 * n8 + 2 * tq]) = make_float2(oc[n8][2], oc[n8][3]);
      }
      if (tq == 0) {
        Ob[w][g][HD] = m0;
        Ob[w][g][HD + 1] = l0;
        Ob[w][g + 8][HD] = m1;
        Ob[w][g + 8][HD + 1] = l1;
      }
    }
    __syncthreads();
    if (w < 4) {
      for (int j = w; j < ng; j += 4) {
        float M = -CUDART_INF_F;
#pragma unroll
        for (int u = 0; u < 4; ++u) M = fmaxf(M, Ob[u][j][HD]);
        float L = 0.f, acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float mu = Ob[u][j][HD];
          if (mu == -CUDART_INF_F) continue;
          const float e = expf(mu - M);
          L += Ob[u][j][HD + 1] * e;
          const float2 v = *reinterpret_cast<const float2*>(&Ob[u][j][2 * lane]);
          acc0 += v.x * e;
          acc1 += v.y * e;
        }
        if (nsp == 1) {
          const float inv = 1.0f / L;
          *reinterpret_cast<__nv_bfloat162*>((__nv_bfloat16*)a.o + (size_t)(g0 + j) * H * HD + head * HD + 2 * lane) =
              __floats2bfloat162_rn(acc0 * inv, acc1 * inv);
        } else {
          float* pp = a.part + (((size_t)(g0 + j) * H + head) * a.kv_splits + sp) * OLD;
          *reinterpret_cast<float2*>(pp + 2 * lane) = make_float2(acc0, acc1);
          if (lane == 0) {
            pp[HD] = M;
            pp[HD + 1] = L;
          }
        }
      }
    }
    // the ring's next loads overwrite the merge buffer: order these generic
    // accesses before them
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    q_base += nt;
  }
  if (a.lens && head == 0 && sp == 0 && tid == 0) a.lens[b * a.L + a.layer] = pos_last + 1;
  if (nsp > 1) dec_merge_splits(a, b, head, s0, s1);
}

// ---------------------------------------------------------------------------
// Prefill / scoring: CTA (sequence, head, 64-row query tile), warp w owns
// query rows 16w .. 16w+15 of the tile.  Key tiles of 64 positions (one TMA
// box of K and one of V, 128-byte swizzled) stream through a 3-stage ring;
// each tile is used by all four warps, then refilled.  Per tile and warp:
// S = Q K^T (32 MMAs), causal mask, online softmax (running max m and sum l
// per row, O rescaled when m grows), O += P V with P as a bf16 hi/lo pair (64
// MMAs).  Rows of one sequence have consecutive positions; row p attends to
// keys 0..p, all in the cache (the QKV epilogue wrote this pass's keys).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) k_attn_fa_mma(const __grid_constant__ CUtensorMap kvmap, AttnArgs a) {
  pdl_wait();
  pdl_launch();
  extern __shared__ unsigned char smem_raw[];
  FaSmem& S = *reinterpret_cast<FaSmem*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  if (*a.rs.nrows == 0) return;
  // grid (row tile, head, sequence): the row tiles of one (sequence, head),
  // which all read the same keys, run next to each other and share them in L2
  const int b = blockIdx.z, head = blockIdx.y;
  const int s0 = a.rs.seq_start[b], s1 = a.rs.seq_start[b + 1];
  const int nrt = (s1 - s0 + FQ - 1) / FQ;
  const int rt = nrt - 1 - (int)blockIdx.x;  // the longest (latest) row tiles start first
  if (rt < 0) return;
  const int g0 = s0 + rt * FQ, g1 = min(s1, g0 + FQ), nr = g1 - g0;
  const int pos_last = a.rs.row_pos[g1 - 1];
  const int ntk = pos_last / FK + 1;
  const int tid = threadIdx.x;
  if (tid == 0) {
    S.abort = 0;
    for (int st = 0; st < FST; ++st)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(saddr(&S.full[st])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int j = 0; j < FST && j < ntk; ++j) fa_issue(S, &kvmap, a, b, head, j, j);
  }
  const int H = a.H;
  const __nv_bfloat16* qg = (const __nv_bfloat16*)a.q;
  for (int i = tid; i < FQ * 8; i += 128) {
    const int r = i >> 3, c = i & 7;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < nr) v = *reinterpret_cast<const uint4*>(qg + (size_t)(g0 + r) * H * HD + head * HD + c * 8);
    *reinterpret_cast<uint4*>(S.Q + r * QLD + c * 8) = v;
  }
  __syncthreads();
  const int w = tid >> 5, lane = tid & 31, g = lane >> 2, tq = lane & 3;
  const int rl0 = 16 * w + g, rl1 = rl0 + 8;
  const int p0 = rl0 < nr ? a.rs.row_pos[g0 + rl0] : -1;
  const int p1 = rl1 < nr ? a.rs.row_pos[g0 + rl1] : -1;
  const int pw = 16 * w < nr ? a.rs.row_pos[g0 + min(nr - 1, 16 * w + 15)] : -1;  // warp's last position
  uint32_t qa[4][4];
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
    ldsm_x4(qa[ks], saddr(S.Q + (16 * w + (lane & 7) + 8 * ((lane >> 3) & 1)) * QLD + (2 * ks + (lane >> 4)) * 8));
  float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F, l0 = 0.f, l1 = 0.f;
  float oc[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) oc[nt][e] = 0.f;
  int failed_at = -1;
  for (int j = 0; j < ntk; ++j) {
    const int stg = j % FST;
    if (!fa_wait(&S.full[stg], (uint32_t)((j / FST) & 1))) S.abort = 1;
    const int k0 = j * FK;
    if (j == ntk - 1 && pos_last + 1 - k0 < FK) {
      // V rows past the last key may be stale or never written: zero them
      // (P is 0 there, and 0 * NaN would poison the sums)
      const int nk = pos_last + 1 - k0;
      for (int i = nk * 8 + tid; i < FK * 8; i += 128)
        *reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(S.V[stg]) + (i >> 3) * 128 + (i & 7) * 16) =
            make_uint4(0, 0, 0, 0);
      __syncthreads();
    }
    if (pw >= k0) {
      const uint32_t kb_ = saddr(S.K[stg]), vb_ = saddr(S.V[stg]);
      float sc[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[nt][e] = 0.f;
        const int r = 8 * nt + (lane & 7);
#pragma unroll
        for (int kp = 0; kp < 2; ++kp) {
          uint32_t kb[4];
          ldsm_x4(kb, kb_ + swz(r, 4 * kp + (lane >> 3)));
          mma_bf16(sc[nt], qa[2 * kp], kb[0], kb[1]);
          mma_bf16(sc[nt], qa[2 * kp + 1], kb[2], kb[3]);
        }
      }
      float t0 = -CUDART_INF_F, t1 = -CUDART_INF_F;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kk = k0 + 8 * nt + 2 * tq + (e & 1);
          const bool hi = e >= 2;
          const float v = kk <= (hi ? p1 : p0) ? sc[nt][e] * a.scale : -CUDART_INF_F;
          sc[nt][e] = v;
          if (hi) t1 = fmaxf(t1, v); else t0 = fmaxf(t0, v);
        }
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) {
        t0 = fmaxf(t0, __shfl_xor_sync(0xffffffffu, t0, o));
        t1 = fmaxf(t1, __shfl_xor_sync(0xffffffffu, t1, o));
      }
      const float n0 = fmaxf(m0, t0), n1 = fmaxf(m1, t1);
      const float c0 = n0 == -CUDART_INF_F ? 1.f : expf(m0 - n0);
      const float c1 = n1 == -CUDART_INF_F ? 1.f : expf(m1 - n1);
      m0 = n0;
      m1 = n1;
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool hi = e >= 2;
          const float m = hi ? n1 : n0;
          const float pr = m == -CUDART_INF_F ? 0.f : expf(sc[nt][e] - m);
          sc[nt][e] = pr;
          if (hi) a1 += pr; else a0 += pr;
        }
      l0 = l0 * c0 + a0;  // this thread's columns; the quad is summed at the end
      l1 = l1 * c1 + a1;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        oc[nt][0] *= c0;
        oc[nt][1] *= c0;
        oc[nt][2] *= c1;
        oc[nt][3] *= c1;
      }
#pragma unroll
      for (int kq = 0; kq < 4; ++kq) {
        uint32_t ph[4], pl[4];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const float x0 = sc[2 * kq + h][2 * rr], x1 = sc[2 * kq + h][2 * rr + 1];
            const __nv_bfloat16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
            ph[2 * h + rr] = pack_bf16(__bfloat162float(h0), __bfloat162float(h1));
            pl[2 * h + rr] = pack_bf16(x0 - __bfloat162float(h0), x1 - __bfloat162float(h1));
          }
        const int r = 16 * kq + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t vb[4];
          ldsm_x4_t(vb, vb_ + swz(r, 2 * np + (lane >> 4)));
          mma_bf16(oc[2 * np], ph, vb[0], vb[1]);
          mma_bf16(oc[2 * np], pl, vb[0], vb[1]);
          mma_bf16(oc[2 * np + 1], ph, vb[2], vb[3]);
          mma_bf16(oc[2 * np + 1], pl, vb[2], vb[3]);
        }
      }
    }
    __syncthreads();  // every warp is done with this stage
    if (S.abort) {
      failed_at = j;
      break;
    }
    if (tid == 0 && j + FST < ntk) fa_issue(S, &kvmap, a, b, head, j + FST, stg);
  }
  if (failed_at >= 0) {
    if (tid == 0) {
      dev_fail(a.status, DEV_ERR_TIMEOUT);
      // tiles failed_at .. failed_at + FST - 1 were issued and not consumed:
      // let those copies land before the CTA leaves (each wait bounded)
      for (int t = failed_at; t < failed_at + FST && t < ntk; ++t)
        if (!fa_wait(&S.full[t % FST], (uint32_t)((t / FST) & 1))) break;
    }
    return;
  }
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  __nv_bfloat16* og = (__nv_bfloat16*)a.o;
  if (rl0 < nr) {
    const float inv = 1.0f / l0;
    __nv_bfloat16* orow = og + (size_t)(g0 + rl0) * H * HD + head * HD;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
      *reinterpret_cast<__nv_bfloat162*>(orow + 8 * nt + 2 * tq) = __floats2bfloat162_rn(oc[nt][0] * inv, oc[nt][1] * inv);
  }
  if (rl1 < nr) {
    const float inv = 1.0f / l1;
    __nv_bfloat16* orow = og + (size_t)(g0 + rl1) * H * HD + head * HD;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
      *reinterpret_cast<__nv_bfloat162*>(orow + 8 * nt + 2 * tq) = __floats2bfloat162_rn(oc[nt][2] * inv, oc[nt][3] * inv);
  }
  if (a.lens && head == 0 && g1 == s1 && tid == 0) a.lens[b * a.L + a.layer] = pos_last + 1;
}

}  // namespace

cudaError_t attn_mma_prepare() {
  cudaError_t e = cudaFuncSetAttribute(k_attn_dec_mma, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)DEC_SMEM_BYTES);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_attn_fa_mma, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FA_SMEM_BYTES);
  return e;
}

void launch_attn_dec_mma(const CUtensorMap* kvmap, const AttnArgs& a, cudaStream_t st) {
  dim3 grid(a.rs.B, a.H, a.kv_splits);
  launch_k(k_attn_dec_mma, grid, DEC_THREADS, DEC_SMEM_BYTES, st, *kvmap, a);
}

void launch_attn_fa_mma(const CUtensorMap* kvmap, const AttnArgs& a, cudaStream_t st) {
  dim3 grid((a.row_groups * ATTN_RPC + FQ - 1) / FQ, a.H, a.rs.B);
  launch_k(k_attn_fa_mma, grid, 128, FA_SMEM_BYTES, st, *kvmap, a);
}

}  // namespace nv
