// Decode / flush attention for bf16 caches with head_dim 64, streamed by
// persistent warps (k_attn_dec_pc).
//
// What it computes is the causal softmax attention of the LLaMA-2 backbone
// ("N-vium: Mixture-of-Exits Transformer for Accelerated Exact Generation",
// section 4) for the rows a decode step or a flush runs at one layer: the
// new token of each sequence plus its deferred rows (section 2 "Inferenz:
// Piggybacking").  For a row at position p, o = sum_j softmax_j(q . k_j /
// sqrt(hd)) v_j over keys j <= p.
//
// Work split: a (sequence, head, 16-row pass) has its keys cut into chunks
// of CH 32-key tiles; each (sequence, head, pass, chunk) is one item.  CH
// is chosen per launch from the total number of tiles, so a launch has
// about four items per warp of the grid and items are nearly equal in size.
// One CTA per SM with eight independent warps; a warp takes the next item
// from a global counter (one ahead, so its loads can start early), and keeps
// its own three-stage TMA ring of 32-key K/V tiles streaming across item
// boundaries.  Per tile: S = q K^T and O += P V on mma.sync m16n8k16 (bf16
// in, fp32 accumulation; P as a bf16 pair hi + lo), online softmax.  An item
// that covers all of a pass's keys writes normalised output rows; otherwise
// it writes unnormalised partials (sum, max, weight sum) per row and chunk,
// and the last item of the (sequence, head) to finish (an arrival counter)
// merges every row's chunks in chunk order, so the result does not depend
// on which warp came last.
//
// Compared with one CTA per (sequence, head) (k_attn_dec_mma): no wave
// quantisation or tail from unequal sequence lengths, no per-CTA start-up
// between items, and a warp's ring never drains at an item boundary.  On
// B200 it measured slower all the same (B=64 decode steps 31% longer), so it
// runs only when NVIUM_DEC_ATTN=pc selects it.
#include <math_constants.h>

#include "common.cuh"
#include "kernels.cuh"
#include "mma_prims.cuh"

namespace nv {
namespace {
using namespace mp;

constexpr int HD = 64;                    // head dim (128-byte rows)
constexpr int RG = 16;                    // rows per pass (one MMA row block)
constexpr int QLD = HD + 8;               // padded Q row: conflict-free ldmatrix
constexpr int OLD = HD + 2;               // partial row: HD sums, max, weight sum
constexpr int TK = 32;                    // keys per tile
constexpr int TBYTES = TK * HD * 2;       // one K or V box: 4 KB
constexpr int NW = 8;                     // warps per CTA
constexpr int NS = 3;                     // ring stages per warp
constexpr int MIN_CH = 4;                 // tiles per chunk, at least (the partial slots hold 128-key splits)
constexpr int MAXB = 512;                 // sequences the in-CTA item table holds
constexpr int RING_BYTES = NW * NS * 2 * TBYTES;
constexpr int Q_BYTES = NW * RG * QLD * 2;
constexpr size_t PC_SMEM_BYTES =
    RING_BYTES + Q_BYTES + NW * NS * 8 /*full barriers*/ + 4 * (MAXB + 1) * 4 /*item table*/ + 1024 /*align*/;
static_assert(PC_SMEM_BYTES <= 227 * 1024, "shared memory of one CTA");

// bounded wait on a ring stage by lane 0; false once 2 s have passed
__device__ __forceinline__ bool stage_wait(uint64_t* bar, uint32_t parity) {
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

// The per-launch item table, in shared memory: cum[b] = items of sequences
// before b; info[b] = passes << 16 | chunks; s0[b] = first row; plast[b] =
// position of b's last row.
struct Table {
  int* cum;
  int* info;
  int* s0;
  int* plast;
};

struct Item {
  int b, head, pass, chunk, nch, npass;
  int t0, t1;     // 32-key tiles [t0, t1)
  int g0, ng;     // rows [g0, g0 + ng)
  int s0, s1, plast;
};

__device__ __forceinline__ Item decode_item(const Table& T, int B, int CH, int i) {
  int lo = 0, hi = B - 1;  // the b with cum[b] <= i < cum[b + 1]
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (T.cum[mid] <= i) lo = mid;
    else hi = mid - 1;
  }
  Item it;
  it.b = lo;
  const int local = i - T.cum[lo];
  it.npass = T.info[lo] >> 16;
  it.nch = T.info[lo] & 0xffff;
  const int per_head = it.npass * it.nch;
  it.head = local / per_head;
  const int rem = local - it.head * per_head;
  it.pass = rem / it.nch;
  it.chunk = rem - it.pass * it.nch;
  it.s0 = T.s0[lo];
  it.s1 = T.s0[lo + 1];
  it.plast = T.plast[lo];
  const int ntk = it.plast / TK + 1;
  it.t0 = it.chunk * CH;
  it.t1 = min(ntk, it.t0 + CH);
  it.g0 = it.s0 + it.pass * RG;
  it.ng = min(RG, it.s1 - it.g0);
  return it;
}

// Last arrival of a (sequence, head): merge each row's chunk partials in
// chunk order and write the normalised output (one warp).
__device__ __forceinline__ void merge_chunks(const AttnArgs& a, const Item& it, int lane) {
  const int H = a.H;
  for (int r = it.s0; r < it.s1; ++r) {
    const float* pp = a.part + ((size_t)r * H + it.head) * a.kv_splits * OLD;
    float M = -CUDART_INF_F;
    for (int c = 0; c < it.nch; ++c) M = fmaxf(M, __ldcg(pp + c * OLD + HD));
    float L = 0.f, acc0 = 0.f, acc1 = 0.f;
    for (int c = 0; c < it.nch; ++c) {
      const float mc = __ldcg(pp + c * OLD + HD);
      if (mc == -CUDART_INF_F) continue;
      const float e = expf(mc - M);
      L += __ldcg(pp + c * OLD + HD + 1) * e;
      const float2 v = __ldcg(reinterpret_cast<const float2*>(pp + c * OLD + 2 * lane));
      acc0 += v.x * e;
      acc1 += v.y * e;
    }
    const float inv = 1.0f / L;
    *reinterpret_cast<__nv_bfloat162*>((__nv_bfloat16*)a.o + (size_t)r * H * HD + it.head * HD + 2 * lane) =
        __floats2bfloat162_rn(acc0 * inv, acc1 * inv);
  }
}

// Q rows of an item, 16 rows x 8 chunks of 16 bytes: lane takes chunks
// lane + 32 k (row (lane + 32 k) / 8, chunk lane % 8); rows past ng are zero
__device__ __forceinline__ void load_q(const AttnArgs& a, const Item& it, int lane, uint4 (&qv)[4]) {
  const __nv_bfloat16* qg = (const __nv_bfloat16*)a.q;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int e = lane + 32 * k, r = e >> 3, c = e & 7;
    qv[k] = r < it.ng ? *reinterpret_cast<const uint4*>(qg + (size_t)(it.g0 + r) * a.H * HD + it.head * HD + c * 8)
                      : make_uint4(0, 0, 0, 0);
  }
}

// the page of each 64- or 128-position page the item's keys touch: lane l
// holds page (t0 * TK) / page_size + l of sequence b
__device__ __forceinline__ int load_page(const AttnArgs& a, const Item& it, int lane) {
  const int p = (it.t0 * TK) / a.kv.page_size + lane;
  const int plast = (it.t1 * TK - 1) / a.kv.page_size;
  return p <= plast ? a.kv.page_table[(size_t)it.b * a.kv.pages_per_seq + p] : 0;
}

__global__ void __launch_bounds__(NW * 32, 1) k_attn_dec_pc(const __grid_constant__ CUtensorMap kvmap, AttnArgs a) {
  pdl_wait();
  pdl_launch();
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ int s_red[NW];
  __shared__ int s_ch;
  if (*a.rs.nrows == 0) return;
  const int B = a.rs.B, H = a.H, tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  uint64_t* bars = (uint64_t*)(sm + RING_BYTES + Q_BYTES);
  Table T;
  T.cum = (int*)(bars + NW * NS);
  T.info = T.cum + MAXB + 1;
  T.s0 = T.info + MAXB + 1;
  T.plast = T.s0 + MAXB + 1;

  // ---- item table (every CTA builds the same one) ----
  if (tid < NW * NS) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(saddr(bars + tid)) : "memory");
  long long tp = 0;  // tile-passes of this thread's sequences
  for (int b = tid; b < B; b += NW * 32) {
    const int s0 = a.rs.seq_start[b], s1 = a.rs.seq_start[b + 1];
    int pl = -1, np = 0;
    if (s1 > s0) {
      pl = a.rs.row_pos[s1 - 1];
      np = (s1 - s0 + RG - 1) / RG;
      tp += (long long)np * (pl / TK + 1);
    }
    T.s0[b] = s0;
    T.plast[b] = pl;
    T.info[b] = np << 16;
  }
  if (tid == 0) T.s0[B] = a.rs.seq_start[B];
#pragma unroll
  for (int o = 16; o; o >>= 1) tp += __shfl_xor_sync(0xffffffffu, tp, o);
  if (lane == 0) s_red[w] = (int)min(tp, (long long)INT_MAX);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  __syncthreads();
  if (tid == 0) {
    long long tot = 0;
    for (int i = 0; i < NW; ++i) tot += s_red[i];
    tot *= H;
    // about four items per warp of the grid; an item's keys span at most 31
    // pages, so a warp's lanes hold all its page ids
    const long long slots = 4ll * NW * gridDim.x;
    const int cap = 30 * a.kv.page_size / TK;
    s_ch = (int)max((long long)MIN_CH, min((long long)cap, (tot + slots - 1) / slots));
  }
  __syncthreads();
  const int CH = s_ch;
  if (w == 0) {
    int run = 0;
    for (int base = 0; base < B; base += 32) {
      const int b = base + lane;
      int n = 0;
      if (b < B) {
        const int np = T.info[b] >> 16;
        if (np) {
          const int nch = (T.plast[b] / TK + 1 + CH - 1) / CH;
          T.info[b] = (np << 16) | nch;
          n = H * np * nch;
        }
      }
      int x = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (b < B) T.cum[b] = run + x - n;
      run += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) T.cum[B] = run;
  }
  __syncthreads();
  const int total = T.cum[B];

  // ---- per warp: items from the global counter, tiles through its ring ----
  unsigned char* ring = sm + w * NS * 2 * TBYTES;  // stage s: K at 2 s TBYTES, V after it
  uint64_t* full = bars + w * NS;
  __nv_bfloat16* qs = (__nv_bfloat16*)(sm + RING_BYTES) + w * RG * QLD;
  int* work = a.dec_ctr + B * H;  // [0]: next item, [1]: warps done
  const int g = lane >> 2, tq = lane & 3;
  auto grab = [&]() {
    int v = 0;
    if (lane == 0) v = atomicAdd(work, 1);
    return __shfl_sync(0xffffffffu, v, 0);
  };
  int cur = grab();
  int nxt = cur < total ? grab() : total;
  Item ic, in;
  uint4 qn[4];              // next item's q rows
  int pc = 0, pn = 0;       // page ids (lane l: l-th page of the item)
  int rp0 = -1, rp1 = -1;   // next item's row positions (rows g, g + 8)
  if (cur < total) {
    ic = decode_item(T, B, CH, cur);
    pc = load_page(a, ic, lane);
  }
  if (nxt < total) {
    in = decode_item(T, B, CH, nxt);
    pn = load_page(a, in, lane);
  }
  // producer cursor: item (0 = current, 1 = next, 2 = none) and tile
  int p_which = cur < total ? 0 : 2, p_tile = cur < total ? ic.t0 : 0;
  int q_issue = 0, q_cons = 0;
  bool dead = false;
  const int ps = a.kv.page_size;
  const size_t hstride = (size_t)ps * HD, pstride = 2 * (size_t)H * hstride;
  const size_t lbase = (size_t)a.layer * a.kv.layer_stride;
  // issue loads while a stage is free (warp-uniform; lane 0 issues)
  auto top_up = [&]() {
    while (!dead && q_issue - q_cons < NS && p_which < 2) {
      const Item& pt = p_which == 0 ? ic : in;
      if (p_tile >= pt.t1) {
        if (p_which == 0 && nxt < total) {
          p_which = 1;
          p_tile = in.t0;
          continue;
        }
        p_which = 2;
        break;
      }
      const int pos = p_tile * TK;
      const int page = __shfl_sync(0xffffffffu, p_which == 0 ? pc : pn, pos / ps - (pt.t0 * TK) / ps);
      if (lane == 0) {
        const int st = q_issue % NS;
        unsigned char* kd = ring + st * 2 * TBYTES;
        // this stage's earlier generic reads and writes come before the copy
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(full + st)),
                     "r"((uint32_t)(2 * TBYTES))
                     : "memory");
        const size_t off = lbase + (size_t)page * pstride + (size_t)pt.head * hstride + (size_t)(pos % ps) * HD;
        tma_box(kd, &kvmap, full + st, (int)(off / HD));
        tma_box(kd + TBYTES, &kvmap, full + st, (int)((off + (size_t)H * hstride) / HD));
      }
      ++q_issue;
      ++p_tile;
    }
  };
  if (cur < total) {
    load_q(a, ic, lane, qn);
    rp0 = g < ic.ng ? a.rs.row_pos[ic.g0 + g] : -1;
    rp1 = g + 8 < ic.ng ? a.rs.row_pos[ic.g0 + g + 8] : -1;
  }
  top_up();

  while (cur < total) {
    const Item it = ic;
    // this item's q rows: registers -> shared memory -> MMA fragments
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int e = lane + 32 * k;
      *reinterpret_cast<uint4*>(qs + (e >> 3) * QLD + (e & 7) * 8) = qn[k];
    }
    __syncwarp();
    uint32_t qa[4][4];
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
      ldsm_x4(qa[ks], saddr(qs + ((lane & 7) + 8 * ((lane >> 3) & 1)) * QLD + (2 * ks + (lane >> 4)) * 8));
    const int p0 = rp0, p1 = rp1;
    // the next item's q rows and row positions, in flight during this one
    if (nxt < total) {
      load_q(a, in, lane, qn);
      rp0 = g < in.ng ? a.rs.row_pos[in.g0 + g] : -1;
      rp1 = g + 8 < in.ng ? a.rs.row_pos[in.g0 + g + 8] : -1;
    }
    float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F, l0 = 0.f, l1 = 0.f;
    float oc[8][4];
#pragma unroll
    for (int n8 = 0; n8 < 8; ++n8)
#pragma unroll
      for (int e = 0; e < 4; ++e) oc[n8][e] = 0.f;
    for (int t = it.t0; t < it.t1 && !dead; ++t) {
      const int st = q_cons % NS;
      int ok = 1;
      if (lane == 0) ok = stage_wait(full + st, (uint32_t)((q_cons / NS) & 1)) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        dead = true;
        if (lane == 0) dev_fail(a.status, DEV_ERR_TIMEOUT);
        break;
      }
      unsigned char* kd = ring + st * 2 * TBYTES;
      unsigned char* vd = kd + TBYTES;
      const int k0 = t * TK;
      if (k0 + TK > it.plast + 1) {
        // V rows past the last key may be stale or never written: zero them
        // (P is 0 there, and 0 * NaN would poison the sums)
        for (int e = (it.plast + 1 - k0) * 8 + lane; e < TK * 8; e += 32)
          *reinterpret_cast<uint4*>(vd + (e >> 3) * 128 + (e & 7) * 16) = make_uint4(0, 0, 0, 0);
        __syncwarp();
      }
      const uint32_t kb_ = saddr(kd), vb_ = saddr(vd);
      float sc[4][4];
#pragma unroll
      for (int n8 = 0; n8 < 4; ++n8) {
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
      for (int n8 = 0; n8 < 4; ++n8)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kk = k0 + 8 * n8 + 2 * tq + (e & 1);
          const bool hi = e >= 2;
          const float v = kk <= (hi ? p1 : p0) ? sc[n8][e] * a.scale : -CUDART_INF_F;
          sc[n8][e] = v;
          if (hi) t1 = fmaxf(t1, v);
          else t0 = fmaxf(t0, v);
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
      for (int n8 = 0; n8 < 4; ++n8)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool hi = e >= 2;
          const float m = hi ? n1 : n0;
          const float pr = m == -CUDART_INF_F ? 0.f : expf(sc[n8][e] - m);
          sc[n8][e] = pr;
          if (hi) a1 += pr;
          else a0 += pr;
        }
      l0 = l0 * c0 + a0;  // this thread's columns; the quad is summed at the end
      l1 = l1 * c1 + a1;
#pragma unroll
      for (int n8 = 0; n8 < 8; ++n8) {
        oc[n8][0] *= c0;
        oc[n8][1] *= c0;
        oc[n8][2] *= c1;
        oc[n8][3] *= c1;
      }
#pragma unroll
      for (int kq = 0; kq < 2; ++kq) {
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
      ++q_cons;
      top_up();
    }
    if (!dead) {
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, o);
        l1 += __shfl_xor_sync(0xffffffffu, l1, o);
      }
#pragma unroll
      for (int hrow = 0; hrow < 2; ++hrow) {
        const int j = g + 8 * hrow;
        if (j >= it.ng) continue;
        const int row = it.g0 + j;
        const float m = hrow ? m1 : m0, l = hrow ? l1 : l0;
        if (it.nch == 1) {
          const float inv = 1.0f / l;
          __nv_bfloat16* orow = (__nv_bfloat16*)a.o + (size_t)row * H * HD + it.head * HD;
#pragma unroll
          for (int n8 = 0; n8 < 8; ++n8)
            *reinterpret_cast<__nv_bfloat162*>(orow + 8 * n8 + 2 * tq) =
                __floats2bfloat162_rn(oc[n8][2 * hrow] * inv, oc[n8][2 * hrow + 1] * inv);
        } else {
          float* pp = a.part + (((size_t)row * H + it.head) * a.kv_splits + it.chunk) * OLD;
#pragma unroll
          for (int n8 = 0; n8 < 8; ++n8)
            *reinterpret_cast<float2*>(pp + 8 * n8 + 2 * tq) = make_float2(oc[n8][2 * hrow], oc[n8][2 * hrow + 1]);
          if (tq == 0) {
            pp[HD] = m;
            pp[HD + 1] = l;
          }
        }
      }
    }
    if (it.nch > 1) {
      // every item of the (sequence, head) arrives once, also after an
      // expired wait, so the counter is back at zero for the next launch
      __threadfence();
      __syncwarp();
      int last = 0;
      if (lane == 0) {
        int* c = a.dec_ctr + it.b * H + it.head;
        last = atomicAdd(c, 1) == it.npass * it.nch - 1;
        if (last) *c = 0;
      }
      if (__shfl_sync(0xffffffffu, last, 0) && !dead) {
        __threadfence();
        merge_chunks(a, it, lane);
      }
    }
    if (a.lens && !dead && it.head == 0 && it.pass == 0 && it.chunk == 0 && lane == 0)
      a.lens[it.b * a.L + a.layer] = it.plast + 1;
    cur = nxt;
    if (cur < total) {
      ic = in;
      pc = pn;
      // the producer had moved on to this item (1), or had issued all of its
      // tiles and stopped for want of a next item (2)
      if (p_which == 1) {
        p_which = 0;
      } else if (p_which == 2) {
        p_which = 0;
        p_tile = ic.t1;
      }
      nxt = grab();
      if (nxt < total) {
        in = decode_item(T, B, CH, nxt);
        pn = load_page(a, in, lane);
      }
      top_up();
    }
  }
  if (lane == 0) {
    // copies still in flight (only after an expired wait) land before the warp leaves
    for (int q = q_cons; q < q_issue; ++q)
      if (!stage_wait(full + q % NS, (uint32_t)((q / NS) & 1))) break;
    // the last warp of the launch to finish resets the item counter
    if (atomicAdd(work + 1, 1) == NW * (int)gridDim.x - 1) {
      work[0] = 0;
      work[1] = 0;
    }
  }
}

}  // namespace

cudaError_t attn_dec_pc_prepare() {
  return cudaFuncSetAttribute(k_attn_dec_pc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PC_SMEM_BYTES);
}

bool attn_dec_pc_fits(const AttnArgs& a) { return a.kv_map32 && a.hd == HD && a.rs.B <= MAXB && a.part; }

void launch_attn_dec_pc(const AttnArgs& a, cudaStream_t st) {
  static int nsm = 0;
  if (!nsm) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm <= 0) nsm = 148;
  }
  launch_k(k_attn_dec_pc, nsm, NW * 32, PC_SMEM_BYTES, st, *a.kv_map32, a);
}

}  // namespace nv
