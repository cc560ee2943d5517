// libnvium kernels: planner + RMSNorm, SIMT GEMM and epilogues, paged
// attention, exit junction and the fused exit-head sampler, scoring.
//
// Method: "N-vium: Mixture-of-Exits Transformer for Accelerated Exact
// Generation" (arXiv 2605.13190).  Section 2 "Architektur" gives the exit
// probability p_k and the mixture pi_mix; section 2 "Inferenz: Piggybacking"
// gives the deferral of the layers above an exit and their batching with
// later tokens; the backbone is LLaMA-2 (section 4).
#include <math_constants.h>

#include <cstdlib>

#include "kernels.cuh"

namespace nv {

bool pdl_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* e = std::getenv("NVIUM_PDL");
    on = (e && e[0] == '0') ? 0 : 1;
  }
  return on == 1;
}

// ---------------------------------------------------------------------------
// reductions (fixed shuffle / tree order: results are deterministic)
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ long long warp_sum_ll(long long v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sum over the block (NT threads); every thread gets the total.
template <int NT>
__device__ float block_sum(float v) {
  __shared__ float s[NT / 32];
  __shared__ float tot;
  v = warp_sum(v);
  if ((threadIdx.x & 31) == 0) s[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    float a = 0.f;
    for (int i = 0; i < NT / 32; ++i) a += s[i];
    tot = a;
  }
  __syncthreads();
  const float r = tot;
  __syncthreads();
  return r;
}

// Exclusive prefix sum of one int per thread over the block; *total = sum.
template <int NT>
__device__ int block_exclusive_scan(int v, int* total) {
  __shared__ int ws[NT / 32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) ws[w] = x;
  __syncthreads();
  if (w == 0) {
    int s = lane < NT / 32 ? ws[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < NT / 32) ws[lane] = s;
  }
  __syncthreads();
  const int excl = x - v + (w ? ws[w - 1] : 0);
  *total = ws[NT / 32 - 1];
  __syncthreads();
  return excl;
}

// Largest b with start[b] <= r (start non-decreasing, start[0] = 0).
__device__ __forceinline__ int find_seq(const int* start, int B, int r) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (start[mid] <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// RMSNorm of one row by one warp: out = rnd(g * h / sqrt(mean(h^2) + eps)).
// The row is read once with 16-byte loads and kept in registers (d <= 2048).
// With Y set, the row is first completed by the residual update
// h += sum_s Y[s] (split-K slices of a GEMM, summed in slice order) and the
// new h is written back.
constexpr int NORM_MAXV = 16;
template <typename T> __device__ __forceinline__ void store4(T* p, float a, float b, float c, float d);
template <> __device__ __forceinline__ void store4<float>(float* p, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}
template <> __device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, float a, float b, float c, float d) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&lo);
  u.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(p) = u;
}
template <typename T>
__device__ __forceinline__ void warp_norm_row(float* __restrict__ h, const T* __restrict__ g, T* __restrict__ out,
                                              int d, float eps, const float* __restrict__ Y = nullptr, int ns = 0,
                                              size_t sstride = 0) {
  const int lane = threadIdx.x & 31, nv = d >> 2;
  float4 x[NORM_MAXV];
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < NORM_MAXV; ++c) {
    const int j = lane + 32 * c;
    if (j < nv) {
      float4 v = reinterpret_cast<const float4*>(h)[j];
      if (Y) {
        float4 ys = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int sp = 0; sp < ns; ++sp) {
          const float4 y = __ldcg(reinterpret_cast<const float4*>(Y + sp * sstride) + j);
          ys.x += y.x;
          ys.y += y.y;
          ys.z += y.z;
          ys.w += y.w;
        }
        v.x += ys.x;
        v.y += ys.y;
        v.z += ys.z;
        v.w += ys.w;
        reinterpret_cast<float4*>(h)[j] = v;
      }
      x[c] = v;
      ss = fmaf(v.x, v.x, ss);
      ss = fmaf(v.y, v.y, ss);
      ss = fmaf(v.z, v.z, ss);
      ss = fmaf(v.w, v.w, ss);
    }
  }
  ss = warp_sum(ss);
  const float inv = 1.0f / sqrtf(ss / (float)d + eps);
#pragma unroll
  for (int c = 0; c < NORM_MAXV; ++c) {
    const int j = lane + 32 * c;
    if (j < nv) {
      const T* gp = g + 4 * j;
      store4<T>(out + 4 * j, x[c].x * inv * ld(gp), x[c].y * inv * ld(gp + 1), x[c].z * inv * ld(gp + 2),
                x[c].w * inv * ld(gp + 3));
    }
  }
}

// ---------------------------------------------------------------------------
// RoPE table: (cos, sin) of pos * theta^(-2i/hd), computed in double.
// ---------------------------------------------------------------------------
__global__ void k_rope_table(float2* cs, int max_seq, int hd, double theta) {
  pdl_wait();
  pdl_launch();
  const int half = hd / 2;
  const long long n = (long long)max_seq * half;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
       idx += (long long)gridDim.x * blockDim.x) {
    const int pos = (int)(idx / half), i = (int)(idx % half);
    const double ang = (double)pos * pow(theta, -2.0 * (double)i / (double)hd);
    cs[idx] = make_float2((float)cos(ang), (float)sin(ang));
  }
}
void launch_rope_table(float2* cs, int max_seq, int hd, double theta, cudaStream_t st) {
  launch_k(k_rope_table, 256, 256, 0, st, cs, max_seq, hd, theta);
}

// ---------------------------------------------------------------------------
// embedding and RMSNorm over an explicit row set (prefill / scoring)
// ---------------------------------------------------------------------------
template <typename T>
__global__ void k_embed_rows(const T* __restrict__ emb, const int* __restrict__ tok, RowSet rs, int d) {
  pdl_wait();
  pdl_launch();
  const int R = *rs.nrows;
  for (int r = blockIdx.x; r < R; r += gridDim.x) {
    const T* e = emb + (size_t)tok[r] * d;
    float* h = rs.h + (size_t)rs.row_hrow[r] * d;
    for (int i = threadIdx.x; i < d; i += blockDim.x) h[i] = ld(e + i);
  }
}
void launch_embed_rows(bool bf16, const void* emb, const int* tok_row, RowSet rs, int d, cudaStream_t st) {
  const int grid = rs.max_rows < 4096 ? rs.max_rows : 4096;
  if (bf16) launch_k(k_embed_rows<__nv_bfloat16>, grid, 256, 0, st, (const __nv_bfloat16*)emb, tok_row, rs, d);
  else launch_k(k_embed_rows<float>, grid, 256, 0, st, (const float*)emb, tok_row, rs, d);
}

template <typename T>
__global__ void k_rmsnorm_rows(RowSet rs, const T* __restrict__ g, T* __restrict__ act, int d, float eps) {
  pdl_wait();
  pdl_launch();
  const int R = *rs.nrows;
  const int wpb = blockDim.x >> 5;
  for (int r = blockIdx.x * wpb + (threadIdx.x >> 5); r < R; r += gridDim.x * wpb)
    warp_norm_row<T>(rs.h + (size_t)rs.row_hrow[r] * d, g, act + (size_t)r * d, d, eps);
}
void launch_rmsnorm_rows(bool bf16, RowSet rs, const void* gain, void* act, int d, float eps, cudaStream_t st) {
  int grid = (rs.max_rows + 7) / 8;
  if (grid > 2048) grid = 2048;
  if (bf16)
    launch_k(k_rmsnorm_rows<__nv_bfloat16>, grid, 256, 0, st, rs, (const __nv_bfloat16*)gain, (__nv_bfloat16*)act, d, eps);
  else launch_k(k_rmsnorm_rows<float>, grid, 256, 0, st, rs, (const float*)gain, (float*)act, d, eps);
}

// Residual update from split-K slices of the output projection, then the MLP
// RMSNorm.  One CTA per row, one float4 of the row per thread (d <= 4 *
// blockDim), every slice's load in flight at once; the row stays in
// registers between the sum of squares and the scaled write.
template <typename T>
__global__ void __launch_bounds__(512) k_resid_norm(RowSet rs, const float* __restrict__ Y, int split_grid, int N,
                                                    int K, size_t sstride, const T* __restrict__ g,
                                                    T* __restrict__ act, int d, float eps) {
  pdl_wait();
  pdl_launch();
  __shared__ float s_red[16];
  const int R = *rs.nrows;
  const int ns = split_grid ? tc_split_count(R, N, K, split_grid, TC_MAX_SPLIT) : 1;
  const int nv = d >> 2, j = threadIdx.x;
  for (int r = blockIdx.x; r < R; r += gridDim.x) {
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    float4* hp = reinterpret_cast<float4*>(rs.h + (size_t)rs.row_hrow[r] * d);
    if (j < nv) {
      const float4* yp = reinterpret_cast<const float4*>(Y + (size_t)r * N) + j;
      float4 v[TC_MAX_SPLIT];
#pragma unroll
      for (int sp = 0; sp < TC_MAX_SPLIT; ++sp)
        v[sp] = sp < ns ? __ldcg(yp + sp * (sstride / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
      float4 ys = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int sp = 0; sp < TC_MAX_SPLIT; ++sp) {
        ys.x += v[sp].x;
        ys.y += v[sp].y;
        ys.z += v[sp].z;
        ys.w += v[sp].w;
      }
      x = hp[j];
      x.x += ys.x;
      x.y += ys.y;
      x.z += ys.z;
      x.w += ys.w;
      hp[j] = x;
    }
    float ss = sumsq4(x);
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
      float t = threadIdx.x < (blockDim.x >> 5) ? s_red[threadIdx.x] : 0.f;
      t = warp_sum(t);
      if (threadIdx.x == 0) s_red[0] = t;
    }
    __syncthreads();
    const float inv = 1.0f / sqrtf(s_red[0] / (float)d + eps);
    __syncthreads();
    if (j < nv) {
      const T* gp = g + 4 * j;
      store4<T>(act + (size_t)r * d + 4 * j, x.x * inv * ld(gp), x.y * inv * ld(gp + 1), x.z * inv * ld(gp + 2),
                x.w * inv * ld(gp + 3));
    }
  }
}
void launch_resid_norm(bool bf16, RowSet rs, const float* Y, int split_grid, int N, int K, size_t sstride,
                       const void* gain, void* act, int d, float eps, cudaStream_t st) {
  int grid = rs.max_rows < 1184 ? rs.max_rows : 1184;
  const int threads = ((d / 4 + 31) / 32) * 32;
  if (bf16)
    launch_k(k_resid_norm<__nv_bfloat16>, grid, threads, 0, st, rs, Y, split_grid, N, K, sstride,
             (const __nv_bfloat16*)gain, (__nv_bfloat16*)act, d, eps);
  else launch_k(k_resid_norm<float>, grid, threads, 0, st, rs, Y, split_grid, N, K, sstride, (const float*)gain,
                (float*)act, d, eps);
}

// ---------------------------------------------------------------------------
// Work-list planner fused with the attention RMSNorm (decode and flush).
//
// Rows of layer m for sequence b (section 2 "Inferenz: Piggybacking", lazy
// reading): when b's new token is still active at m, its deferred positions
// [len[b][m], t_b) followed by the new position t_b; when the sequence must
// complete early (its deferred store is full) the deferred positions alone;
// in flush mode every deferred position [len[b][m], t_b).  The layers between
// two exits keep equal cache lengths, so a plan made at a block's first layer
// serves the whole block (counters count it for a.nlayers layers).  Every CTA
// computes the same prefix sums in shared memory; CTA 0 publishes the list.
// ---------------------------------------------------------------------------
template <typename T, int NT>
__global__ void __launch_bounds__(NT) k_plan_norm(PlanArgs a, const T* __restrict__ gain, T* __restrict__ act,
                                                  int d, float eps) {
  pdl_wait();
  pdl_launch();
  extern __shared__ int s_start[];  // [B+1]
  __shared__ long long s_kv[NT / 32];
  const int B = a.B, tid = threadIdx.x;
  const int ipt = (B + NT - 1) / NT;
  const int b0 = tid * ipt;
  int local = 0;
  long long kvr = 0;
  for (int i = 0; i < ipt; ++i) {
    const int b = b0 + i;
    if (b >= B) break;
    const int tb = a.t[b], lb = a.lens[b * a.L + a.layer];
    int cnt = 0;
    if (a.mode == 1) {
      cnt = tb - lb;
    } else {
      const int ac = a.active[b];
      if (ac || a.force[b]) cnt = tb - lb + (ac ? 1 : 0);
    }
    if (cnt < 0) cnt = 0;
    s_start[b + 1] = cnt;
    local += cnt;
    if (cnt > 0) kvr += (long long)(lb + cnt) * a.kv_pos_bytes;
  }
  int total;
  int run = block_exclusive_scan<NT>(local, &total);
  for (int i = 0; i < ipt; ++i) {
    const int b = b0 + i;
    if (b >= B) break;
    run += s_start[b + 1];
    s_start[b + 1] = run;
  }
  if (tid == 0) s_start[0] = 0;
  __syncthreads();
  if (total > a.max_rows) {
    if (blockIdx.x == 0 && tid == 0) {
      dev_fail(a.status, DEV_ERR_ROWS);
      *a.nrows = 0;
    }
    return;
  }
  if (blockIdx.x == 0) {
    for (int b = tid; b <= B; b += NT) a.seq_start[b] = s_start[b];
    for (int r = tid; r < total; r += NT) {
      const int b = find_seq(s_start, B, r);
      const int pos = a.lens[b * a.L + a.layer] + (r - s_start[b]);
      a.row_b[r] = b;
      a.row_pos[r] = pos;
      a.row_hrow[r] = b * a.cap + pos % a.cap;
    }
    // bytes the layer must move: weights once, K/V of positions 0..last per sequence
    kvr = warp_sum_ll(kvr);
    if ((tid & 31) == 0) s_kv[tid >> 5] = kvr;
    __syncthreads();
    if (tid == 0) {
      *a.nrows = total;
      if (total > 0 && a.counters) {
        long long kv = 0;
        for (int i = 0; i < NT / 32; ++i) kv += s_kv[i];
        // the same rows run every layer of the block this plan serves
        const unsigned long long nl = (unsigned long long)(a.nlayers > 0 ? a.nlayers : 1);
        atomicAdd((unsigned long long*)&a.counters[NV_CTR_ROWS], (unsigned long long)total * nl);
        atomicAdd((unsigned long long*)&a.counters[NV_CTR_LAYERS_RUN], nl);
        atomicAdd((unsigned long long*)&a.counters[NV_CTR_WEIGHT_BYTES], (unsigned long long)a.weight_bytes * nl);
        atomicAdd((unsigned long long*)&a.counters[NV_CTR_KV_READ_BYTES], (unsigned long long)kv * nl);
        atomicAdd((unsigned long long*)&a.counters[NV_CTR_KV_WRITE_BYTES],
                  (unsigned long long)((long long)total * a.kv_pos_bytes) * nl);
      }
    }
  }
  const int wpb = NT / 32;
  for (int r = blockIdx.x * wpb + (tid >> 5); r < total; r += gridDim.x * wpb) {
    const int b = find_seq(s_start, B, r);
    const int pos = a.lens[b * a.L + a.layer] + (r - s_start[b]);
    const int hrow = b * a.cap + pos % a.cap;
    warp_norm_row<T>(const_cast<float*>(a.h) + (size_t)hrow * d, gain, act + (size_t)r * d, d, eps);
  }
}
void launch_plan_norm(bool bf16, const PlanArgs& a, const void* gain, void* act, int d, float eps, int grid,
                      cudaStream_t st) {
  const size_t sm = (size_t)(a.B + 1) * sizeof(int);
  if (bf16)
    launch_k(k_plan_norm<__nv_bfloat16, 256>, grid, 256, sm, st, a, (const __nv_bfloat16*)gain, (__nv_bfloat16*)act, d, eps);
  else launch_k(k_plan_norm<float, 256>, grid, 256, sm, st, a, (const float*)gain, (float*)act, d, eps);
}

// ---------------------------------------------------------------------------
// SIMT GEMM, Y[r][n] = sum_k X[r][k] W[n][k] (fp32 accumulate, k ascending).
// The fp32 model's contraction (tensor-core tf32 would lose the 1e-4 bound).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) k_gemm_simt(const T* __restrict__ X, int ldx, const T* __restrict__ W,
                                                   int N, int K, const int* __restrict__ nrows, float* __restrict__ Y) {
  pdl_wait();
  pdl_launch();
  __shared__ float Xs[16][68];
  __shared__ float Ws[16][68];
  const int R = *nrows;
  const int n0 = blockIdx.x * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int lr = threadIdx.x >> 2, lk = (threadIdx.x & 3) * 4;
  for (int r0 = blockIdx.y * 64; r0 < R; r0 += gridDim.y * 64) {
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int k0 = 0; k0 < K; k0 += 16) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k = k0 + lk + j;
        const int r = r0 + lr, n = n0 + lr;
        Xs[lk + j][lr] = (r < R && k < K) ? ld(X + (size_t)r * ldx + k) : 0.f;
        Ws[lk + j][lr] = (n < N && k < K) ? ld(W + (size_t)n * K + k) : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) {
        float av[4], bv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          av[i] = Xs[kk][ty * 4 + i];
          bv[i] = Ws[kk][tx * 4 + i];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = r0 + ty * 4 + i;
      if (r >= R) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = n0 + tx * 4 + j;
        if (n < N) Y[(size_t)r * N + n] = acc[i][j];
      }
    }
  }
}
void launch_gemm_simt(bool bf16, const void* X, int ldx, const void* W, int N, int K, const int* nrows,
                      int max_rows, float* Y, cudaStream_t st) {
  int gy = (max_rows + 63) / 64;
  if (gy > 64) gy = 64;
  dim3 grid((N + 63) / 64, gy);
  if (bf16)
    launch_k(k_gemm_simt<__nv_bfloat16>, grid, 256, 0, st, (const __nv_bfloat16*)X, ldx, (const __nv_bfloat16*)W, N, K,
                                                     nrows, Y);
  else launch_k(k_gemm_simt<float>, grid, 256, 0, st, (const float*)X, ldx, (const float*)W, N, K, nrows, Y);
}

// ---------------------------------------------------------------------------
// GEMM epilogues (split partial sums added in fixed order)
//   EPI_QKV:    RoPE on q and k (rotate-half pairs), q -> q_out, k and v ->
//               the paged KV cache at the row's position.
//   EPI_RESID:  h[row] += y.
//   EPI_SWIGLU: u = silu(gate) * up, gate/up interleaved in blocks of G rows.
//   EPI_STORE:  out = y.
// ---------------------------------------------------------------------------
// Sum of the split-K slices of one output, in slice order.  All loads are
// issued before the first add (the slices sit in L2; a dependent chain of
// loads would serialise their latency).
__device__ __forceinline__ float epi_sum(const EpiArgs& a, int ns, int r, int n) {
  const float* p = a.Y + (size_t)r * a.N + n;
  float v[TC_MAX_SPLIT];
#pragma unroll
  for (int s = 0; s < TC_MAX_SPLIT; ++s) v[s] = s < ns ? __ldcg(p + s * a.split_stride) : 0.f;
  float y = 0.f;
#pragma unroll
  for (int s = 0; s < TC_MAX_SPLIT; ++s) y += v[s];
  return y;
}

template <typename T>
__global__ void __launch_bounds__(256) k_epilogue(EpiArgs a) {
  pdl_wait();
  pdl_launch();
  const int R = *a.rs.nrows;
  const int ns = a.split_grid ? tc_split_count(R, a.N, a.split_K, a.split_grid, TC_MAX_SPLIT) : 1;
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long tid0 = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (a.mode == EPI_QKV) {
    const int half = a.hd / 2;
    const long long per_row = 3LL * a.H * half;
    for (long long idx = tid0; idx < (long long)R * per_row; idx += stride) {
      const int r = (int)(idx / per_row);
      const int rem = (int)(idx % per_row);
      const int h3 = rem / half, i = rem % half;
      const int part = h3 / a.H, head = h3 % a.H;
      const int c0 = h3 * a.hd + i;
      float y0 = epi_sum(a, ns, r, c0), y1 = epi_sum(a, ns, r, c0 + half);
      const int pos = a.rs.row_pos[r];
      if (part < 2) {
        const float2 u = rope_pair(y0, y1, a.rope[(size_t)pos * half + i]);
        y0 = u.x;
        y1 = u.y;
      }
      if (part == 0) {
        T* q = (T*)a.q_out + (size_t)r * a.H * a.hd + head * a.hd;
        q[i] = cvt<T>(y0);
        q[i + half] = cvt<T>(y1);
      } else {
        T* kv = (T*)a.kv.base + a.kv.offset(a.layer, a.rs.row_b[r], pos, head, part - 1);
        kv[i] = cvt<T>(y0);
        kv[i + half] = cvt<T>(y1);
      }
    }
  } else if (a.mode == EPI_RESID) {
    for (long long idx = tid0; idx < (long long)R * a.N; idx += stride) {
      const int r = (int)(idx / a.N), n = (int)(idx % a.N);
      a.rs.h[(size_t)a.rs.row_hrow[r] * a.d + n] += epi_sum(a, ns, r, n);
    }
  } else if (a.mode == EPI_SWIGLU) {
    for (long long idx = tid0; idx < (long long)R * a.F; idx += stride) {
      const int r = (int)(idx / a.F), j = (int)(idx % a.F);
      const int blk = j / a.G, jj = j % a.G;
      const float g = epi_sum(a, ns, r, blk * 2 * a.G + jj);
      const float u = epi_sum(a, ns, r, blk * 2 * a.G + a.G + jj);
      ((T*)a.u_out)[(size_t)r * a.F + j] = cvt<T>(swiglu(g, u));
    }
  } else {
    for (long long idx = tid0; idx < (long long)R * a.N; idx += stride) {
      const int r = (int)(idx / a.N), n = (int)(idx % a.N);
      a.out[(size_t)r * a.N + n] = epi_sum(a, ns, r, n);
    }
  }
}
void launch_epilogue(bool bf16, const EpiArgs& a, int grid, cudaStream_t st) {
  if (bf16) launch_k(k_epilogue<__nv_bfloat16>, grid, 256, 0, st, a);
  else launch_k(k_epilogue<float>, grid, 256, 0, st, a);
}

// ---------------------------------------------------------------------------
// Paged attention with per-(sequence, layer) cache lengths, SIMT (the fp32
// model's prefill and scoring attention, and the NVIUM_ATTN=simt comparison
// path; bf16 models with head_dim 64 use k_attn_fa_mma).
//
// CTA (b, head, z): z = row group * kv_splits + split.  The row group is up to
// 32 consecutive rows of sequence b (ascending positions p); row p attends
// causally to keys 0..p of this layer, which are either in the cache already
// or were written by this layer's QKV epilogue (the deferred rows of the same
// chunk).  Keys are streamed in tiles of 64 from one page (page_size is a
// multiple of 64); each tile is loaded once and reused by every row of the
// group.  Online softmax in fp32; with kv_splits > 1 the unnormalised
// partials are merged by k_attn_combine in split order.
// ---------------------------------------------------------------------------
template <typename T, int HD>
__global__ void __launch_bounds__(128) k_attention(AttnArgs a) {
  pdl_wait();
  pdl_launch();
  constexpr int NW = 4, RPW = ATTN_RPC / NW, KT = ATTN_KT, DPL = HD / 32;
  __shared__ float Ks[KT][HD + 1];
  __shared__ float Vs[KT][HD];
  __shared__ float Qs[ATTN_RPC][HD];
  const int b = blockIdx.x, head = blockIdx.y, z = blockIdx.z;
  const int rg = z / a.kv_splits, sp = z % a.kv_splits;
  if (*a.rs.nrows == 0) return;
  const int s0 = a.rs.seq_start[b], s1 = a.rs.seq_start[b + 1];
  const int g0 = s0 + rg * ATTN_RPC;
  if (g0 >= s1) return;
  const int g1 = min(s1, g0 + ATTN_RPC), nr = g1 - g0;
  const int pos_last = a.rs.row_pos[g1 - 1];
  const int nt = pos_last / KT + 1;
  const int tps = (nt + a.kv_splits - 1) / a.kv_splits;
  const int t0 = sp * tps, t1 = min(nt, t0 + tps);
  const int H = a.H;
  const T* qg = (const T*)a.q;
  for (int i = threadIdx.x; i < nr * HD; i += blockDim.x) {
    const int r = i / HD, dd = i % HD;
    Qs[r][dd] = ld(qg + (size_t)(g0 + r) * H * HD + head * HD + dd);
  }
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float m[RPW], l[RPW], acc[RPW][DPL];
  int pos[RPW];
#pragma unroll
  for (int j = 0; j < RPW; ++j) {
    const int ri = w + NW * j;
    pos[j] = ri < nr ? a.rs.row_pos[g0 + ri] : -1;
    m[j] = -CUDART_INF_F;
    l[j] = 0.f;
#pragma unroll
    for (int c = 0; c < DPL; ++c) acc[j][c] = 0.f;
  }
  const T* kvb = (const T*)a.kv.base;
  for (int tt = t0; tt < t1; ++tt) {
    const int k0 = tt * KT;
    __syncthreads();
    const T* Kg = kvb + a.kv.offset(a.layer, b, k0, head, 0);
    const T* Vg = kvb + a.kv.offset(a.layer, b, k0, head, 1);
    const int nk = min(KT, pos_last + 1 - k0);
    for (int i = threadIdx.x; i < KT * HD; i += blockDim.x) {
      const int kk = i / HD, dd = i % HD;
      const bool ok = kk < nk;
      Ks[kk][dd] = ok ? ld(Kg + i) : 0.f;
      Vs[kk][dd] = ok ? ld(Vg + i) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < RPW; ++j) {
      const int p = pos[j];
      if (p < k0) continue;
      const int ri = w + NW * j;
      float sa = 0.f, sb = 0.f;
#pragma unroll 8
      for (int dd = 0; dd < HD; ++dd) {
        const float qv = Qs[ri][dd];
        sa = fmaf(qv, Ks[lane][dd], sa);
        sb = fmaf(qv, Ks[lane + 32][dd], sb);
      }
      sa = (k0 + lane <= p) ? sa * a.scale : -CUDART_INF_F;
      sb = (k0 + lane + 32 <= p) ? sb * a.scale : -CUDART_INF_F;
      const float mn = fmaxf(m[j], warp_max(fmaxf(sa, sb)));
      const float corr = expf(m[j] - mn);
      const float pa = expf(sa - mn), pb = expf(sb - mn);
      l[j] = l[j] * corr + warp_sum(pa + pb);
#pragma unroll
      for (int c = 0; c < DPL; ++c) acc[j][c] *= corr;
#pragma unroll 4
      for (int kk = 0; kk < 32; ++kk) {
        const float wa = __shfl_sync(0xffffffffu, pa, kk);
        const float wb = __shfl_sync(0xffffffffu, pb, kk);
#pragma unroll
        for (int c = 0; c < DPL; ++c) {
          acc[j][c] = fmaf(wa, Vs[kk][lane + 32 * c], acc[j][c]);
          acc[j][c] = fmaf(wb, Vs[kk + 32][lane + 32 * c], acc[j][c]);
        }
      }
      m[j] = mn;
    }
  }
#pragma unroll
  for (int j = 0; j < RPW; ++j) {
    const int ri = w + NW * j;
    if (ri >= nr) continue;
    const int r = g0 + ri;
    if (a.kv_splits == 1) {
      const float inv = 1.0f / l[j];
      T* o = (T*)a.o + (size_t)r * H * HD + head * HD;
#pragma unroll
      for (int c = 0; c < DPL; ++c) o[lane + 32 * c] = cvt<T>(acc[j][c] * inv);
    } else {
      float* pp = a.part + (((size_t)r * H + head) * a.kv_splits + sp) * (HD + 2);
#pragma unroll
      for (int c = 0; c < DPL; ++c) pp[lane + 32 * c] = acc[j][c];
      if (lane == 0) {
        pp[HD] = m[j];
        pp[HD + 1] = l[j];
      }
    }
  }
  if (a.lens && head == 0 && sp == 0 && g1 == s1 && threadIdx.x == 0) a.lens[b * a.L + a.layer] = pos_last + 1;
}

template <typename T, int HD>
__global__ void k_attn_combine(AttnArgs a) {
  pdl_wait();
  pdl_launch();
  constexpr int DPL = HD / 32;
  const int R = *a.rs.nrows;
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int item = blockIdx.x * wpb + (threadIdx.x >> 5); item < R * a.H; item += gridDim.x * wpb) {
    const int r = item / a.H, head = item % a.H;
    const float* pp = a.part + ((size_t)r * a.H + head) * a.kv_splits * (HD + 2);
    float M = -CUDART_INF_F;
    for (int s = 0; s < a.kv_splits; ++s) M = fmaxf(M, pp[s * (HD + 2) + HD]);
    float L = 0.f, acc[DPL];
#pragma unroll
    for (int c = 0; c < DPL; ++c) acc[c] = 0.f;
    for (int s = 0; s < a.kv_splits; ++s) {
      const float ms = pp[s * (HD + 2) + HD];
      if (ms == -CUDART_INF_F) continue;
      const float e = expf(ms - M);
      L += pp[s * (HD + 2) + HD + 1] * e;
#pragma unroll
      for (int c = 0; c < DPL; ++c) acc[c] += pp[s * (HD + 2) + lane + 32 * c] * e;
    }
    T* o = (T*)a.o + (size_t)r * a.H * HD + head * HD;
#pragma unroll
    for (int c = 0; c < DPL; ++c) o[lane + 32 * c] = cvt<T>(acc[c] / L);
  }
}

// ---------------------------------------------------------------------------
// Decode attention, SIMT (the fp32 model's and the comparison path; bf16
// models with head_dim 64 use k_attn_dec_mma): CTA (b, head, chunk) handles
// keys [chunk*128, chunk*128 + 128) of sequence b at this layer for every row
// of b whose position reaches the chunk.  One thread issues TMA bulk copies of the chunk's K and V pages
// (each page of one head is contiguous), completing on an mbarrier, so the
// whole 2 x 16 KB chunk is in flight at once.  Scores: one lane per key,
// 16-byte reads of the key row in a per-lane rotated order (conflict-free);
// P.V: one lane per HD/32 dims.  Unnormalised partials (m, l, acc) per
// (row, head, chunk) are merged by k_attn_dec_combine in chunk order.
// Rows of 128 bytes (HD * sizeof(T) == 128) only.
// ---------------------------------------------------------------------------
constexpr int DEC_CK = 128;  // keys per chunk (two 64-position pages)
constexpr int DEC_RG = 8;    // rows per register group in k_attn_dec

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Bounded wait of the whole CTA on an mbarrier phase.  Every thread polls;
// only thread 0 decides that 2 s have passed and says so through `abort`, so
// all threads leave together (after the closing barrier) either way.
__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* status) {
  unsigned long long t0 = 0;
  for (uint32_t i = 0;; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    if (ok) break;
    if ((i & 63u) == 0u) {
      if (threadIdx.x == 0) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        if (i == 0) t0 = t;
        else if (t - t0 > 2000000000ull) *abort = 1;
      }
      if (*abort) break;
    }
  }
  __syncthreads();
  if (*abort) {
    if (threadIdx.x == 0) dev_fail(status, DEV_ERR_TIMEOUT);
    return false;
  }
  return true;
}

template <typename T, int HD>
__global__ void __launch_bounds__(128) k_attn_dec(AttnArgs a) {
  pdl_wait();
  pdl_launch();
  static_assert(HD * sizeof(T) == 128, "128-byte rows");
  constexpr int NW = 4, DPL = HD / 32, EPC = 16 / sizeof(T);
  static_assert(NW * 32 == DEC_CK, "one key per thread");
  __shared__ __align__(128) T Ks[DEC_CK * HD];
  __shared__ __align__(128) T Vs[DEC_CK * HD];
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_abort;
  const int b = blockIdx.x, head = blockIdx.y, chunk = blockIdx.z;
  if (*a.rs.nrows == 0) return;
  const int s0 = a.rs.seq_start[b], s1 = a.rs.seq_start[b + 1];
  if (s0 >= s1) return;
  const int pos_last = a.rs.row_pos[s1 - 1];
  const int k0 = chunk * DEC_CK;
  if (k0 > pos_last) return;
  const int nk = min(DEC_CK, pos_last + 1 - k0);
  const int npages = (nk + a.kv.page_size - 1) / a.kv.page_size;  // page_size == 64 here
  const uint32_t bytes_per_page = (uint32_t)(a.kv.page_size * HD * sizeof(T));
  const T* kvb = (const T*)a.kv.base;
  if (threadIdx.x == 0) {
    s_abort = 0;
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&bar)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(&bar)),
                 "r"(2u * npages * bytes_per_page)
                 : "memory");
    for (int pg = 0; pg < npages; ++pg) {
      const int pos = k0 + pg * a.kv.page_size;
      const T* kg = kvb + a.kv.offset(a.layer, b, pos, head, 0);
      const T* vg = kvb + a.kv.offset(a.layer, b, pos, head, 1);
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
              smem_addr(Ks + pg * a.kv.page_size * HD)),
          "l"(kg), "r"(bytes_per_page), "r"(smem_addr(&bar))
          : "memory");
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
              smem_addr(Vs + pg * a.kv.page_size * HD)),
          "l"(vg), "r"(bytes_per_page), "r"(smem_addr(&bar))
          : "memory");
    }
  }
  __syncthreads();
  if (!bounded_wait(&bar, 0, &s_abort, a.status)) return;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = a.H;
  const T* qg = (const T*)a.q;
  // rows of b whose position reaches this chunk: positions are contiguous.
  // Warp w takes keys [32w, 32w+32) of the chunk (one key per lane) for up to
  // DEC_RG rows at a time, keeping each row's softmax state in registers;
  // the four warps merge once per row group.
  const int pos0 = a.rs.row_pos[s0];
  const int first = max(s0, s0 + (k0 - pos0));
  __shared__ float Qr[DEC_RG][HD];
  __shared__ float Wst[NW][DEC_RG][HD + 2];
  const int kk = 32 * w + lane;
  const uint4* krow = (const uint4*)(Ks + kk * HD);
  for (int g0 = first; g0 < s1; g0 += DEC_RG) {
    const int ng = min(DEC_RG, s1 - g0);
    for (int i = threadIdx.x; i < ng * HD; i += blockDim.x)
      Qr[i / HD][i % HD] = ld(qg + (size_t)(g0 + i / HD) * H * HD + head * HD + i % HD);
    __syncthreads();
    // this lane's key, once, as eight 16-byte chunks read in a per-lane
    // rotated order (conflict-free); kc[c8] holds chunk (c8 + lane) % 8
    uint4 kc[8];
#pragma unroll
    for (int c8 = 0; c8 < 8; ++c8) kc[c8] = krow[(c8 + lane) & 7];
#pragma unroll 1
    for (int j = 0; j < ng; ++j) {
      const int p = pos0 + (g0 + j - s0);
      float sc = -CUDART_INF_F;
      if (kk < nk && k0 + kk <= p) {
        float acc = 0.f;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          const float* qc = &Qr[j][((c8 + lane) & 7) * EPC];
          const T* kp = (const T*)&kc[c8];
#pragma unroll
          for (int e = 0; e < EPC; ++e) acc = fmaf(qc[e], ld(kp + e), acc);
        }
        sc = acc * a.scale;
      }
      const float mw = warp_max(sc);
      float o[DPL];
#pragma unroll
      for (int d = 0; d < DPL; ++d) o[d] = 0.f;
      float lw = 0.f;
      if (mw != -CUDART_INF_F) {
        const float pk = expf(sc - mw);
        lw = warp_sum(pk);
        const int kmax = min(32, min(nk, p + 1 - k0) - 32 * w);
#pragma unroll 8
        for (int src = 0; src < 32; ++src) {
          const float pw = __shfl_sync(0xffffffffu, pk, src);
          if (src >= kmax) break;  // rows past the row's keys hold stale data
          const T* vrow = Vs + (32 * w + src) * HD + lane * DPL;
#pragma unroll
          for (int d = 0; d < DPL; ++d) o[d] = fmaf(pw, ld(vrow + d), o[d]);
        }
      }
#pragma unroll
      for (int d = 0; d < DPL; ++d) Wst[w][j][lane * DPL + d] = o[d];
      if (lane == 0) {
        Wst[w][j][HD] = mw;
        Wst[w][j][HD + 1] = lw;
      }
    }
    __syncthreads();
    for (int j = w; j < ng; j += NW) {
      float M = -CUDART_INF_F;
#pragma unroll
      for (int q = 0; q < NW; ++q) M = fmaxf(M, Wst[q][j][HD]);
      float L = 0.f, acc[DPL];
#pragma unroll
      for (int d = 0; d < DPL; ++d) acc[d] = 0.f;
#pragma unroll
      for (int q = 0; q < NW; ++q) {
        const float mq = Wst[q][j][HD];
        if (mq == -CUDART_INF_F) continue;
        const float e = expf(mq - M);
        L += Wst[q][j][HD + 1] * e;
#pragma unroll
        for (int d = 0; d < DPL; ++d) acc[d] += Wst[q][j][lane * DPL + d] * e;
      }
      float* pp = a.part + (((size_t)(g0 + j) * H + head) * a.kv_splits + chunk) * (HD + 2);
#pragma unroll
      for (int d = 0; d < DPL; ++d) pp[lane * DPL + d] = acc[d];
      if (lane == 0) {
        pp[HD] = M;
        pp[HD + 1] = L;
      }
    }
    __syncthreads();
  }
  if (a.lens && head == 0 && chunk == 0 && threadIdx.x == 0) a.lens[b * a.L + a.layer] = pos_last + 1;
}

// Merge the chunk partials of each (row, head): chunks 0 .. pos/128.
template <typename T, int HD>
__global__ void k_attn_dec_combine(AttnArgs a) {
  pdl_wait();
  pdl_launch();
  constexpr int DPL = HD / 32;
  const int R = *a.rs.nrows;
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  for (int item = blockIdx.x * wpb + (threadIdx.x >> 5); item < R * a.H; item += gridDim.x * wpb) {
    const int r = item / a.H, head = item % a.H;
    const int nch = a.rs.row_pos[r] / DEC_CK + 1;
    const float* pp = a.part + ((size_t)r * a.H + head) * a.kv_splits * (HD + 2);
    float M = -CUDART_INF_F;
    for (int c = 0; c < nch; ++c) M = fmaxf(M, pp[c * (HD + 2) + HD]);
    float L = 0.f, acc[DPL];
#pragma unroll
    for (int d = 0; d < DPL; ++d) acc[d] = 0.f;
    for (int c = 0; c < nch; ++c) {
      const float e = expf(pp[c * (HD + 2) + HD] - M);
      L += pp[c * (HD + 2) + HD + 1] * e;
#pragma unroll
      for (int d = 0; d < DPL; ++d) acc[d] += pp[c * (HD + 2) + lane * DPL + d] * e;
    }
    T* o = (T*)a.o + (size_t)r * a.H * HD + head * HD;
    const float inv = 1.0f / L;
#pragma unroll
    for (int d = 0; d < DPL; ++d) o[lane * DPL + d] = cvt<T>(acc[d] * inv);
  }
}

template <typename T, int HD>
static void attention_dec_t(const AttnArgs& a, cudaStream_t st) {
  int g = (a.rs.max_rows * a.H + 7) / 8;
  if (g > 4096) g = 4096;
  if (sizeof(T) == 2 && HD == 64 && attn_dec_pc_fits(a)) {
    launch_attn_dec_pc(a, st);
    return;
  }
  if (a.kv_map && sizeof(T) == 2 && HD == 64) {
    AttnArgs m = a;
    m.kv_splits = a.dec_splits;
    launch_attn_dec_mma(a.kv_map, m, st);
    return;
  }
  dim3 grid(a.rs.B, a.H, a.kv_splits);
  launch_k(k_attn_dec<T, HD>, grid, 128, 0, st, a);
  launch_k(k_attn_dec_combine<T, HD>, g, 256, 0, st, a);
}
void launch_attention_decode(bool bf16, const AttnArgs& a, cudaStream_t st) {
  if (bf16) attention_dec_t<__nv_bfloat16, 64>(a, st);
  else attention_dec_t<float, 32>(a, st);
}
int attention_decode_launches(bool bf16, const AttnArgs& a) {
  if (bf16 && a.kv_map) return 1;
  return 2;
}

template <typename T, int HD>
static void attention_t(const AttnArgs& a, cudaStream_t st) {
  dim3 grid(a.rs.B, a.H, a.row_groups * a.kv_splits);
  launch_k(k_attention<T, HD>, grid, 128, 0, st, a);
  if (a.kv_splits > 1) {
    int g = (a.rs.max_rows * a.H + 7) / 8;
    if (g > 4096) g = 4096;
    launch_k(k_attn_combine<T, HD>, g, 256, 0, st, a);
  }
}
void launch_attention(bool bf16, const AttnArgs& a, cudaStream_t st) {
  if (bf16 && a.hd == 64 && a.kv_map && a.kv_splits == 1 && a.rs.B <= 65535) {
    if (a.q_map) launch_attn_fa_tc(a.kv_map, a.q_map, a, st);
    else launch_attn_fa_mma(a.kv_map, a, st);
    return;
  }
  if (a.hd == 64) {
    if (bf16) attention_t<__nv_bfloat16, 64>(a, st); else attention_t<float, 64>(a, st);
  } else {
    if (bf16) attention_t<__nv_bfloat16, 32>(a, st); else attention_t<float, 32>(a, st);
  }
}

// ---------------------------------------------------------------------------
// Decode step begin / end
// ---------------------------------------------------------------------------
template <typename T>
__global__ void k_step_begin(StepArgs a) {
  pdl_wait();
  pdl_launch();
  const int b = blockIdx.x;
  const int tb = a.t[b];
  if (threadIdx.x == 0) {
    a.active[b] = 1;
    a.exit_id[b] = 0;
    // a sequence whose deferred store would overflow completes its deferred
    // rows in this step (the values do not change, only when they are made)
    const int pending = tb - a.lens[b * a.L + a.L - 1];
    const int f = (pending + 1 >= a.cap) ? 1 : 0;
    a.force[b] = f;
    if (f && a.counters) atomicAdd((unsigned long long*)&a.counters[NV_CTR_FORCED], 1ull);
    for (int k = 0; k < a.n_exits; ++k) {
      a.stop[k * a.B + b] = 0;
      a.router_p[k * a.B + b] = CUDART_NAN_F;
    }
    if (b == 0) {
      *a.seed_dev = a.seed;
      for (int k = 0; k < a.n_exits; ++k) a.nstop[k] = 0;
    }
  }
  const T* e = (const T*)a.emb + (size_t)a.tok[b] * a.d;
  float* h = a.hbuf + ((size_t)b * a.cap + tb % a.cap) * a.d;
  for (int i = threadIdx.x; i < a.d; i += blockDim.x) h[i] = ld(e + i);
}
void launch_step_begin(bool bf16, const StepArgs& a, cudaStream_t st) {
  if (bf16) launch_k(k_step_begin<__nv_bfloat16>, a.B, 256, 0, st, a);
  else launch_k(k_step_begin<float>, a.B, 256, 0, st, a);
}

__global__ void k_step_end(StepArgs a) {
  pdl_wait();
  pdl_launch();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b == 0 && a.counters) atomicAdd((unsigned long long*)&a.counters[NV_CTR_STEPS], 1ull);
  if (b >= a.B) return;
  const int tokn = a.sampled[b];
  a.out_tok[b] = tokn;
  a.out_exit[b] = a.exit_id[b];
  a.tok[b] = tokn;
  a.t[b] += 1;
}
void launch_step_end(const StepArgs& a, cudaStream_t st) {
  launch_k(k_step_end, (a.B + 255) / 256, 256, 0, st, a);
}

// ---------------------------------------------------------------------------
// Exit junction k (section 2 "Architektur": router w_k, stop/continue).
// n_k = RMSNorm_k(h) (rounded to the model dtype), z = r_k . n_k + b_k or,
// with a router MLP of width r, z = v . silu(U n_k + c) + b_k;
// w_k = sigmoid(z) (0 when routing is forced to the last exit), and the token
// stops here iff u_k < w_k; the last exit always stops.  u_k is the Philox
// uniform of counter (b, t, 0, k/4), lane k%4 (k 0-based).
// ---------------------------------------------------------------------------
// Router MLP of one row, by one warp over the hidden units j = j0, j0 + dj,
// ...: returns this warp's share of sum_j v_j silu(U_j . n + c_j) (in every
// lane); n is the row's exit-normalised state in the model dtype.
template <typename T>
__device__ __forceinline__ float router_mlp_part(const T* __restrict__ n, const T* __restrict__ U,
                                                 const float* __restrict__ c, const float* __restrict__ v, int d,
                                                 int r, int j0, int dj) {
  const int lane = threadIdx.x & 31;
  float z = 0.f;
  for (int j = j0; j < r; j += dj) {
    const T* u = U + (size_t)j * d;
    float a = 0.f;
    for (int i = lane; i < d; i += 32) a = fmaf(ld(n + i), ld(u + i), a);
    a = warp_sum(a) + c[j];
    z = fmaf(v[j], a / (1.0f + expf(-a)), z);
  }
  return z;
}

template <typename T>
__global__ void __launch_bounds__(256) k_junction(JuncArgs a) {
  pdl_wait();
  pdl_launch();
  const int b = blockIdx.x;
  if (!a.active[b]) return;
  const int tb = a.t[b];
  const float* h = a.hbuf + ((size_t)b * a.cap + tb % a.cap) * a.d;
  const T* g = (const T*)a.norm;
  const bool last = a.k == a.n_exits - 1;
  float ss = 0.f;
  for (int i = threadIdx.x; i < a.d; i += 256) ss = fmaf(h[i], h[i], ss);
  ss = block_sum<256>(ss);
  const float inv = 1.0f / sqrtf(ss / (float)a.d + a.eps);
  T* out = (T*)a.exit_act + (size_t)b * a.d;
  const T* rw = (const T*)a.router_w;
  float z = 0.f;
  for (int i = threadIdx.x; i < a.d; i += 256) {
    const float n = rnd<T>(h[i] * inv * ld(g + i));
    out[i] = cvt<T>(n);
    if (!last) z = fmaf(n, ld(rw + i), z);
  }
  if (!last && a.router_hidden > 0) {
    // every thread's n_k is in exit_act: the eight warps split the hidden units
    __syncthreads();
    const float zp = router_mlp_part<T>(out, (const T*)a.router_w1, a.router_b1, a.router_w2, a.d, a.router_hidden,
                                        threadIdx.x >> 5, 8);
    z = (threadIdx.x & 31) == 0 ? zp : 0.f;
  }
  z = block_sum<256>(z);
  if (threadIdx.x == 0) {
    bool stop = true;
    if (!last) {
      const float w = (a.router_mode == NV_ROUTER_FORCE_LAST) ? 0.f : 1.0f / (1.0f + expf(-(z + a.router_b)));
      a.router_p[b] = w;
      const unsigned long long seed = *a.seed;
      const uint4 r = philox4x32_10(make_uint4((uint32_t)b, (uint32_t)tb, STREAM_EXIT, (uint32_t)(a.k / 4)),
                                    (uint32_t)seed, (uint32_t)(seed >> 32));
      const float u = uniform01(lane_of(r, a.k % 4));
      stop = u < w;
    }
    if (stop) {
      a.active[b] = 0;
      a.exit_id[b] = a.k + 1;
      a.stop[b] = 1;
      const int before = atomicAdd(a.nstop, 1);
      if (a.counters) {
        atomicAdd((unsigned long long*)&a.counters[NV_CTR_EXIT0 + a.k], 1ull);
        if (before == 0) atomicAdd((unsigned long long*)&a.counters[NV_CTR_HEAD_BYTES], (unsigned long long)a.head_bytes);
      }
    }
  }
}
void launch_junction(bool bf16, const JuncArgs& a, cudaStream_t st) {
  if (bf16) launch_k(k_junction<__nv_bfloat16>, a.B, 256, 0, st, a);
  else launch_k(k_junction<float>, a.B, 256, 0, st, a);
}

// ---------------------------------------------------------------------------
// Exit adapter (section 2 "Architektur": all exits share the final LM head,
// light adapter MLPs map the intermediate states to its geometry).  One CTA
// per sequence that stopped here: hidden = silu(W1 n_k) (rounded to the model
// dtype: it multiplies W2), m = h + W2 hidden (fp32), head input = final
// RMSNorm of m.  Shared memory: hidden [a] and m [d].
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) k_exit_adapter(AdapterArgs p) {
  pdl_wait();
  pdl_launch();
  const int b = blockIdx.x;
  if (!p.stop[b]) return;
  extern __shared__ float s_ad[];
  float* s_hid = s_ad;
  float* s_m = s_ad + p.a;
  T* x = (T*)p.exit_act + (size_t)b * p.d;
  const float* h = p.hbuf + ((size_t)b * p.cap + p.t[b] % p.cap) * p.d;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int j = w; j < p.a; j += 8) {
    const T* u = (const T*)p.w1 + (size_t)j * p.d;
    float acc = 0.f;
    for (int i = lane; i < p.d; i += 32) acc = fmaf(ld(x + i), ld(u + i), acc);
    acc = warp_sum(acc);
    if (lane == 0) s_hid[j] = rnd<T>(acc / (1.0f + expf(-acc)));
  }
  __syncthreads();
  float ss = 0.f;
  for (int i = threadIdx.x; i < p.d; i += 256) {
    const T* v = (const T*)p.w2 + (size_t)i * p.a;
    float o = 0.f;
    for (int j = 0; j < p.a; ++j) o = fmaf(ld(v + j), s_hid[j], o);
    const float m = h[i] + o;
    s_m[i] = m;
    ss = fmaf(m, m, ss);
  }
  ss = block_sum<256>(ss);
  const float inv = 1.0f / sqrtf(ss / (float)p.d + p.eps);
  const T* g = (const T*)p.final_norm;
  for (int i = threadIdx.x; i < p.d; i += 256) x[i] = cvt<T>(rnd<T>(s_m[i] * inv * ld(g + i)));
}
void launch_exit_adapter(bool bf16, const AdapterArgs& a, cudaStream_t st) {
  const size_t sm = (size_t)(a.a + a.d) * sizeof(float);
  if (bf16) launch_k(k_exit_adapter<__nv_bfloat16>, a.B, 256, sm, st, a);
  else launch_k(k_exit_adapter<float>, a.B, 256, sm, st, a);
}
cudaError_t exit_adapter_prepare(bool bf16, int d, int a) {
  const size_t sm = (size_t)(a + d) * sizeof(float);
  if (sm <= 48 * 1024) return cudaSuccess;
  return bf16 ? cudaFuncSetAttribute(k_exit_adapter<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)
              : cudaFuncSetAttribute(k_exit_adapter<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
}

template <typename T>
__global__ void k_silu_rows(const int* __restrict__ nrows, const float* __restrict__ Y, int a, T* __restrict__ u) {
  pdl_wait();
  pdl_launch();
  const size_t n = (size_t)(*nrows) * a;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const float y = Y[i];
    u[i] = cvt<T>(rnd<T>(y / (1.0f + expf(-y))));
  }
}
void launch_silu_rows(bool bf16, const int* nrows, const float* Y, int a, void* u, int max_rows, cudaStream_t st) {
  long long g = ((long long)max_rows * a + 255) / 256;
  const int grid = (int)(g < 4096 ? (g < 1 ? 1 : g) : 4096);
  if (bf16) launch_k(k_silu_rows<__nv_bfloat16>, grid, 256, 0, st, nrows, Y, a, (__nv_bfloat16*)u);
  else launch_k(k_silu_rows<float>, grid, 256, 0, st, nrows, Y, a, (float*)u);
}

template <typename T>
__global__ void k_adapter_norm_rows(RowSet rs, const float* __restrict__ Y, const T* __restrict__ g,
                                    T* __restrict__ act, int d, float eps) {
  pdl_wait();
  pdl_launch();
  const int R = *rs.nrows;
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  for (int r = blockIdx.x * wpb + (threadIdx.x >> 5); r < R; r += gridDim.x * wpb) {
    const float* h = rs.h + (size_t)rs.row_hrow[r] * d;
    const float* y = Y + (size_t)r * d;
    float ss = 0.f;
    for (int i = lane; i < d; i += 32) {
      const float m = h[i] + y[i];
      ss = fmaf(m, m, ss);
    }
    ss = warp_sum(ss);
    const float inv = 1.0f / sqrtf(ss / (float)d + eps);
    for (int i = lane; i < d; i += 32) act[(size_t)r * d + i] = cvt<T>(rnd<T>((h[i] + y[i]) * inv * ld(g + i)));
  }
}
void launch_adapter_norm_rows(bool bf16, RowSet rs, const float* Y, const void* final_norm, void* act, int d,
                              float eps, cudaStream_t st) {
  int grid = (rs.max_rows + 7) / 8;
  if (grid > 2048) grid = 2048;
  if (bf16)
    launch_k(k_adapter_norm_rows<__nv_bfloat16>, grid, 256, 0, st, rs, Y, (const __nv_bfloat16*)final_norm,
             (__nv_bfloat16*)act, d, eps);
  else launch_k(k_adapter_norm_rows<float>, grid, 256, 0, st, rs, Y, (const float*)final_norm, (float*)act, d, eps);
}

// ---------------------------------------------------------------------------
// Fused exit-head sampler (exact sampling, section 3; Gumbel-max reading),
// for the batches the tensor-core head does not take.  For the rows that
// stopped at exit k: logit_v = W_k[v] . n_k, score_v = logit_v + Gumbel(U_v)
// with U_v from counter (b, t, 1, v/4) lane v%4, running argmax (ties to the
// lowest v) and online log-sum-exp of the logits.  Logits never leave the
// chip; each CTA writes one partial per row, merged by k_head_reduce in CTA
// order.
//
// One CTA per SM streams a contiguous range of head rows (a multiple of four,
// the rows of one Philox draw) through a shared-memory ring: a producer
// thread copies HS_ROWS rows per stage with one bulk copy (cp.async.bulk,
// completion counted on the stage's mbarrier).  The consumer warps form two
// teams that take alternate stages; in a stage, warp q of the team takes the
// q-th group of four rows: one Philox draw serves the group, the four dot
// products share each activation chunk and run as independent chains, and
// the stage goes back to the producer as soon as the rows are in registers.
// A warp draws the Gumbel noise of its next groups together (one lane per
// stopped row, group and row of the group), and the four lanes 4r'+j keep
// stopped row r's running argmax and log-sum-exp over the rows v = j mod 4,
// merged once at the end.  Stopped rows beyond one pass (rp rows, at most
// HS_RP) are taken in further passes over the same range.
// ---------------------------------------------------------------------------
constexpr int HS_TEAM = 4;                       // warps per team: the groups of a stage
constexpr int HS_WARPS = 2 * HS_TEAM;            // consumer warps
constexpr int HS_THREADS = 32 * (HS_WARPS + 1);  // + one producer warp
constexpr int HS_ROWS = 4 * HS_TEAM;             // head rows per stage
constexpr int HS_MAX_STAGES = 8;
constexpr int HS_MAXC = 8;                       // 16-byte chunks of a row per lane (d * size <= 4096 bytes)
constexpr int HS_RP = 16;                        // stopped rows per pass
constexpr int HS_SLOTS = HS_RP / 8;              // running states per lane (8 rows x 4 lanes per slot)
constexpr size_t HS_DYN_MAX = 208 * 1024;        // dynamic shared memory of one CTA

struct HeadPlan {
  int rp = 0, stages = 0;
  size_t act_off = 0, ring_off = 0, bytes = 0;
};
// list of stopped rows [B] | rp activation rows | ring of `stages` x HS_ROWS head rows
static HeadPlan head_plan(int B, int d, size_t esz) {
  HeadPlan p;
  const size_t rowb = (size_t)d * esz, stage = HS_ROWS * rowb;
  auto al = [](size_t x) { return (x + 127) / 128 * 128; };
  p.act_off = al((size_t)B * 4);
  if (rowb % 16 || rowb > 16 * 32 * HS_MAXC || p.act_off + rowb + 2 * stage > HS_DYN_MAX) return HeadPlan{};
  size_t rp = (size_t)(B < HS_RP ? B : HS_RP);
  const size_t rp_fit = (HS_DYN_MAX - p.act_off - 2 * stage) / rowb;
  if (rp > rp_fit) rp = rp_fit;
  p.rp = (int)rp;
  p.ring_off = al(p.act_off + rp * rowb);
  size_t ns = (HS_DYN_MAX - p.ring_off) / stage;
  if (ns > HS_MAX_STAGES) ns = HS_MAX_STAGES;
  p.stages = (int)ns;
  p.bytes = p.ring_off + ns * stage;
  return p;
}
bool head_sample_fits(int B, int d, size_t esz) { return head_plan(B, d, esz).stages >= 2; }

__device__ __forceinline__ void hs_bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_addr(dst)),
               "l"(src), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
}
__device__ __forceinline__ bool hs_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait of one thread on an mbarrier phase: false when 2 s passed
// (the thread raises `abort` and the device error word) or another thread
// raised `abort`.
__device__ __forceinline__ bool hs_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* status,
                                        unsigned long long limit_ns = 2000000000ull) {
  if (hs_try_wait(bar, parity)) return true;
  unsigned long long t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  for (uint32_t i = 1;; ++i) {
    if (hs_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0u) {
      if (*abort) return false;
      unsigned long long t;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
      if (t - t0 > limit_ns) {
        *abort = 1;
        dev_fail(status, DEV_ERR_TIMEOUT);
        return false;
      }
    }
  }
}
// c + w.lo * a.lo, then + w.hi * a.hi for two packed bf16 pairs: each step
// one fused multiply-add of two bf16 values into fp32 (their product is exact
// in fp32), so the result equals fmaf on the converted values
__device__ __forceinline__ float fma_bf16x2_seq(uint32_t w, uint32_t a, float c) {
  asm("{\n\t.reg .b16 wl, wh, al, ah;\n\tmov.b32 {wl, wh}, %1;\n\tmov.b32 {al, ah}, %2;\n\t"
      "fma.rn.f32.bf16 %0, wl, al, %0;\n\tfma.rn.f32.bf16 %0, wh, ah, %0;\n\t}"
      : "+f"(c)
      : "r"(w), "r"(a));
  return c;
}
// one head row into a stopped row's running state: argmax of the Gumbel
// score (rows arrive in increasing v, so the first maximum is kept) and the
// online log-sum-exp of the logits
__device__ __forceinline__ void hs_update(float sc, float logit, int v, float& best_s, int& best_v, float& best_l,
                                          float& mx, float& se) {
  if (sc > best_s) {
    best_s = sc;
    best_v = v;
    best_l = logit;
  }
  if (logit > mx) {
    se = se * expf(mx - logit) + 1.0f;
    mx = logit;
  } else {
    se += expf(logit - mx);
  }
}
// barrier of the consumer warps only (the producer warp keeps streaming)
__device__ __forceinline__ void hs_cbar() { asm volatile("bar.sync 1, %0;" ::"r"(HS_WARPS * 32) : "memory"); }
__device__ __forceinline__ bool hs_cbar_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\tbar.red.or.pred p, 1, %2, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(HS_WARPS * 32)
      : "memory");
  return r != 0;
}

// MAXC: 16-byte chunks of a head row per lane (a row is 32 * MAXC chunks at most)
template <typename T, int MAXC>
__global__ void __launch_bounds__(HS_THREADS, 1) k_head_sample(HeadArgs a) {
  pdl_wait();
  pdl_launch();
  constexpr int EPC = 16 / sizeof(T);
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ float s_part[HS_WARPS][HS_RP][HEAD_PART];
  __shared__ float s_gm[HS_WARPS][4 * HS_RP];  // Gumbel noise of a warp's next groups
  __shared__ int s_b[HS_RP], s_t[HS_RP];
  __shared__ __align__(8) uint64_t s_full[HS_MAX_STAGES], s_empty[HS_MAX_STAGES];
  __shared__ int s_n;
  __shared__ volatile int s_abort;
  int* s_list = (int*)smem;                          // [B]
  T* s_act = (T*)(smem + a.act_off);                 // [rp][d]
  T* ring = (T*)(smem + a.ring_off);                 // [stages][HS_ROWS][d]
  const int B = a.B, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int d = a.d, V = a.V, NS = a.stages, RP = a.rp;
  // compact the rows that stopped here, in sequence order
  if (w == 0) {
    int n = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int b = b0 + lane;
      const bool st = b < B && a.stop[b] != 0;
      const unsigned m = __ballot_sync(0xffffffffu, st);
      if (st) s_list[n + __popc(m & ((1u << lane) - 1u))] = b;
      n += __popc(m);
    }
    if (lane == 0) {
      s_n = n;
      s_abort = 0;
      for (int s = 0; s < NS; ++s) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&s_full[s])) : "memory");
        asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(&s_empty[s])), "r"(HS_TEAM)
                     : "memory");
      }
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
  }
  __syncthreads();
  const int n = s_n;
  if (n == 0) return;
  // this CTA's head rows [rbeg, rend): whole groups of four
  const int groups = (V + 3) / 4;
  const int gpc = (groups + gridDim.x - 1) / gridDim.x;
  const int rbeg = min(V, (int)blockIdx.x * gpc * 4), rend = min(V, rbeg + gpc * 4);
  const int nst = (rend - rbeg + HS_ROWS - 1) / HS_ROWS;  // stages per pass
  const int passes = (n + RP - 1) / RP;
  if (w == HS_WARPS) {
    // producer: the same stage sequence, pass after pass
    if (lane != 0) return;
    const T* head = (const T*)a.head;
    int i = 0;
    bool ok = true;
    for (int p = 0; p < passes && ok; ++p) {
      for (int s = 0; s < nst; ++s, ++i) {
        const int slot = i % NS;
        if (i >= NS && !hs_wait(&s_empty[slot], (uint32_t)((i / NS - 1) & 1), &s_abort, a.status)) {
          ok = false;
          break;
        }
        const int r0 = rbeg + s * HS_ROWS, nr = min(HS_ROWS, rend - r0);
        const uint32_t bytes = (uint32_t)((size_t)nr * d * sizeof(T));
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(&s_full[slot])),
                     "r"(bytes)
                     : "memory");
        hs_bulk_load(ring + (size_t)slot * HS_ROWS * d, head + (size_t)r0 * d, bytes, &s_full[slot]);
      }
    }
    // no copy may still be landing when the CTA's shared memory goes: wait
    // (bounded) for the last stages issued; after a normal run the consumers
    // have already seen them complete
    int never = 0;
    for (int j = max(0, i - NS); j < i; ++j)
      hs_wait(&s_full[j % NS], (uint32_t)((j / NS) & 1), &never, nullptr, 100000000ull);
    return;
  }
  // consumers
  const int nchunk = d / EPC;  // 16-byte chunks per row
  const unsigned long long seed = *a.seed;
  int i = 0;  // stage sequence number, as the producer counts it
  for (int p0 = 0; p0 < n; p0 += RP) {
    const int nr = min(RP, n - p0);
    hs_cbar();  // the previous pass's rows and partials are no longer read
    for (int x = tid; x < nr * nchunk; x += HS_WARPS * 32) {
      const int r = x / nchunk, c = x % nchunk;
      ((uint4*)s_act)[(size_t)r * nchunk + c] = ((const uint4*)((const T*)a.exit_act + (size_t)s_list[p0 + r] * d))[c];
    }
    if (tid < nr) {
      s_b[tid] = s_list[p0 + tid];
      s_t[tid] = a.t[s_list[p0 + tid]];
    }
    hs_cbar();
    // Lane 4r' + j keeps the running state of stopped row r = 8t + r' (slot t)
    // over this warp's rows v with v % 4 == j.
    float best_s[HS_SLOTS], best_l[HS_SLOTS], mx[HS_SLOTS], se[HS_SLOTS];
    int best_v[HS_SLOTS];
#pragma unroll
    for (int t = 0; t < HS_SLOTS; ++t) {
      best_s[t] = -CUDART_INF_F;
      best_l[t] = 0.f;
      mx[t] = -CUDART_INF_F;
      se[t] = 0.f;
      best_v[t] = 0x7fffffff;
    }
    bool ok = true;
    const int team = w / HS_TEAM, q = w % HS_TEAM;
    const int jl = lane & 3, rl = lane >> 2;
    // Gumbel noise is drawn for G of this warp's groups at a time (its stages
    // s, s + 2, ...): entry (k, r, j), one Philox draw per (stopped row,
    // group), is computed by lane (k nr + r) 4 + j (+ 32 per round)
    const int G = nr <= 8 ? 8 / nr : 1;
    int kg = 0;  // this warp's groups so far in the pass
    for (int s = 0; s < nst; ++s, ++i) {
      if ((i & 1) != team) continue;
      const int slot = i % NS;
      const int v0 = rbeg + s * HS_ROWS + 4 * q;  // this warp's group: rows v0 .. v0 + nv - 1
      const int nv = min(4, rend - v0);
      const int kb = kg % G;
      ++kg;
      if (kb == 0) {
        __syncwarp();  // the previous batch has been read
        for (int x = lane; x < 4 * nr * G; x += 32) {
          const int k = x / (4 * nr), r = (x >> 2) % nr, j = x & 3;
          const int s2 = s + 2 * k, v = rbeg + s2 * HS_ROWS + 4 * q + j;
          float g = 0.f;
          if (s2 < nst && v < rend) {
            const uint4 rb = philox4x32_10(
                make_uint4((uint32_t)s_b[r], (uint32_t)s_t[r], STREAM_GUMBEL, (uint32_t)(v >> 2)), (uint32_t)seed,
                (uint32_t)(seed >> 32));
            g = -logf(-logf(uniform01(lane_of(rb, j))));
          }
          s_gm[w][x] = g;
        }
        __syncwarp();
      }
      // lane 0 waits, the warp follows its verdict
      int got = 1;
      if (lane == 0) got = hs_wait(&s_full[slot], (uint32_t)((i / NS) & 1), &s_abort, a.status) ? 1 : 0;
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) {
        ok = false;
        break;
      }
      uint4 wv[4][MAXC];
      if (nv > 0) {
        const uint4* wrow = (const uint4*)(ring + ((size_t)slot * HS_ROWS + 4 * q) * d);
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int c = 0; c < MAXC; ++c)
            if (j < nv && lane + 32 * c < nchunk) wv[j][c] = wrow[(size_t)j * nchunk + lane + 32 * c];
      }
      // the rows are in registers: hand the stage back
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(&s_empty[slot])) : "memory");
      if (nv <= 0) continue;
      for (int r = 0; r < nr; ++r) {
        const uint4* arow = (const uint4*)s_act + (size_t)r * nchunk;
        float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < MAXC; ++c) {
          if (lane + 32 * c < nchunk) {
            const uint4 av = arow[lane + 32 * c];
            if constexpr (sizeof(T) == 2) {
              const uint32_t* aw = (const uint32_t*)&av;
#pragma unroll
              for (int k = 0; k < 4; ++k)
#pragma unroll
                for (int j = 0; j < 4; ++j) part[j] = fma_bf16x2_seq(((const uint32_t*)&wv[j][c])[k], aw[k], part[j]);
            } else {
              const T* ap = (const T*)&av;
#pragma unroll
              for (int e = 0; e < EPC; ++e) {
                const float x = ld(ap + e);
#pragma unroll
                for (int j = 0; j < 4; ++j) part[j] = fmaf(ld((const T*)&wv[j][c] + e), x, part[j]);
              }
            }
          }
        }
        // four butterflies, interleaved: every lane ends with the four sums
#pragma unroll
        for (int o = 16; o; o >>= 1)
#pragma unroll
          for (int j = 0; j < 4; ++j) part[j] += __shfl_xor_sync(0xffffffffu, part[j], o);
        if (rl == (r & 7) && jl < nv) {
          const float logit = jl == 0 ? part[0] : jl == 1 ? part[1] : jl == 2 ? part[2] : part[3];
          const float sc = logit + s_gm[w][(kb * nr + r) * 4 + jl];
          static_assert(HS_SLOTS == 2, "two state slots");
          if (r < 8) hs_update(sc, logit, v0 + jl, best_s[0], best_v[0], best_l[0], mx[0], se[0]);
          else hs_update(sc, logit, v0 + jl, best_s[1], best_v[1], best_l[1], mx[1], se[1]);
        }
      }
    }
    // every consumer leaves together when any of them gave up
    if (hs_cbar_or(!ok || s_abort)) return;
    // the four lanes of a stopped row merge (argmax ties to the lowest v)
#pragma unroll
    for (int t = 0; t < HS_SLOTS; ++t) {
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) {
        const float bs2 = __shfl_xor_sync(0xffffffffu, best_s[t], o);
        const int bv2 = __shfl_xor_sync(0xffffffffu, best_v[t], o);
        const float bl2 = __shfl_xor_sync(0xffffffffu, best_l[t], o);
        const float m2 = __shfl_xor_sync(0xffffffffu, mx[t], o);
        const float s2 = __shfl_xor_sync(0xffffffffu, se[t], o);
        if (bs2 > best_s[t] || (bs2 == best_s[t] && bv2 < best_v[t])) {
          best_s[t] = bs2;
          best_v[t] = bv2;
          best_l[t] = bl2;
        }
        const float mn = fmaxf(mx[t], m2);
        if (mn != -CUDART_INF_F) {
          se[t] = (mx[t] == -CUDART_INF_F ? 0.f : se[t] * expf(mx[t] - mn)) +
                  (m2 == -CUDART_INF_F ? 0.f : s2 * expf(m2 - mn));
          mx[t] = mn;
        }
      }
      const int r = 8 * t + rl;
      if (jl == 0 && r < nr) {
        s_part[w][r][0] = best_s[t];
        s_part[w][r][1] = __int_as_float(best_v[t]);
        s_part[w][r][2] = best_l[t];
        s_part[w][r][3] = mx[t];
        s_part[w][r][4] = se[t];
      }
    }
    hs_cbar();
    if (tid < nr) {
      float bs = -CUDART_INF_F, bl = 0.f, M = -CUDART_INF_F, S = 0.f;
      int bv = 0x7fffffff;
      for (int ww = 0; ww < HS_WARPS; ++ww) {
        const float sc = s_part[ww][tid][0];
        const int v = __float_as_int(s_part[ww][tid][1]);
        if (sc > bs || (sc == bs && v < bv)) {
          bs = sc;
          bv = v;
          bl = s_part[ww][tid][2];
        }
        const float m2 = s_part[ww][tid][3], s2 = s_part[ww][tid][4];
        if (m2 == -CUDART_INF_F) continue;
        if (m2 > M) {
          S = S * expf(M - m2) + s2;
          M = m2;
        } else {
          S += s2 * expf(m2 - M);
        }
      }
      float* out = a.part + ((size_t)s_b[tid] * a.nblk + blockIdx.x) * HEAD_PART;
      out[0] = bs;
      out[1] = __int_as_float(bv);
      out[2] = bl;
      out[3] = M;
      out[4] = S;
    }
  }
}
template <int MAXC>
static void launch_head_sample_c(bool bf16, const HeadArgs& b, size_t bytes, cudaStream_t st) {
  if (bf16) launch_k(k_head_sample<__nv_bfloat16, MAXC>, b.nblk, HS_THREADS, bytes, st, b);
  else launch_k(k_head_sample<float, MAXC>, b.nblk, HS_THREADS, bytes, st, b);
}
void launch_head_sample(bool bf16, const HeadArgs& a, cudaStream_t st) {
  const size_t esz = bf16 ? 2 : 4;
  const HeadPlan p = head_plan(a.B, a.d, esz);  // the state checked head_sample_fits
  HeadArgs b = a;
  b.rp = p.rp;
  b.stages = p.stages;
  b.act_off = (int)p.act_off;
  b.ring_off = (int)p.ring_off;
  // the register tile of four rows fits the row length
  const int per_lane = ((int)(a.d * esz / 16) + 31) / 32;
  if (per_lane <= 2) launch_head_sample_c<2>(bf16, b, p.bytes, st);
  else if (per_lane <= 4) launch_head_sample_c<4>(bf16, b, p.bytes, st);
  else if (per_lane <= 6) launch_head_sample_c<6>(bf16, b, p.bytes, st);
  else launch_head_sample_c<HS_MAXC>(bf16, b, p.bytes, st);
}

__global__ void k_head_reduce(HeadArgs a) {
  pdl_wait();
  pdl_launch();
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (b >= a.B || !a.stop[b]) return;
  float bs = -CUDART_INF_F, bl = 0.f, M = -CUDART_INF_F, S = 0.f;
  int bv = 0x7fffffff;
  for (int c = lane; c < a.nblk; c += 32) {
    const float* p = a.part + ((size_t)b * a.nblk + c) * HEAD_PART;
    const float s = p[0];
    const int v = __float_as_int(p[1]);
    if (s > bs || (s == bs && v < bv)) {
      bs = s;
      bv = v;
      bl = p[2];
    }
    const float m2 = p[3], s2 = p[4];
    if (m2 == -CUDART_INF_F) continue;
    if (m2 > M) {
      S = S * expf(M - m2) + s2;
      M = m2;
    } else {
      S += s2 * expf(m2 - M);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float s2 = __shfl_xor_sync(0xffffffffu, bs, o);
    const int v2 = __shfl_xor_sync(0xffffffffu, bv, o);
    const float l2 = __shfl_xor_sync(0xffffffffu, bl, o);
    const float M2 = __shfl_xor_sync(0xffffffffu, M, o);
    const float S2 = __shfl_xor_sync(0xffffffffu, S, o);
    if (s2 > bs || (s2 == bs && v2 < bv)) {
      bs = s2;
      bv = v2;
      bl = l2;
    }
    const float Mn = fmaxf(M, M2);
    if (Mn != -CUDART_INF_F) {
      S = (M == -CUDART_INF_F ? 0.f : S * expf(M - Mn)) + (M2 == -CUDART_INF_F ? 0.f : S2 * expf(M2 - Mn));
      M = Mn;
    }
  }
  if (lane == 0) {
    a.sampled[b] = bv;
    if (a.logp) a.logp[b] = bl - (M + logf(S));
  }
}
void launch_head_reduce(const HeadArgs& a, cudaStream_t st) {
  launch_k(k_head_reduce, (a.B + 7) / 8, 256, 0, st, a);
}

// ---------------------------------------------------------------------------
// Scoring (section 2: the mixture and its cross-entropy)
// ---------------------------------------------------------------------------
template <typename T>
__global__ void k_exit_rows(RowSet rs, ExitDev e, int rh, int k, int n_exits, T* __restrict__ act,
                            float* __restrict__ z, int d, float eps) {
  pdl_wait();
  pdl_launch();
  const int R = *rs.nrows;
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  const bool last = k == n_exits - 1;
  const T* g = (const T*)e.norm;
  const T* rw = (const T*)e.router_w;
  for (int r = blockIdx.x * wpb + (threadIdx.x >> 5); r < R; r += gridDim.x * wpb) {
    const float* h = rs.h + (size_t)rs.row_hrow[r] * d;
    float ss = 0.f;
    for (int i = lane; i < d; i += 32) ss = fmaf(h[i], h[i], ss);
    ss = warp_sum(ss);
    const float inv = 1.0f / sqrtf(ss / (float)d + eps);
    float zz = 0.f;
    for (int i = lane; i < d; i += 32) {
      const float n = rnd<T>(h[i] * inv * ld(g + i));
      act[(size_t)r * d + i] = cvt<T>(n);
      if (!last && rh == 0) zz = fmaf(n, ld(rw + i), zz);
    }
    if (!last && rh > 0) {
      __syncwarp();
      zz = router_mlp_part<T>(act + (size_t)r * d, (const T*)e.router_w1, e.router_b1, e.router_w2, d, rh, 0, 1);
    } else {
      zz = warp_sum(zz);
    }
    if (!last && lane == 0) z[(size_t)r * (n_exits - 1) + k] = zz + e.router_b;
  }
}
void launch_exit_rows(bool bf16, RowSet rs, const ExitDev& e, int router_hidden, int k, int n_exits, void* act,
                      float* z, int d, float eps, cudaStream_t st) {
  int grid = (rs.max_rows + 7) / 8;
  if (grid > 2048) grid = 2048;
  if (bf16)
    launch_k(k_exit_rows<__nv_bfloat16>, grid, 256, 0, st, rs, e, router_hidden, k, n_exits, (__nv_bfloat16*)act, z,
             d, eps);
  else launch_k(k_exit_rows<float>, grid, 256, 0, st, rs, e, router_hidden, k, n_exits, (float*)act, z, d, eps);
}

// log pi_k(target) = logit[target] - LSE(logits), one warp per row.
__global__ void k_lse_target(const float* __restrict__ Y, int r_begin, int n, int V, const int* __restrict__ target,
                             float* __restrict__ logpi, int k, int n_exits) {
  pdl_wait();
  pdl_launch();
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < n; i += gridDim.x * wpb) {
    const float* y = Y + (size_t)i * V;
    float m = -CUDART_INF_F;
    for (int v = lane; v < V; v += 32) m = fmaxf(m, y[v]);
    m = warp_max(m);
    float s = 0.f;
    for (int v = lane; v < V; v += 32) s += expf(y[v] - m);
    s = warp_sum(s);
    const int r = r_begin + i;
    if (lane == 0) logpi[(size_t)r * n_exits + k] = y[target[r]] - (m + logf(s));
  }
}
void launch_lse_target(const float* Y, int r_begin, int n, int V, const int* target, float* logpi, int k,
                       int n_exits, cudaStream_t st) {
  int grid = (n + 7) / 8;
  if (grid > 4096) grid = 4096;
  if (grid < 1) grid = 1;
  launch_k(k_lse_target, grid, 256, 0, st, Y, r_begin, n, V, target, logpi, k, n_exits);
}

// Combine the per-tile (max, sum exp) partials of one row in tile order,
// one warp per row: each lane merges tiles lane, lane + 32, ... in order,
// then the lanes merge in a fixed butterfly.
__global__ void k_lse_combine(const float2* __restrict__ part, const float* __restrict__ tgt, int n, int nblk,
                              float* __restrict__ logpi, int k, int n_exits) {
  pdl_wait();
  pdl_launch();
  const int lane = threadIdx.x & 31, wpb = blockDim.x >> 5;
  for (int r = blockIdx.x * wpb + (threadIdx.x >> 5); r < n; r += gridDim.x * wpb) {
    const float2* p = part + (size_t)r * nblk;
    float M = -CUDART_INF_F, S = 0.f;
    for (int b = lane; b < nblk; b += 32) {
      const float2 v = p[b];
      const float Mn = fmaxf(M, v.x);
      S = S * expf(M - Mn) + v.y * expf(v.x - Mn);
      M = Mn;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float M2 = __shfl_xor_sync(0xffffffffu, M, o);
      const float S2 = __shfl_xor_sync(0xffffffffu, S, o);
      const float Mn = fmaxf(M, M2);
      S = (M == -CUDART_INF_F ? 0.f : S * expf(M - Mn)) + (M2 == -CUDART_INF_F ? 0.f : S2 * expf(M2 - Mn));
      M = Mn;
    }
    if (lane == 0) logpi[(size_t)r * n_exits + k] = tgt[r] - (M + logf(S));
  }
}
void launch_lse_combine(const float2* part, const float* tgt, int n, int nblk, float* logpi, int k, int n_exits,
                        cudaStream_t st) {
  int grid = (n + 7) / 8;
  if (grid > 4096) grid = 4096;
  if (grid < 1) grid = 1;
  launch_k(k_lse_combine, grid, 256, 0, st, part, tgt, n, nblk, logpi, k, n_exits);
}

__device__ __forceinline__ float log_sigmoid(float z) {
  // log sigma(z) = -softplus(-z) = min(z, 0) - log1p(exp(-|z|))
  return fminf(z, 0.f) - log1pf(expf(-fabsf(z)));
}

// log pi_mix = LSE_k(log p_k + log pi_k), log p_k = log sigma(z_k) + sum_{j<k} log sigma(-z_j).
// log pi_mix = LSE_k(log p_k + log pi_k) per row; with `depth`, also the
// expected normalised layer depth sum_k p_k * exit_frac[k] (section 2
// "Training": the compute penalty is the expected normalised depth).
__global__ void k_mixture(const float* __restrict__ z, const float* __restrict__ logpi, int R, int n_exits, int mode,
                          float* __restrict__ logp, float* __restrict__ depth, ExitFrac ef) {
  pdl_wait();
  pdl_launch();
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= R) return;
  float terms[NV_MAX_EXITS];
  float acc = 0.f, M = -CUDART_INF_F, dep = 0.f;
  for (int k = 0; k < n_exits; ++k) {
    float lp;
    if (mode == NV_ROUTER_FORCE_LAST) {
      lp = (k == n_exits - 1) ? 0.f : -CUDART_INF_F;
    } else if (k < n_exits - 1) {
      const float zk = z[(size_t)r * (n_exits - 1) + k];
      lp = log_sigmoid(zk) + acc;
      acc += log_sigmoid(-zk);
    } else {
      lp = acc;
    }
    if (lp != -CUDART_INF_F) dep += expf(lp) * ef.f[k];
    terms[k] = lp + logpi[(size_t)r * n_exits + k];
    M = fmaxf(M, terms[k]);
  }
  float s = 0.f;
  for (int k = 0; k < n_exits; ++k) s += (terms[k] == -CUDART_INF_F) ? 0.f : expf(terms[k] - M);
  logp[r] = M + logf(s);
  if (depth) depth[r] = dep;
}

// *out = scale * mean(x[0..R)), accumulated in double in a fixed order
__global__ void k_mean(const float* __restrict__ x, int R, float scale, float* __restrict__ out) {
  pdl_wait();
  pdl_launch();
  __shared__ double s[256];
  double a = 0.0;
  for (int r = threadIdx.x; r < R; r += 256) a += (double)x[r];
  s[threadIdx.x] = a;
  __syncthreads();
  for (int o = 128; o; o >>= 1) {
    if (threadIdx.x < o) s[threadIdx.x] += s[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) *out = (float)((double)scale * s[0] / (double)R);
}

__global__ void k_philox(unsigned long long seed, const uint4* ctr, int n, uint4* out) {
  pdl_wait();
  pdl_launch();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = philox4x32_10(ctr[i], (uint32_t)seed, (uint32_t)(seed >> 32));
}
void launch_philox(unsigned long long seed, const void* ctr, int n, void* out, cudaStream_t st) {
  launch_k(k_philox, (n + 255) / 256, 256, 0, st, seed, (const uint4*)ctr, n, (uint4*)out);
}

// Sets a graph conditional to "some sequence still active or forced to
// complete its deferred rows"; when set, counts the launches of the block it
// guards.
__global__ void k_set_cond(cudaGraphConditionalHandle h, const int* __restrict__ active,
                           const int* __restrict__ force, int B, long long* counters, const int* block_launches) {
  pdl_wait();
  pdl_launch();
  int any = 0;
  for (int b = threadIdx.x; b < B; b += blockDim.x) any |= active[b] | force[b];
  any = __syncthreads_or(any);
  if (threadIdx.x == 0) {
    cudaGraphSetConditional(h, any ? 1u : 0u);
    if (any && counters)
      atomicAdd((unsigned long long*)&counters[NV_CTR_LAUNCHES], (unsigned long long)*block_launches);
  }
}
void launch_set_cond(cudaGraphConditionalHandle h, const int* active, const int* force, int B, long long* counters,
                     const int* block_launches, cudaStream_t st) {
  launch_k(k_set_cond, 1, 256, 0, st, h, active, force, B, counters, block_launches);
}

template <int MAXC>
static cudaError_t head_sample_smem_limit() {
  cudaError_t e = cudaFuncSetAttribute(k_head_sample<__nv_bfloat16, MAXC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)HS_DYN_MAX);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_head_sample<float, MAXC>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)HS_DYN_MAX);
  return e;
}
cudaError_t kernels_set_smem_limits(size_t plan_bytes) {
  cudaError_t e = head_sample_smem_limit<2>();
  if (e == cudaSuccess) e = head_sample_smem_limit<4>();
  if (e == cudaSuccess) e = head_sample_smem_limit<6>();
  if (e == cudaSuccess) e = head_sample_smem_limit<HS_MAXC>();
  if (e == cudaSuccess && plan_bytes > 48 * 1024) {
    e = cudaFuncSetAttribute(k_plan_norm<__nv_bfloat16, 256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)plan_bytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_plan_norm<float, 256>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan_bytes);
  }
  return e;
}

int launch_mixture(const float* z, const float* logpi, int R, int n_exits, int mode, float* logp, float* mean_nll,
                   float* depth, float* mean_depth, const ExitFrac& ef, cudaStream_t st) {
  int n = 1;
  launch_k(k_mixture, (R + 255) / 256, 256, 0, st, z, logpi, R, n_exits, mode, logp, depth, ef);
  if (mean_nll) {
    launch_k(k_mean, 1, 256, 0, st, (const float*)logp, R, -1.0f, mean_nll);
    ++n;
  }
  if (depth && mean_depth) {
    launch_k(k_mean, 1, 256, 0, st, (const float*)depth, R, 1.0f, mean_depth);
    ++n;
  }
  return n;
}

}  // namespace nv
