// Launchers for libnvium's kernels (host side).  Every launcher takes
// `bf16` to pick the element type of weights / activations / KV cache.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "gemm.cuh"

namespace nv {

constexpr int ATTN_KT = 64;    // keys per attention tile; page_size must be a multiple
constexpr int ATTN_RPC = 32;   // rows per attention CTA (row group)
constexpr int HEAD_PART = 5;   // floats per head partial: score, id, logit, max, sumexp

void launch_rope_table(float2* cs, int max_seq, int hd, double theta, cudaStream_t st);

void launch_embed_rows(bool bf16, const void* emb, const int* tok_row, RowSet rs, int d, cudaStream_t st);
void launch_rmsnorm_rows(bool bf16, RowSet rs, const void* gain, void* act, int d, float eps, cudaStream_t st);
// h[row] += sum of the split-K slices Y[s][row] (a GEMM's partial sums), then
// act[row] = RMSNorm(h[row]) * gain.
void launch_resid_norm(bool bf16, RowSet rs, const float* Y, int split_grid, int N, int K, size_t sstride,
                       const void* gain, void* act, int d, float eps, cudaStream_t st);

struct PlanArgs {
  int B, L, cap, layer, mode;  // mode 0: decode step (lazy rule), 1: flush
  const int* t;
  const int* active;
  const int* force;
  const int* lens;       // [B][L]
  int* row_b;
  int* row_pos;
  int* row_hrow;
  int* seq_start;        // [B+1]
  int* nrows;
  int max_rows;
  int* status;
  long long* counters;
  int nlayers;              // layers this plan serves (a block between exits has one row set)
  long long weight_bytes;   // this layer's weight bytes
  long long kv_pos_bytes;   // K+V bytes of one position of one layer
  const float* h;           // residual ring [B][cap][d]
};
void launch_plan_norm(bool bf16, const PlanArgs& a, const void* gain, void* act, int d, float eps,
                      int grid, cudaStream_t st);

// Y[r][n] = sum_k X[r][k] W[n][k], fp32 out, rows r < *nrows.
void launch_gemm_simt(bool bf16, const void* X, int ldx, const void* W, int N, int K, const int* nrows,
                      int max_rows, float* Y, cudaStream_t st);

struct EpiArgs {
  int mode;
  const float* Y;        // [nsplit][rows][N] partial sums
  int split_grid;        // 0: one slice; else the GEMM grid (see tc_split_count)
  int split_K;           // the GEMM's K (for tc_split_count)
  size_t split_stride;   // elements between partial-sum slices
  int N;
  RowSet rs;
  int d;
  // EPI_QKV
  int H, hd;
  const float2* rope;    // [max_seq][hd/2] (cos, sin)
  void* q_out;           // [max_rows][H*hd]
  KVView kv;
  int layer;
  // EPI_SWIGLU
  int F, G;
  void* u_out;           // [max_rows][F]
  // EPI_STORE
  float* out;
  // EPI_HEAD: rows are sequences b; logits of vocabulary tile n0/128 give one
  // Gumbel-argmax / log-sum-exp partial per stopped sequence
  const int* stop;                 // [B] stopped at this exit
  const int* t;                    // [B] position of the token being processed
  const unsigned long long* seed;  // Philox key
  float* head_part;                // [B][nblk][HEAD_PART]
  int nblk;
  // EPI_LSE: rows r of the launch are scoring rows r_begin + r
  const int* lse_target;           // [rows] target token of each scoring row (offset to the launch's first row)
  float2* lse_part;                // [rows][nblk] (max, sum exp(logit - max)) per 128-token tile
  float* lse_tgt;                  // [rows] logit of the target token
};
void launch_epilogue(bool bf16, const EpiArgs& a, int grid, cudaStream_t st);

struct AttnArgs {
  RowSet rs;
  const void* q;
  void* o;
  KVView kv;
  int layer, H, hd;
  int kv_splits, row_groups;
  float scale;
  float* part;     // [max_rows][H][kv_splits][hd+2] when kv_splits > 1
  int* lens;       // when set: lens[b*L+layer] = last row position + 1
  int L;
  int* status;     // device status word (bounded-wait expiry)
  const CUtensorMap* kv_map;  // host copy of the KV pool's 128-byte-row map (bf16, hd 64), or null
  const CUtensorMap* q_map;   // prefill / scoring: map of q (boxes of 64 x 128 rows) for the tcgen05 kernel, or null
  int dec_splits;             // MMA decode attention: key-range splits per (sequence, head)
  int* dec_ctr;               // [B][H] split arrival counters + 2 item counters (zero between launches)
  const CUtensorMap* kv_map32;  // decode / flush: the pool's map with 32-row boxes for k_attn_dec_pc, or null
};
void launch_attention(bool bf16, const AttnArgs& a, cudaStream_t st);
// Decode / flush attention.  bf16 with head_dim 64 and a KV tensor map: the
// warp-MMA kernel below (a.dec_splits key-range splits).  Otherwise the SIMT
// kernel: 128-key chunks (grid z = kv_splits = chunks of max_seq), TMA bulk
// loads of K/V pages, partials merged per row by a combine kernel.  Both
// need head_dim * element size == 128 bytes and page_size 64 or 128.
constexpr int ATTN_DEC_CK = 128;
void launch_attention_decode(bool bf16, const AttnArgs& a, cudaStream_t st);
// kernels launch_attention_decode runs for these arguments (1 or 2)
int attention_decode_launches(bool bf16, const AttnArgs& a);
// bf16 / head_dim 64 attention on warp MMAs (attn_mma.cu); both need
// a.kv_map.  Decode: grid z = a.kv_splits key-range splits; with more than
// one, partials in the row-group kernel's slots, merged by the last split
// CTA of each (sequence, head) (a.dec_ctr).
// Prefill / scoring (kv_splits == 1): 64-row query tiles, grid z from
// a.row_groups (units of ATTN_RPC rows).
cudaError_t attn_mma_prepare();
void launch_attn_dec_mma(const CUtensorMap* kvmap, const AttnArgs& a, cudaStream_t st);
void launch_attn_fa_mma(const CUtensorMap* kvmap, const AttnArgs& a, cudaStream_t st);
// Prefill / scoring on tcgen05 (attn_tc.cu): 128-row query tiles, S and the
// per-tile P V in TMEM; needs a.kv_map and a.q_map.
cudaError_t attn_tc_prepare();
// Decode / flush on persistent warps (attn_dec.cu): items of (sequence,
// head, 16-row pass, key chunk) taken from a counter in a.dec_ctr[B*H], each
// warp streaming 32-key tiles through its own TMA ring; needs a.kv_map32,
// a.part with a.kv_splits 128-key slots per (row, head), and B <= 512.
cudaError_t attn_dec_pc_prepare();
bool attn_dec_pc_fits(const AttnArgs& a);
void launch_attn_dec_pc(const AttnArgs& a, cudaStream_t st);
void launch_attn_fa_tc(const CUtensorMap* kvmap, const CUtensorMap* qmap, const AttnArgs& a, cudaStream_t st);

struct StepArgs {
  int B, L, cap, d, n_exits;
  int* t;
  int* tok;
  int* active;
  int* exit_id;
  int* force;
  int* stop;             // [n_exits][B]
  int* nstop;            // [n_exits]
  float* router_p;       // [n_exits][B] w_k of this step (NaN: junction not reached)
  const int* lens;
  float* hbuf;
  const void* emb;
  unsigned long long* seed_dev;
  unsigned long long seed;
  long long* counters;
  // step end
  const int* sampled;
  int* out_tok;
  int* out_exit;
};
void launch_step_begin(bool bf16, const StepArgs& a, cudaStream_t st);
void launch_step_end(const StepArgs& a, cudaStream_t st);

struct JuncArgs {
  int B, cap, d, k, n_exits, router_mode;
  float eps;
  const int* t;
  int* active;
  int* exit_id;
  int* stop;             // [B] flags of this exit
  float* router_p;       // [B] w_k of this exit's junction, per sequence
  const float* hbuf;
  const void* norm;
  const void* router_w;
  float router_b;
  int router_hidden;     // router MLP width (0: scalar router)
  const void* router_w1; // [r][d] model dtype
  const float* router_b1;
  const float* router_w2;
  void* exit_act;        // [B][d]
  const unsigned long long* seed;
  long long* counters;
  int* nstop;            // stops at this exit in this step (zeroed at step begin)
  long long head_bytes;  // counted once per exit that has a stop
};
void launch_junction(bool bf16, const JuncArgs& a, cudaStream_t st);

// Exit adapter in front of the shared head (decode): for every sequence that
// stopped at this exit, exit_act[b] (n_k on entry) becomes the final
// RMSNorm of m = h + W2 silu(W1 n_k).
struct AdapterArgs {
  int B, cap, d, a;
  float eps;
  const int* t;
  const int* stop;        // [B] flags of this exit
  const float* hbuf;
  const void* w1;         // [a][d]
  const void* w2;         // [d][a]
  const void* final_norm; // [d] (the last exit's norm)
  void* exit_act;         // [B][d]
};
void launch_exit_adapter(bool bf16, const AdapterArgs& a, cudaStream_t st);
cudaError_t exit_adapter_prepare(bool bf16, int d, int a);
// Scoring side of the same adapter, after the two GEMMs of W1 and W2:
// u = silu(Y) (model dtype) over the [rows][a] hidden, and act = final
// RMSNorm of h + Y over the [rows][d] output.
void launch_silu_rows(bool bf16, const int* nrows, const float* Y, int a, void* u, int max_rows, cudaStream_t st);
void launch_adapter_norm_rows(bool bf16, RowSet rs, const float* Y, const void* final_norm, void* act, int d,
                              float eps, cudaStream_t st);

struct HeadArgs {
  int B, d, V, k;
  const int* t;
  const int* stop;       // [B] flags of this exit
  const void* exit_act;  // [B][d]
  const void* head;      // [V][d]
  const unsigned long long* seed;
  float* part;           // [B][nblk][HEAD_PART]
  int nblk;
  long long* counters;
  long long head_bytes;
  int* status;           // device error word (a bounded wait that ran out)
  // shared-memory plan of the sampler, filled by launch_head_sample
  int rp, stages, act_off, ring_off;
  // reduce
  int* sampled;
  float* logp;
};
// The small-batch sampler runs one CTA per SM (nblk = the SM count) and
// needs its stopped-row list, one pass of rows and a ring of at least two
// stages in shared memory; false when B and d leave no such plan.
bool head_sample_fits(int B, int d, size_t esz);
void launch_head_sample(bool bf16, const HeadArgs& a, cudaStream_t st);
void launch_head_reduce(const HeadArgs& a, cudaStream_t st);

// scoring
// Scoring rows at exit k: act = RMSNorm_k(h) (model dtype) and the router
// logit z[r][k] (scalar router, or the router MLP when router_hidden > 0).
void launch_exit_rows(bool bf16, RowSet rs, const ExitDev& e, int router_hidden, int k, int n_exits, void* act,
                      float* z, int d, float eps, cudaStream_t st);
void launch_lse_target(const float* Y, int r_begin, int n, int V, const int* target, float* logpi, int k,
                       int n_exits, cudaStream_t st);
// log pi_k(target) of rows [0, n) from the fused head epilogue's per-tile
// partials (EPI_LSE): LSE over the nblk tiles in tile order, minus nothing
// else: logpi[r][k] = tgt[r] - (M + log S).
void launch_lse_combine(const float2* part, const float* tgt, int n, int nblk, float* logpi, int k, int n_exits,
                        cudaStream_t st);
// Sets conditional `h` to (any active[b] or force[b]); when set, adds
// *block_launches to counters[NV_CTR_LAUNCHES].
void launch_set_cond(cudaGraphConditionalHandle h, const int* active, const int* force, int B, long long* counters,
                     const int* block_launches, cudaStream_t st);
void launch_philox(unsigned long long seed, const void* ctr, int n, void* out, cudaStream_t st);

// Opt-in shared memory for the head sampler and the planner.
cudaError_t kernels_set_smem_limits(size_t plan_bytes);

// Normalised depth of each exit: exit_layers[k] / n_layers.
struct ExitFrac {
  float f[NV_MAX_EXITS];
};
// log pi_mix per row, optional mean NLL, optional expected normalised depth
// per row and its mean; returns the number of kernels launched.
int launch_mixture(const float* z, const float* logpi, int R, int n_exits, int mode, float* logp, float* mean_nll,
                   float* depth, float* mean_depth, const ExitFrac& ef, cudaStream_t st);

}  // namespace nv
