// libnvium C ABI: model packing, decode state, and the host-side order of
// kernel launches for prefill, decode steps, flush and scoring.
//
// The decode step follows section 2 "Inferenz: Piggybacking" of the N-vium
// summary (arXiv 2605.13190): per layer one packed pass over the new tokens
// still active at that depth and the deferred rows of their sequences.  All
// control flow inside a step is on the device (row counts, stop decisions),
// so a step is one CUDA graph replay.
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include "gemm.cuh"
#include "gemm_tc.cuh"
#include "kernels.cuh"
#include "layer_tc.cuh"

namespace nv {
static thread_local std::string g_err;
void set_error(const std::string& msg) { g_err = msg; }
}  // namespace nv

using namespace nv;

namespace {

template <typename T>
nv_status dalloc(T** p, size_t count) {
  *p = nullptr;
  if (count == 0) count = 1;
  cudaError_t e = cudaMalloc((void**)p, count * sizeof(T));
  if (e != cudaSuccess) {
    set_error(std::string("cudaMalloc of ") + std::to_string(count * sizeof(T)) + " bytes: " + cudaGetErrorString(e));
    cudaGetLastError();
    return NV_ERR_OOM;
  }
  return NV_OK;
}
nv_status dalloc_bytes(void** p, size_t bytes) { return dalloc((unsigned char**)p, bytes); }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// bf16 / head_dim 64 attention runs on the warp-MMA kernels unless
// NVIUM_ATTN=simt selects the SIMT ones (kept for comparison)
bool mma_attention_enabled() {
  const char* ev = std::getenv("NVIUM_ATTN");
  return !(ev && std::string(ev) == "simt");
}

// prefill / scoring attention on tcgen05 unless NVIUM_ATTN=mma (the warp-MMA
// kernel) or NVIUM_ATTN=simt selects another engine
bool tc_attention_enabled() {
  const char* ev = std::getenv("NVIUM_ATTN");
  return !(ev && (std::string(ev) == "simt" || std::string(ev) == "mma"));
}

// NVIUM_DEC_ATTN=pc: decode / flush attention on persistent warps
// (k_attn_dec_pc) instead of one CTA per (sequence, head, key split)
// (k_attn_dec_mma).  Both give the path's results; measured on B200 the
// persistent one is slower (B=64 decode 9.4k against 12.3k tokens/s, B=1
// 562 against 614), so it is an option, not the default
bool dec_pc_attention_enabled() {
  const char* ev = std::getenv("NVIUM_DEC_ATTN");
  return mma_attention_enabled() && ev && std::string(ev) == "pc";
}

// NVIUM_LAYER_KERNEL=1: decode and flush layers run as one persistent kernel
// after attention (layer_tc.cu), which gives the same bits as the default
// per-kernel path; measured on B200 it is slower (its seven cross-CTA
// hand-offs per layer cost more than the per-kernel path's launches, which
// overlap through programmatic dependent launch and pull the next GEMM's
// weights into L2), so it is an option, not the default
bool layer_kernel_enabled() {
  const char* ev = std::getenv("NVIUM_LAYER_KERNEL");
  return ev && ev[0] == '1';
}

constexpr int kTileCounters = 1024;  // >= N/128 of any split GEMM
size_t tc_split_stride_elems(int N) { return nv::tc_split_stride((size_t)N); }

// grow-only device buffer
struct Buf {
  void* p = nullptr;
  size_t bytes = 0;
  nv_status need(size_t n) {
    if (n <= bytes) return NV_OK;
    if (p) cudaFree(p);
    p = nullptr;
    bytes = 0;
    NV_TRY(dalloc_bytes(&p, n));
    bytes = n;
    return NV_OK;
  }
  void release() {
    if (p) cudaFree(p);
    p = nullptr;
    bytes = 0;
  }
  template <typename T> T* as() const { return (T*)p; }
};

}  // namespace

struct nv_model {
  nv_config cfg;
  bool bf16 = false;
  size_t esz = 4;
  int d = 0, H = 0, hd = 0, HQ = 0, F = 0, V = 0, L = 0, NE = 0, G = 0;
  void* pool = nullptr;
  void* tok_emb = nullptr;
  std::vector<LayerDev> layers;
  std::vector<ExitDev> exits;
  std::vector<int> exit_at;  // layer (0-based) -> exit index, or -1
  float2* rope = nullptr;
  long long layer_weight_bytes = 0;
  int gemm_kind = GEMM_SIMT;
  bool tc_attention = false;  // prefill/scoring attention on the tcgen05 kernel (attn_tc.cu)
  bool layer_kernel = false;  // decode/flush layers on the persistent kernel (layer_tc.cu)
  GemmPlanCache* gemm_plans = nullptr;
  // scoring scratch
  Buf sc_h, sc_act, sc_u, sc_ctr, sc_q, sc_o, sc_Y, sc_kv, sc_part, sc_z, sc_logpi, sc_logp, sc_i32, sc_nll,
      sc_depth, sc_mdepth, sc_lse_part, sc_lse_tgt;
};

struct nv_state {
  nv_model* m = nullptr;
  int B = 0, cap = 0, max_seq = 0, ps = 0, pps = 0, max_rows = 0;
  // paged KV
  void* kv = nullptr;
  size_t kv_layer_stride = 0;
  CUtensorMap kv_map;        // the pool as rows of 128 bytes (bf16, head_dim 64)
  bool kv_map_ok = false;
  CUtensorMap kv_map32;      // the same with boxes of 32 rows (persistent decode attention)
  bool kv_map32_ok = false;
  int dec_splits = 1;        // key-range splits per (sequence, head) of the MMA decode attention
  int* dec_ctr = nullptr;    // [B][H] split arrival counters of the decode attention, + 2 item counters
  int n_pages = 0;
  int* page_table = nullptr;
  std::vector<int> h_page_table;
  int next_free_page = 0;
  // per-sequence device state
  int *t = nullptr, *tok = nullptr, *lens = nullptr, *active = nullptr, *exit_id = nullptr, *force = nullptr;
  int *stop = nullptr, *sampled = nullptr, *out_tok = nullptr, *out_exit = nullptr;
  int *nstop = nullptr, *d_B = nullptr, *d_block_launches = nullptr;
  bool tc_head = false;  // exit heads on tensor cores (bf16, B >= 16)
  int *prompt_len = nullptr, *prompt_last = nullptr;
  float* logp = nullptr;
  float* router_p = nullptr;  // [NV_MAX_EXITS][B] router probabilities of the last step
  bool stepped = false;       // a decode step has run since nv_prefill
  float* hbuf = nullptr;
  // work list and activations
  int *row_b = nullptr, *row_pos = nullptr, *row_hrow = nullptr, *seq_start = nullptr, *nrows = nullptr;
  void *act = nullptr, *u = nullptr, *q = nullptr, *o = nullptr, *exit_act = nullptr;
  int* tile_counters = nullptr;
  int* lt_sync = nullptr;      // [L][lt_sync_ints] counters of the persistent layer kernel
  size_t lt_sync_ints = 0;
  float* lt_ygu = nullptr;     // its gate/up split slices
  float *Y = nullptr, *attn_part = nullptr, *head_part = nullptr;
  size_t Y_elems = 0;
  int head_nblk = 0, kv_splits = 1, row_groups = 1;
  bool dec_attn = false;
  unsigned long long* seed_dev = nullptr;
  long long* counters = nullptr;
  int* status = nullptr;
  // host mirrors
  std::vector<int> h_prompt_len, h_t;
  long long launches_per_step = 0, launches_total = 0;
  bool prefilled = false;
  cudaGraphExec_t graph = nullptr;
  cudaStream_t cap_stream = nullptr, cap_stream2 = nullptr;
  long long block_launches[NV_MAX_EXITS] = {0};
  bool cond_graph = false;
  std::vector<void*> allocs;
  // prefill scratch
  // prefill working set, kept between calls (grow-only)
  Buf pf_rows, pf_h, pf_act, pf_u, pf_q, pf_o, pf_Y, pf_ctr;
  // page-table uploads go through a pinned copy, reusable once `pt_done` fired
  int* h_pt_pinned = nullptr;
  cudaEvent_t pt_done = nullptr;
  bool pt_pending = false;
};

namespace {

RowSet state_rowset(nv_state* s) {
  RowSet rs;
  rs.nrows = s->nrows;
  rs.row_b = s->row_b;
  rs.row_pos = s->row_pos;
  rs.row_hrow = s->row_hrow;
  rs.seq_start = s->seq_start;
  rs.h = s->hbuf;
  rs.max_rows = s->max_rows;
  rs.B = s->B;
  return rs;
}

KVView state_kv(nv_state* s) {
  KVView kv;
  kv.base = s->kv;
  kv.layer_stride = s->kv_layer_stride;
  kv.page_table = s->page_table;
  kv.pages_per_seq = s->pps;
  kv.page_size = s->ps;
  kv.H = s->m->H;
  kv.hd = s->m->hd;
  return kv;
}

struct LayerIO {
  RowSet rs;
  KVView kv;
  void* act;           // [rows][d] normed activations
  void* u;             // [rows][F] SwiGLU output
  void* q;
  void* o;
  int* tile_counters;  // split-K arrival counters (zeroed)
  float* Y;
  float* attn_part;
  int kv_splits, row_groups;
  int* lens;           // nullable: per-(seq, layer) lengths to advance
  int L;
  int epi_grid;
  bool dec_attn;       // chunked decode attention (else row-group attention)
  const CUtensorMap* kv_map;  // nullable: TMA view of the KV pool for the MMA attention kernels
  const CUtensorMap* kv_map32;  // nullable: the same with 32-row boxes (persistent decode attention)
  int dec_splits;             // key-range splits of the MMA decode attention
  int* dec_ctr;               // its per-(sequence, head) split arrival counters
  bool prefetch_next;  // the last GEMM of a layer prefetches the next layer's QKV weights
  bool split_k;        // few rows expected (decode, flush): let the GEMM split K
  int* status;
  int* lt_sync;        // non-null: decode/flush layers on the persistent layer kernel
  size_t lt_sync_ints;
  float* lt_ygu;
};

// Per-kernel event timing for nv_decode_step_profiled (null when capturing).
struct Prof {
  cudaStream_t st = nullptr;
  std::vector<cudaEvent_t> pool;
  size_t used = 0;
  struct Rec {
    int kind;
    cudaEvent_t a, b;
    long long bytes, flops;
    int kernels;
  };
  std::vector<Rec> recs;
  // host copies of the current layer's work list
  int R = 0;
  long long kv_read = 0;
  cudaEvent_t ev() {
    if (used == pool.size()) {
      cudaEvent_t e;
      cudaEventCreate(&e);
      pool.push_back(e);
    }
    return pool[used++];
  }
  cudaEvent_t open_a = nullptr;
  void begin() {
    open_a = ev();
    cudaEventRecord(open_a, st);
  }
  void end(int kind, long long bytes, long long flops, int kernels) {
    cudaEvent_t b = ev();
    cudaEventRecord(b, st);
    recs.push_back(Rec{kind, open_a, b, bytes, flops, kernels});
  }
  ~Prof() {
    for (cudaEvent_t e : pool) cudaEventDestroy(e);
  }
};

// Runs `launch` bracketed by events when profiling; counts launches.
template <typename F>
void timed(Prof* prof, long long* launches, int nlaunch, int kind, long long bytes, long long flops, F&& launch) {
  if (prof) prof->begin();
  launch();
  if (prof) prof->end(kind, bytes, flops, nlaunch);
  if (launches) *launches += nlaunch;
}

// Everything of layer `layer` after the attention RMSNorm (act holds the
// normed rows): QKV + RoPE + KV write, attention, O + residual, MLP norm,
// gate/up + SwiGLU, down + residual.  With `next_norm` (the next layer's
// attention-norm gain, when it runs the same rows) the down projection's
// residual is followed by that norm, so act is ready for the next layer.
// The persistent decode-layer kernel's arguments for layer `layer`:
// MLP part of this layer (when `mlp`), then the next layer's norm and QKV
// when it runs the same rows (`next_norm`), or this layer's QKV alone.
LayerTcRun layer_tc_args(nv_model* M, int layer, const LayerIO& io, bool mlp, const void* next_norm) {
  const LayerDev& Lw = M->layers[layer];
  LayerTcRun r{};
  r.rs = io.rs;
  r.kv = io.kv;
  r.rope = M->rope;
  r.o = io.o;
  r.act = io.act;
  r.u = io.u;
  r.q = io.q;
  r.Y = io.Y;
  r.Ygu = io.lt_ygu;
  r.sync = io.lt_sync + (size_t)layer * io.lt_sync_ints;
  r.status = io.status;
  r.d = M->d;
  r.HQ = M->HQ;
  r.H = M->H;
  r.hd = M->hd;
  r.F = M->F;
  r.eps = M->cfg.rms_eps;
  if (mlp) {
    r.w_o = Lw.w_o;
    r.w_gu = Lw.w_gu;
    r.w_d = Lw.w_d;
    r.mlp_norm = Lw.mlp_norm;
    r.flags = LT_MLP;
    if (next_norm) {
      r.flags |= LT_NORM2 | LT_QKV;
      r.norm2 = next_norm;
      r.w_qkv = M->layers[layer + 1].w_qkv;
      r.kv_layer = layer + 1;
    }
  } else {
    r.flags = LT_QKV;
    r.w_qkv = Lw.w_qkv;
    r.kv_layer = layer;
  }
  return r;
}

nv_status layer_body(nv_model* M, int layer, const LayerIO& io, cudaStream_t st, Prof* prof = nullptr,
                     long long* launches = nullptr, const void* next_norm = nullptr, bool qkv_ready = false) {
  const LayerDev& Lw = M->layers[layer];
  const bool bf = M->bf16;
  const long long es = (long long)M->esz;
  const long long R = prof ? prof->R : 0;
  const long long d = M->d, HQ = M->HQ, F = M->F;
  nv_status gst = NV_OK;
  EpiArgs e{};
  e.rs = io.rs;
  e.d = M->d;
  e.H = M->H;
  e.hd = M->hd;
  e.rope = M->rope;
  e.kv = io.kv;
  e.layer = layer;  // scoring's single-layer scratch has layer_stride 0
  e.F = M->F;
  e.G = M->G;
  e.q_out = io.q;
  e.u_out = io.u;
  // algorithmic bytes of Y = X W^T + epilogue: W once, X once, outputs once
  // the weights each GEMM pulls into L2 for the one after it
  const LayerDev* nextL = layer + 1 < M->L ? &M->layers[layer + 1] : nullptr;
  auto gemm = [&](int mode, const void* X, long long ldx, const void* W, long long N, long long K, long long out_bytes,
                  const void* pf, long long pf_bytes) {
    e.mode = mode;
    e.N = (int)N;
    // decode and flush may split K when the rows fit one tile and the feature
    // tiles cannot fill the GPU (tc_split_count); the persistent decode-layer
    // kernel splits every part the same way, so the two decode paths agree
    // bit for bit
    const bool split = io.split_k;
    timed(prof, launches, gemm_launch_count(M->gemm_kind, bf, split, &e), NV_K_GEMM,
          N * K * es + R * K * es + out_bytes,
          2 * R * N * K, [&] {
            gst = gemm_run(M->gemm_plans, M->gemm_kind, bf, X, (int)ldx, W, (int)N, (int)K, io.rs.nrows,
                           io.rs.max_rows, io.Y, split, &e, io.tile_counters, io.epi_grid, pf,
                           pf ? (size_t)pf_bytes : 0, st);
          });
    return gst;
  };
  const bool persistent = io.lt_sync && io.split_k && M->layer_kernel;
  const long long wq_bytes = 3 * HQ * d * es, wmlp_bytes = (d * HQ + 3 * F * d) * es;
  if (persistent) {
    // QKV + RoPE + KV write, unless the previous layer's launch did it
    if (!qkv_ready) {
      const LayerTcRun r = layer_tc_args(M, layer, io, false, nullptr);
      timed(prof, launches, 1, NV_K_GEMM, wq_bytes + R * d * es + R * 3 * HQ * es, 2 * R * 3 * HQ * d,
            [&] { gst = layer_tc_launch(gemm_tc_plans(M->gemm_plans), r, st); });
      NV_TRY(gst);
    }
  } else {
    // QKV + RoPE + KV write (fused epilogue)
    NV_TRY(gemm(EPI_QKV, io.act, d, Lw.w_qkv, 3 * HQ, d, R * 3 * HQ * es, Lw.w_o, d * HQ * es));
  }
  // attention
  AttnArgs a{};
  a.rs = io.rs;
  a.q = io.q;
  a.o = io.o;
  a.kv = io.kv;
  a.layer = layer;
  a.H = M->H;
  a.hd = M->hd;
  a.kv_splits = io.kv_splits;
  a.row_groups = io.row_groups;
  a.scale = 1.0f / sqrtf((float)M->hd);
  a.part = io.attn_part;
  a.lens = io.lens;
  a.L = io.L;
  a.status = io.status;
  a.kv_map = io.kv_map;
  CUtensorMap qmap;
  if (!io.dec_attn && io.kv_map && M->tc_attention) {
    gst = tc_map(gemm_tc_plans(M->gemm_plans), io.q, (uint64_t)HQ, (uint64_t)io.rs.max_rows, (uint64_t)HQ, 128,
                 &qmap);
    NV_TRY(gst);
    a.q_map = &qmap;
  }
  a.dec_splits = io.dec_splits;
  a.dec_ctr = io.dec_ctr;
  a.kv_map32 = io.dec_attn ? io.kv_map32 : nullptr;
  const int attn_launches = io.dec_attn ? attention_decode_launches(bf, a) : (io.kv_splits > 1 ? 2 : 1);
  timed(prof, launches, attn_launches, NV_K_ATTENTION,
        (prof ? prof->kv_read : 0) + 2 * R * HQ * es, 0, [&] {
          if (io.dec_attn) launch_attention_decode(bf, a, st);
          else launch_attention(bf, a, st);
        });
  if (persistent) {
    // everything after attention, and the next layer's QKV when it runs the same rows
    const LayerTcRun r = layer_tc_args(M, layer, io, true, next_norm);
    const long long b = wmlp_bytes + (next_norm ? wq_bytes : 0) + R * HQ * es + R * d * 8;
    const long long f = 2 * R * (d * HQ + 3 * F * d + (next_norm ? 3 * HQ * d : 0));
    timed(prof, launches, 1, NV_K_GEMM, b, f, [&] { gst = layer_tc_launch(gemm_tc_plans(M->gemm_plans), r, st); });
    return gst;
  }
  // output projection + residual, MLP RMSNorm
  if (M->gemm_kind == GEMM_TC && io.split_k) {
    // split-K slices of the projection are summed into h by the norm kernel
    int sg = 0;
    timed(prof, launches, 1, NV_K_GEMM, d * HQ * es + R * HQ * es + R * d * 4, 2 * R * d * HQ, [&] {
      gst = gemm_run(M->gemm_plans, M->gemm_kind, bf, io.o, (int)HQ, Lw.w_o, (int)d, (int)HQ, io.rs.nrows,
                     io.rs.max_rows, io.Y, true, nullptr, io.tile_counters, io.epi_grid, Lw.w_gu,
                     (size_t)(2 * F * d * es), st, &sg);
    });
    NV_TRY(gst);
    timed(prof, launches, 1, NV_K_NORM, R * d * (8 + es), 0, [&] {
      launch_resid_norm(bf, io.rs, io.Y, sg, M->d, M->HQ, tc_split_stride_elems(M->d), Lw.mlp_norm, io.act, M->d,
                        M->cfg.rms_eps, st);
    });
  } else {
    NV_TRY(gemm(EPI_RESID, io.o, HQ, Lw.w_o, d, HQ, R * d * 8, Lw.w_gu, 2 * F * d * es));
    timed(prof, launches, 1, NV_K_NORM, R * d * (4 + es), 0,
          [&] { launch_rmsnorm_rows(bf, io.rs, Lw.mlp_norm, io.act, M->d, M->cfg.rms_eps, st); });
  }
  NV_TRY(gemm(EPI_SWIGLU, io.act, d, Lw.w_gu, 2 * F, d, R * F * es, Lw.w_d, d * F * es));
  const void* pf_next = io.prefetch_next && nextL ? nextL->w_qkv : nullptr;
  if (next_norm && M->gemm_kind == GEMM_TC && io.split_k) {
    // down projection slices summed into h by the norm kernel, which also
    // writes the next layer's normed rows
    int sg = 0;
    timed(prof, launches, 1, NV_K_GEMM, d * F * es + R * F * es + R * d * 4, 2 * R * d * F, [&] {
      gst = gemm_run(M->gemm_plans, M->gemm_kind, bf, io.u, (int)F, Lw.w_d, (int)d, (int)F, io.rs.nrows,
                     io.rs.max_rows, io.Y, true, nullptr, io.tile_counters, io.epi_grid, pf_next,
                     (size_t)(3 * HQ * d * es), st, &sg);
    });
    NV_TRY(gst);
    timed(prof, launches, 1, NV_K_NORM, R * d * (8 + es), 0, [&] {
      launch_resid_norm(bf, io.rs, io.Y, sg, M->d, M->F, tc_split_stride_elems(M->d), next_norm, io.act, M->d,
                        M->cfg.rms_eps, st);
    });
    return NV_OK;
  }
  NV_TRY(gemm(EPI_RESID, io.u, F, Lw.w_d, d, F, R * d * 8, pf_next, 3 * HQ * d * es));
  if (next_norm)
    timed(prof, launches, 1, NV_K_NORM, R * d * (4 + es), 0,
          [&] { launch_rmsnorm_rows(bf, io.rs, next_norm, io.act, M->d, M->cfg.rms_eps, st); });
  return NV_OK;
}

// Layers between two exits run the same rows (exits happen only after a
// block's last layer, and a block's layers keep equal cache lengths), so a
// block is planned once, at its first layer.
int block_layers(const nv_model* M, int layer) {
  int n = 1;
  while (layer + n - 1 < M->L - 1 && M->exit_at[layer + n - 1] < 0) ++n;
  return n;
}
// the next layer's attention-norm gain when it runs the same rows as `layer`
const void* next_norm_in_block(const nv_model* M, int layer) {
  return (layer + 1 < M->L && M->exit_at[layer] < 0) ? M->layers[layer + 1].attn_norm : nullptr;
}

LayerIO state_io(nv_state* s) {
  LayerIO io{};
  io.rs = state_rowset(s);
  io.kv = state_kv(s);
  io.act = s->act;
  io.u = s->u;
  io.tile_counters = s->tile_counters;
  io.q = s->q;
  io.o = s->o;
  io.Y = s->Y;
  io.attn_part = s->attn_part;
  io.kv_splits = s->kv_splits;
  io.row_groups = s->row_groups;
  io.lens = s->lens;
  io.L = s->m->L;
  // split-K epilogues: a few rows per sequence at small batch, where a
  // smaller grid starts sooner; 8 CTAs per SM otherwise
  io.epi_grid = s->B <= 8 ? 296 : 1184;
  io.dec_attn = s->dec_attn;
  io.kv_map = s->kv_map_ok ? &s->kv_map : nullptr;
  io.kv_map32 = s->kv_map32_ok ? &s->kv_map32 : nullptr;
  io.dec_splits = s->dec_splits;
  io.dec_ctr = s->dec_ctr;
  io.prefetch_next = true;
  io.split_k = true;
  io.status = s->status;
  io.lt_sync = s->lt_sync;
  io.lt_sync_ints = s->lt_sync_ints;
  io.lt_ygu = s->lt_ygu;
  return io;
}

PlanArgs state_plan(nv_state* s, int layer, int mode) {
  nv_model* M = s->m;
  PlanArgs p{};
  p.B = s->B;
  p.L = M->L;
  p.cap = s->cap;
  p.layer = layer;
  p.mode = mode;
  p.t = s->t;
  p.active = s->active;
  p.force = s->force;
  p.lens = s->lens;
  p.row_b = s->row_b;
  p.row_pos = s->row_pos;
  p.row_hrow = s->row_hrow;
  p.seq_start = s->seq_start;
  p.nrows = s->nrows;
  p.max_rows = s->max_rows;
  p.status = s->status;
  p.counters = s->counters;
  p.nlayers = 1;
  p.weight_bytes = M->layer_weight_bytes;
  p.kv_pos_bytes = (long long)2 * M->HQ * (long long)M->esz;
  p.h = s->hbuf;
  return p;
}

int plan_grid(nv_state* s) {
  int g = (s->B * 2 + 7) / 8;
  if (g < 1) g = 1;
  if (g > 148) g = 148;
  return g;
}

// Read the current layer's row count and attended KV bytes (profiling only).
nv_status prof_read_plan(nv_state* s, Prof* prof, cudaStream_t st) {
  NV_CUDA_TRY(cudaStreamSynchronize(st));
  int R = 0;
  NV_CUDA_TRY(cudaMemcpy(&R, s->nrows, 4, cudaMemcpyDeviceToHost));
  prof->R = R;
  prof->kv_read = 0;
  if (R > 0) {
    std::vector<int> start(s->B + 1), pos(R);
    NV_CUDA_TRY(cudaMemcpy(start.data(), s->seq_start, (s->B + 1) * 4, cudaMemcpyDeviceToHost));
    NV_CUDA_TRY(cudaMemcpy(pos.data(), s->row_pos, (size_t)R * 4, cudaMemcpyDeviceToHost));
    for (int b = 0; b < s->B; ++b)
      if (start[b + 1] > start[b]) prof->kv_read += (long long)(pos[start[b + 1] - 1] + 1) * 2 * s->m->HQ * s->m->esz;
  }
  return NV_OK;
}

// Layers [l0, l1) of a decode step, with the junction and exit head at every
// exit layer among them.
nv_status record_layers(nv_state* s, cudaStream_t st, Prof* prof, long long* launches, int l0, int l1) {
  nv_model* M = s->m;
  const bool bf = M->bf16;
  const long long es = (long long)M->esz;
  LayerIO io = state_io(s);
  for (int layer = l0; layer < l1; ++layer) {
    if (layer == l0 || M->exit_at[layer - 1] >= 0) {
      PlanArgs p = state_plan(s, layer, 0);
      p.nlayers = block_layers(M, layer);
      timed(prof, launches, 1, NV_K_PLAN_NORM, 0, 0, [&] {
        launch_plan_norm(bf, p, M->layers[layer].attn_norm, s->act, M->d, M->cfg.rms_eps, plan_grid(s), st);
      });
      if (prof) {
        NV_TRY(prof_read_plan(s, prof, st));
        prof->recs.back().bytes = (long long)prof->R * M->d * (4 + es);
      }
    }
    const bool block_start = layer == l0 || M->exit_at[layer - 1] >= 0;
    NV_TRY(layer_body(M, layer, io, st, prof, launches, next_norm_in_block(M, layer), !block_start));
    const int k = M->exit_at[layer];
    if (k < 0) continue;
    JuncArgs j{};
    j.B = s->B;
    j.cap = s->cap;
    j.d = M->d;
    j.k = k;
    j.n_exits = M->NE;
    j.router_mode = M->cfg.router_mode;
    j.eps = M->cfg.rms_eps;
    j.t = s->t;
    j.active = s->active;
    j.exit_id = s->exit_id;
    j.stop = s->stop + (size_t)k * s->B;
    j.router_p = s->router_p + (size_t)k * s->B;
    j.hbuf = s->hbuf;
    j.norm = M->exits[k].norm;
    j.router_w = M->exits[k].router_w;
    j.router_b = M->exits[k].router_b;
    j.router_hidden = M->cfg.router_hidden;
    j.router_w1 = M->exits[k].router_w1;
    j.router_b1 = M->exits[k].router_b1;
    j.router_w2 = M->exits[k].router_w2;
    j.exit_act = s->exit_act;
    j.seed = s->seed_dev;
    j.counters = s->counters;
    j.nstop = s->nstop + k;
    j.head_bytes = (long long)M->V * M->d * es;
    timed(prof, launches, 1, NV_K_JUNCTION, (long long)s->B * M->d * (4 + es), 0,
          [&] { launch_junction(bf, j, st); });
    if (M->cfg.adapter_hidden && k < M->NE - 1) {
      // the shared head reads the adapter's output, not n_k
      AdapterArgs ad{};
      ad.B = s->B;
      ad.cap = s->cap;
      ad.d = M->d;
      ad.a = M->cfg.adapter_hidden;
      ad.eps = M->cfg.rms_eps;
      ad.t = s->t;
      ad.stop = j.stop;
      ad.hbuf = s->hbuf;
      ad.w1 = M->exits[k].adapter_w1;
      ad.w2 = M->exits[k].adapter_w2;
      ad.final_norm = M->exits[M->NE - 1].norm;
      ad.exit_act = s->exit_act;
      timed(prof, launches, 1, NV_K_JUNCTION, 2LL * ad.a * M->d * es, 4LL * s->B * ad.a * M->d,
            [&] { launch_exit_adapter(bf, ad, st); });
    }
    HeadArgs h{};
    h.B = s->B;
    h.d = M->d;
    h.V = M->V;
    h.k = k;
    h.t = s->t;
    h.stop = j.stop;
    h.exit_act = s->exit_act;
    h.head = M->exits[k].head;
    h.seed = s->seed_dev;
    h.part = s->head_part;
    h.nblk = s->head_nblk;
    h.counters = s->counters;
    h.status = s->status;
    h.head_bytes = (long long)M->V * M->d * es;
    h.sampled = s->sampled;
    h.logp = s->logp;
    long long hb = 0, hf = 0;
    if (prof) {
      // rows that stop at this exit: known once the junction has run
      NV_CUDA_TRY(cudaStreamSynchronize(st));
      std::vector<int> stop(s->B);
      NV_CUDA_TRY(cudaMemcpy(stop.data(), j.stop, s->B * 4, cudaMemcpyDeviceToHost));
      long long n = 0;
      for (int v : stop) n += v;
      if (n) hb = h.head_bytes + n * M->d * es;
      hf = 2 * n * (long long)M->V * M->d;
    }
    nv_status hst = NV_OK;
    timed(prof, launches, 2, NV_K_HEAD, hb, hf, [&] {
      if (s->tc_head) {
        // tensor-core head over every sequence's exit state; columns of
        // sequences that did not stop here are ignored, and nothing runs
        // when no sequence stopped here
        EpiArgs he{};
        he.mode = EPI_HEAD;
        he.stop = j.stop;
        he.t = s->t;
        he.seed = s->seed_dev;
        he.head_part = s->head_part;
        he.nblk = M->V / 128;
        hst = tc_gemm_run(gemm_tc_plans(M->gemm_plans), s->exit_act, M->d, M->exits[k].head, M->V, M->d, s->d_B,
                          s->B, s->Y, false, &he, nullptr, nullptr, 0, st, nullptr, s->nstop + k);
        h.nblk = M->V / 128;
      } else {
        launch_head_sample(bf, h, st);
      }
      launch_head_reduce(h, st);
    });
    NV_TRY(hst);
  }
  return NV_OK;
}

void record_step_end(nv_state* s, cudaStream_t st, Prof* prof, long long* launches) {
  StepArgs sa{};
  sa.B = s->B;
  sa.t = s->t;
  sa.tok = s->tok;
  sa.exit_id = s->exit_id;
  sa.counters = s->counters;
  sa.sampled = s->sampled;
  sa.out_tok = s->out_tok;
  sa.out_exit = s->out_exit;
  timed(prof, launches, 1, NV_K_STEP, 0, 0, [&] { launch_step_end(sa, st); });
}

// Launches of one decode step after step_begin, all layers in order: the
// profiled path (each launch bracketed by events) and the flat graph.
nv_status record_step(nv_state* s, cudaStream_t st, Prof* prof = nullptr) {
  long long* launches = &s->launches_per_step;
  *launches = 1;  // step_begin, launched outside the graph
  NV_TRY(record_layers(s, st, prof, launches, 0, s->m->L));
  record_step_end(s, st, prof, launches);
  return NV_OK;
}

// The decode-step graph with the layers between two exits in a conditional
// node: a block runs only if some sequence is still active after the
// previous junction (or must complete its deferred rows), so layers that no
// token reaches cost no launches.  Host-side launch count: the unconditional
// part; each block that runs adds its own count on the device.
nv_status build_conditional_step_graph(nv_state* s, cudaGraph_t* out) {
  nv_model* M = s->m;
  cudaGraph_t g = nullptr;
  NV_CUDA_TRY(cudaGraphCreate(&g, 0));
  auto fail = [&](cudaError_t e, const char* what) {
    set_error(std::string(what) + ": " + cudaGetErrorString(e));
    cudaGetLastError();
    cudaGraphDestroy(g);
    return NV_ERR_CUDA;
  };
  std::vector<cudaGraphConditionalHandle> hs(M->NE);
  for (int k = 1; k < M->NE; ++k) {
    cudaError_t e = cudaGraphConditionalHandleCreate(&hs[k], g, 0, cudaGraphCondAssignDefault);
    if (e != cudaSuccess) return fail(e, "cudaGraphConditionalHandleCreate");
  }
  cudaStream_t st = s->cap_stream, st2 = s->cap_stream2;
  cudaError_t e = cudaStreamBeginCaptureToGraph(st, g, nullptr, nullptr, 0, cudaStreamCaptureModeThreadLocal);
  if (e != cudaSuccess) return fail(e, "cudaStreamBeginCaptureToGraph");
  long long host_launches = 1;  // step_begin
  nv_status rs = record_layers(s, st, nullptr, &host_launches, 0, M->cfg.exit_layers[0]);
  for (int k = 1; k < M->NE && rs == NV_OK; ++k) {
    long long block = 0;
    const int l0 = M->cfg.exit_layers[k - 1], l1 = M->cfg.exit_layers[k];
    // the block's launch count is written to d_block_launches[k] after capture
    launch_set_cond(hs[k], s->active, s->force, s->B, s->counters, s->d_block_launches + k, st);
    ++host_launches;
    cudaStreamCaptureStatus cs;
    cudaGraph_t capg = nullptr;
    const cudaGraphNode_t* deps = nullptr;
    const cudaGraphEdgeData* ed = nullptr;
    size_t nd = 0;
    e = cudaStreamGetCaptureInfo_v3(st, &cs, nullptr, &capg, &deps, &ed, &nd);
    if (e != cudaSuccess) {
      rs = NV_ERR_CUDA;
      set_error(std::string("cudaStreamGetCaptureInfo: ") + cudaGetErrorString(e));
      break;
    }
    cudaGraphNodeParams cp = {};
    cp.type = cudaGraphNodeTypeConditional;
    cp.conditional.handle = hs[k];
    cp.conditional.type = cudaGraphCondTypeIf;
    cp.conditional.size = 1;
    cudaGraphNode_t node;
    std::vector<cudaGraphNode_t> dv(deps, deps + nd);
    e = cudaGraphAddNode(&node, capg, dv.data(), nd, &cp);
    if (e == cudaSuccess) e = cudaStreamUpdateCaptureDependencies(st, &node, 1, cudaStreamSetCaptureDependencies);
    if (e != cudaSuccess) {
      rs = NV_ERR_CUDA;
      set_error(std::string("adding a conditional node: ") + cudaGetErrorString(e));
      break;
    }
    e = cudaStreamBeginCaptureToGraph(st2, cp.conditional.phGraph_out[0], nullptr, nullptr, 0,
                                      cudaStreamCaptureModeThreadLocal);
    if (e != cudaSuccess) {
      rs = NV_ERR_CUDA;
      set_error(std::string("capturing a conditional body: ") + cudaGetErrorString(e));
      break;
    }
    rs = record_layers(s, st2, nullptr, &block, l0, l1);
    cudaGraph_t tmp = nullptr;
    e = cudaStreamEndCapture(st2, &tmp);
    if (rs == NV_OK && e != cudaSuccess) {
      rs = NV_ERR_CUDA;
      set_error(std::string("ending a conditional body: ") + cudaGetErrorString(e));
    }
    s->block_launches[k] = block;
  }
  record_step_end(s, st, nullptr, &host_launches);
  cudaGraph_t done = nullptr;
  e = cudaStreamEndCapture(st, &done);
  if (rs != NV_OK) {
    cudaGraphDestroy(g);
    return rs;
  }
  if (e != cudaSuccess) return fail(e, "cudaStreamEndCapture");
  int counts[NV_MAX_EXITS] = {0};
  for (int k = 0; k < M->NE; ++k) counts[k] = (int)s->block_launches[k];
  e = cudaMemcpy(s->d_block_launches, counts, sizeof(counts), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return fail(e, "cudaMemcpy");
  s->launches_per_step = host_launches;
  *out = g;
  return NV_OK;
}

nv_status check_status(nv_state* s) {
  int v = 0;
  NV_CUDA_TRY(cudaMemcpy(&v, s->status, sizeof(int), cudaMemcpyDeviceToHost));
  if (v == DEV_OK) {
    int* g = gemm_status_ptr(s->m->gemm_plans);
    if (g) NV_CUDA_TRY(cudaMemcpy(&v, g, sizeof(int), cudaMemcpyDeviceToHost));
  }
  if (v == DEV_OK) return NV_OK;
  const char* what = v == DEV_ERR_ROWS ? "a per-layer work list exceeded its capacity"
                     : v == DEV_ERR_KV ? "a KV position beyond the page table"
                     : v == DEV_ERR_TIMEOUT ? "a bounded device wait ran out"
                                            : "unknown device error";
  set_error(std::string("device reported: ") + what);
  return v == DEV_ERR_TIMEOUT ? NV_ERR_TIMEOUT : NV_ERR_CAPACITY;
}

// Give sequence b physical pages for positions [0, upto).
nv_status ensure_pages(nv_state* s, int b, int upto, bool* changed) {
  const int need = (upto + s->ps - 1) / s->ps;
  if (need > s->pps) {
    set_error("sequence length exceeds max_seq");
    return NV_ERR_CAPACITY;
  }
  for (int i = 0; i < need; ++i) {
    int& e = s->h_page_table[(size_t)b * s->pps + i];
    if (e < 0) {
      if (s->next_free_page >= s->n_pages) {
        set_error("KV page pool exhausted");
        return NV_ERR_CAPACITY;
      }
      e = s->next_free_page++;
      *changed = true;
    }
  }
  return NV_OK;
}

// Stream-ordered upload of the host page table: copied into a pinned buffer
// (after the previous upload has read it) and sent asynchronously, so a
// decode step that opens a page does not stall the host.
nv_status upload_page_table(nv_state* s, cudaStream_t st) {
  const size_t bytes = s->h_page_table.size() * sizeof(int);
  if (s->pt_pending) NV_CUDA_TRY(cudaEventSynchronize(s->pt_done));
  std::memcpy(s->h_pt_pinned, s->h_page_table.data(), bytes);
  NV_CUDA_TRY(cudaMemcpyAsync(s->page_table, s->h_pt_pinned, bytes, cudaMemcpyHostToDevice, st));
  NV_CUDA_TRY(cudaEventRecord(s->pt_done, st));
  s->pt_pending = true;
  return NV_OK;
}

nv_status validate_config(const nv_config* c) {
  auto bad = [](const char* m) {
    set_error(std::string("invalid config: ") + m);
    return NV_ERR_INVALID_ARG;
  };
  if (!c) return bad("null");
  if (c->n_layers < 1 || c->n_layers > NV_MAX_LAYERS) return bad("n_layers");
  if (c->n_exits < 1 || c->n_exits > NV_MAX_EXITS) return bad("n_exits");
  if (c->d_model < 32 || c->n_heads < 1 || c->d_ff < 1 || c->vocab < 4) return bad("sizes");
  if (c->head_dim != 32 && c->head_dim != 64) return bad("head_dim must be 32 or 64");
  if (c->dtype != NV_F32 && c->dtype != NV_BF16) return bad("dtype");
  const int epc = c->dtype == NV_BF16 ? 8 : 4;
  if (c->d_model % epc || c->d_ff % epc || (c->n_heads * c->head_dim) % epc)
    return bad("d_model, d_ff and n_heads*head_dim must be multiples of 16 bytes");
  if (c->d_model / epc > 256) return bad("d_model too large for the exit-head kernel");
  int prev = 0;
  for (int k = 0; k < c->n_exits; ++k) {
    if (c->exit_layers[k] <= prev || c->exit_layers[k] > c->n_layers) return bad("exit_layers must increase");
    prev = c->exit_layers[k];
  }
  if (prev != c->n_layers) return bad("last exit must follow the last layer");
  if (c->max_batch < 1 || c->max_batch > 16384) return bad("max_batch");
  if (c->max_seq < 2) return bad("max_seq");
  if (c->page_size < ATTN_KT || c->page_size % ATTN_KT) return bad("page_size must be a multiple of 64");
  if (c->max_pending < 2) return bad("max_pending must be >= 2");
  if (c->router_mode != NV_ROUTER_NORMAL && c->router_mode != NV_ROUTER_FORCE_LAST) return bad("router_mode");
  if (c->router_hidden < 0 || c->router_hidden > 1024) return bad("router_hidden must be in [0, 1024]");
  if (c->adapter_hidden < 0 || c->adapter_hidden > 4096) return bad("adapter_hidden must be in [0, 4096]");
  if (c->adapter_hidden && c->dtype == NV_BF16 && c->adapter_hidden % 128) return bad("bf16 adapter_hidden % 128");
  if (!(c->rms_eps > 0.f) || !(c->rope_theta > 1.f)) return bad("rms_eps / rope_theta");
  return NV_OK;
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* nv_last_error(void) { return g_err.c_str(); }

nv_status nv_create(const nv_config* cfg, const nv_weights* w, nv_model** out) {
  if (!out) {
    set_error("out is null");
    return NV_ERR_INVALID_ARG;
  }
  *out = nullptr;
  NV_TRY(validate_config(cfg));
  if (!w || !w->tok_emb || !w->layers || !w->exits) {
    set_error("weights: null pointer");
    return NV_ERR_INVALID_ARG;
  }
  nv_model* M = new nv_model();
  M->cfg = *cfg;
  M->bf16 = cfg->dtype == NV_BF16;
  M->esz = M->bf16 ? 2 : 4;
  M->d = cfg->d_model;
  M->H = cfg->n_heads;
  M->hd = cfg->head_dim;
  M->HQ = M->H * M->hd;
  M->F = cfg->d_ff;
  M->V = cfg->vocab;
  M->L = cfg->n_layers;
  M->NE = cfg->n_exits;
  M->G = (M->F % 64 == 0) ? 64 : M->F;
  M->exit_at.assign(M->L, -1);
  for (int k = 0; k < M->NE; ++k) M->exit_at[cfg->exit_layers[k] - 1] = k;
  const size_t esz = M->esz, d = M->d, HQ = M->HQ, F = M->F, V = M->V;
  for (int i = 0; i < M->L; ++i) {
    const nv_layer_weights& lw = w->layers[i];
    if (!lw.attn_norm || !lw.wq || !lw.wk || !lw.wv || !lw.wo || !lw.mlp_norm || !lw.wg || !lw.wu || !lw.wd) {
      set_error("weights: null layer tensor");
      delete M;
      return NV_ERR_INVALID_ARG;
    }
  }
  const int RH = cfg->router_hidden, AH = cfg->adapter_hidden;
  for (int k = 0; k < M->NE; ++k) {
    const nv_exit_weights& ew = w->exits[k];
    const bool last = k == M->NE - 1;
    const bool router_ok = last || (RH ? (ew.router_w1 && ew.router_b1 && ew.router_w2) : ew.router_w != nullptr);
    const bool head_ok = AH ? (last ? ew.head != nullptr : (ew.adapter_w1 && ew.adapter_w2)) : ew.head != nullptr;
    if (!ew.norm || !head_ok || !router_ok) {
      set_error("weights: null exit tensor");
      delete M;
      return NV_ERR_INVALID_ARG;
    }
  }
  // pool layout
  const size_t A = 256;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, A);
    return o;
  };
  const size_t o_emb = take(V * d * esz);
  std::vector<size_t> o_l(M->L * 6);
  for (int i = 0; i < M->L; ++i) {
    o_l[i * 6 + 0] = take(d * esz);
    o_l[i * 6 + 1] = take(3 * HQ * d * esz);
    o_l[i * 6 + 2] = take(d * HQ * esz);
    o_l[i * 6 + 3] = take(d * esz);
    o_l[i * 6 + 4] = take(2 * F * d * esz);
    o_l[i * 6 + 5] = take(d * F * esz);
  }
  // heads: identical pointers share one packed copy
  std::vector<size_t> o_e(M->NE * 3), o_r(M->NE * 3, 0), o_a(M->NE * 2, 0);
  // with adapters every exit reads the last exit's head: pack it first
  const size_t o_shared = AH ? take(V * d * esz) : 0;
  for (int k = 0; k < M->NE; ++k) {
    o_e[k * 3 + 0] = take(d * esz);
    int same = -1;
    for (int j = 0; j < k; ++j)
      if (w->exits[j].head == w->exits[k].head) same = j;
    o_e[k * 3 + 1] = AH ? o_shared : (same >= 0 ? o_e[same * 3 + 1] : take(V * d * esz));
    if (AH && k < M->NE - 1) {  // adapter W1 [a, d], W2 [d, a]
      o_a[k * 2 + 0] = take((size_t)AH * d * esz);
      o_a[k * 2 + 1] = take((size_t)AH * d * esz);
    }
    o_e[k * 3 + 2] = take(d * esz);
    if (RH && k < M->NE - 1) {  // router MLP: U [r, d], c [r], v [r]
      o_r[k * 3 + 0] = take((size_t)RH * d * esz);
      o_r[k * 3 + 1] = take((size_t)RH * 4);
      o_r[k * 3 + 2] = take((size_t)RH * 4);
    }
  }
  const size_t o_rope = take((size_t)cfg->max_seq * (M->hd / 2) * sizeof(float2));
  nv_status st = dalloc_bytes(&M->pool, off);
  if (st != NV_OK) {
    delete M;
    return st;
  }
  unsigned char* P = (unsigned char*)M->pool;
  auto cp = [&](size_t o, const void* src, size_t bytes) -> nv_status {
    NV_CUDA_TRY(cudaMemcpy(P + o, src, bytes, cudaMemcpyDefault));
    return NV_OK;
  };
#define NV_CP(o, src, bytes)         \
  do {                               \
    nv_status _s = cp(o, src, bytes); \
    if (_s != NV_OK) {               \
      nv_destroy(M);                 \
      return _s;                     \
    }                                \
  } while (0)
  NV_CP(o_emb, w->tok_emb, V * d * esz);
  M->tok_emb = P + o_emb;
  M->layers.resize(M->L);
  for (int i = 0; i < M->L; ++i) {
    const nv_layer_weights& lw = w->layers[i];
    const size_t qkv = o_l[i * 6 + 1], gu = o_l[i * 6 + 4];
    NV_CP(o_l[i * 6 + 0], lw.attn_norm, d * esz);
    NV_CP(qkv, lw.wq, HQ * d * esz);
    NV_CP(qkv + HQ * d * esz, lw.wk, HQ * d * esz);
    NV_CP(qkv + 2 * HQ * d * esz, lw.wv, HQ * d * esz);
    NV_CP(o_l[i * 6 + 2], lw.wo, d * HQ * esz);
    NV_CP(o_l[i * 6 + 3], lw.mlp_norm, d * esz);
    // gate/up interleaved in blocks of G rows: [g0..gG-1, u0..uG-1, gG.., ...]
    const size_t blk = (size_t)M->G * d * esz, nblk = F / M->G;
    cudaError_t e1 = cudaMemcpy2D(P + gu, 2 * blk, lw.wg, blk, blk, nblk, cudaMemcpyDefault);
    cudaError_t e2 = cudaMemcpy2D(P + gu + blk, 2 * blk, lw.wu, blk, blk, nblk, cudaMemcpyDefault);
    if (e1 != cudaSuccess || e2 != cudaSuccess) {
      set_error(std::string("packing gate/up: ") + cudaGetErrorString(e1 != cudaSuccess ? e1 : e2));
      nv_destroy(M);
      return NV_ERR_CUDA;
    }
    NV_CP(o_l[i * 6 + 5], lw.wd, d * F * esz);
    M->layers[i] = LayerDev{P + o_l[i * 6 + 0], P + qkv, P + o_l[i * 6 + 2], P + o_l[i * 6 + 3], P + gu,
                            P + o_l[i * 6 + 5]};
  }
  M->exits.resize(M->NE);
  for (int k = 0; k < M->NE; ++k) {
    const nv_exit_weights& ew = w->exits[k];
    NV_CP(o_e[k * 3 + 0], ew.norm, d * esz);
    if (!AH || k == M->NE - 1) NV_CP(o_e[k * 3 + 1], ew.head, V * d * esz);
    if (k < M->NE - 1 && ew.router_w) NV_CP(o_e[k * 3 + 2], ew.router_w, d * esz);
    M->exits[k] = ExitDev{P + o_e[k * 3 + 0], P + o_e[k * 3 + 1], P + o_e[k * 3 + 2], ew.router_b,
                          nullptr, nullptr, nullptr, nullptr, nullptr};
    if (AH && k < M->NE - 1) {
      NV_CP(o_a[k * 2 + 0], ew.adapter_w1, (size_t)AH * d * esz);
      NV_CP(o_a[k * 2 + 1], ew.adapter_w2, (size_t)AH * d * esz);
      M->exits[k].adapter_w1 = P + o_a[k * 2 + 0];
      M->exits[k].adapter_w2 = P + o_a[k * 2 + 1];
    }
    if (RH && k < M->NE - 1) {
      NV_CP(o_r[k * 3 + 0], ew.router_w1, (size_t)RH * d * esz);
      NV_CP(o_r[k * 3 + 1], ew.router_b1, (size_t)RH * 4);
      NV_CP(o_r[k * 3 + 2], ew.router_w2, (size_t)RH * 4);
      M->exits[k].router_w1 = P + o_r[k * 3 + 0];
      M->exits[k].router_b1 = (const float*)(P + o_r[k * 3 + 1]);
      M->exits[k].router_w2 = (const float*)(P + o_r[k * 3 + 2]);
    }
  }
#undef NV_CP
  M->rope = (float2*)(P + o_rope);
  launch_rope_table(M->rope, cfg->max_seq, M->hd, (double)cfg->rope_theta, 0);
  M->layer_weight_bytes = (long long)(4 * HQ * d + 3 * F * d) * (long long)esz;
  // the tcgen05 engine tiles N by 128 and K by 64: every packed weight of the
  // model must fit (QKV, O, gate/up, down, the heads, the adapters), and the
  // fused QKV epilogue wants whole 128-feature tiles of q, k and v; other
  // bf16 shapes run on the SIMT engine
  const bool tc_shapes = d % 128 == 0 && HQ % 128 == 0 && (2 * F) % 128 == 0 && F % 64 == 0 &&
                         V % 128 == 0 && cfg->adapter_hidden % 128 == 0;
  M->gemm_kind = (M->bf16 && tc_shapes) ? gemm_default_kind() : GEMM_SIMT;
  M->tc_attention = M->gemm_kind == GEMM_TC && M->hd == 64 && M->HQ % 64 == 0 && tc_attention_enabled();
  M->layer_kernel = M->gemm_kind == GEMM_TC && layer_kernel_enabled() &&
                    layer_tc_supported(M->d, M->HQ, M->hd, M->F, M->bf16) && M->G == 64;
  M->gemm_plans = gemm_plans_create();
  // kernels that need more than 48 KB of dynamic shared memory
  nv_status gs = gemm_prepare(M->gemm_kind, M->bf16);
  if (gs == NV_OK && M->layer_kernel) gs = layer_tc_prepare();
  if (gs != NV_OK) {
    nv_destroy(M);
    return gs;
  }
  {
    cudaError_t e2 = kernels_set_smem_limits((size_t)(cfg->max_batch + 1) * 4);
    if (e2 == cudaSuccess && M->bf16 && M->hd == 64) e2 = attn_mma_prepare();
    if (e2 == cudaSuccess && M->bf16 && M->hd == 64) e2 = attn_dec_pc_prepare();
    if (e2 == cudaSuccess && M->tc_attention) e2 = attn_tc_prepare();
    if (e2 == cudaSuccess && cfg->adapter_hidden) e2 = exit_adapter_prepare(M->bf16, M->d, cfg->adapter_hidden);
    if (e2 != cudaSuccess) {
      set_error(std::string("shared memory limits: ") + cudaGetErrorString(e2));
      nv_destroy(M);
      return NV_ERR_UNSUPPORTED;
    }
  }
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    set_error(std::string("nv_create: ") + cudaGetErrorString(e));
    nv_destroy(M);
    return NV_ERR_CUDA;
  }
  *out = M;
  return NV_OK;
}

nv_status nv_destroy(nv_model* M) {
  if (!M) return NV_ERR_INVALID_ARG;
  cudaDeviceSynchronize();
  if (M->pool) cudaFree(M->pool);
  gemm_plans_destroy(M->gemm_plans);
  for (Buf* b : {&M->sc_h, &M->sc_act, &M->sc_u, &M->sc_ctr, &M->sc_q, &M->sc_o, &M->sc_Y, &M->sc_kv, &M->sc_part, &M->sc_z,
                 &M->sc_logpi, &M->sc_logp, &M->sc_i32, &M->sc_nll, &M->sc_depth, &M->sc_mdepth, &M->sc_lse_part,
                 &M->sc_lse_tgt})
    b->release();
  delete M;
  return NV_OK;
}

nv_status nv_state_create(nv_model* M, int B, nv_state** out) {
  if (!M || !out) {
    set_error("null argument");
    return NV_ERR_INVALID_ARG;
  }
  *out = nullptr;
  if (B < 1 || B > M->cfg.max_batch) {
    set_error("B must be in [1, max_batch]");
    return NV_ERR_INVALID_ARG;
  }
  nv_state* s = new nv_state();
  s->m = M;
  s->B = B;
  s->cap = M->cfg.max_pending;
  s->max_seq = M->cfg.max_seq;
  s->ps = M->cfg.page_size;
  s->pps = (s->max_seq + s->ps - 1) / s->ps;
  s->max_rows = B * (s->cap + 1);
  s->n_pages = B * s->pps;
  s->h_page_table.assign((size_t)B * s->pps, -1);
  const size_t esz = M->esz, d = M->d, HQ = M->HQ, F = M->F;
  const size_t page_elems = (size_t)2 * M->H * s->ps * M->hd;
  s->kv_layer_stride = (size_t)s->n_pages * page_elems;
  // attention: 128-key chunks (one CTA each) when rows are 128 bytes and pages
  // hold 64 or 128 positions; otherwise row groups with a few key splits
  s->dec_attn = (size_t)M->hd * M->esz == 128 && (s->ps == 64 || s->ps == 128);
  if (s->dec_attn) {
    s->kv_splits = (s->max_seq + ATTN_DEC_CK - 1) / ATTN_DEC_CK;
  } else {
    int ks = (2 * 148 + B * M->H - 1) / (B * M->H);
    s->kv_splits = ks < 1 ? 1 : (ks > 16 ? 16 : ks);
  }
  s->row_groups = (s->cap + 1 + ATTN_RPC - 1) / ATTN_RPC;
  // the small-batch sampler runs one CTA per SM
  s->head_nblk = tc_sm_count();
  const size_t wide = d > F ? d : F;
  s->Y_elems = gemm_workspace_elems(M->gemm_kind, (size_t)s->max_rows, (size_t)(3 * HQ > 2 * F ? 3 * HQ : 2 * F));
  nv_status st = NV_OK;
  auto A = [&](void** p, size_t bytes) {
    if (st != NV_OK) return;
    st = dalloc_bytes(p, bytes);
    if (st == NV_OK) s->allocs.push_back(*p);
  };
  A(&s->kv, (size_t)M->L * s->kv_layer_stride * esz);
  A((void**)&s->page_table, s->h_page_table.size() * 4);
  for (int** p : {&s->t, &s->tok, &s->active, &s->exit_id, &s->force, &s->sampled, &s->out_tok, &s->out_exit,
                  &s->prompt_len, &s->prompt_last})
    A((void**)p, (size_t)B * 4);
  A((void**)&s->lens, (size_t)B * M->L * 4);
  A((void**)&s->stop, (size_t)B * M->NE * 4);
  A((void**)&s->nstop, (size_t)NV_MAX_EXITS * 4);
  A((void**)&s->d_B, 4);
  A((void**)&s->d_block_launches, NV_MAX_EXITS * 4);
  A((void**)&s->logp, (size_t)B * 4);
  A((void**)&s->router_p, (size_t)NV_MAX_EXITS * B * 4);
  A((void**)&s->hbuf, (size_t)B * s->cap * d * 4);
  for (int** p : {&s->row_b, &s->row_pos, &s->row_hrow}) A((void**)p, (size_t)s->max_rows * 4);
  A((void**)&s->seq_start, (size_t)(B + 1) * 4);
  A((void**)&s->nrows, 4);
  A(&s->act, (size_t)s->max_rows * wide * esz);
  A(&s->u, (size_t)s->max_rows * F * esz);
  A((void**)&s->tile_counters, (size_t)kTileCounters * 4);
  if (M->layer_kernel) {
    s->lt_sync_ints = layer_tc_sync_ints(s->max_rows, M->F);
    A((void**)&s->lt_sync, (size_t)M->L * s->lt_sync_ints * 4);
    A((void**)&s->lt_ygu, layer_tc_gu_floats(M->F) * 4);
  }
  A(&s->q, (size_t)s->max_rows * HQ * esz);
  A(&s->o, (size_t)s->max_rows * HQ * esz);
  A(&s->exit_act, (size_t)B * d * esz);
  A((void**)&s->Y, s->Y_elems * 4);
  A((void**)&s->attn_part, (size_t)s->max_rows * M->H * s->kv_splits * (M->hd + 2) * 4);
  // partials of the sampler (one per CTA) or of the tensor-core head (one per 128 vocab rows)
  A((void**)&s->head_part, (size_t)B * std::max(s->head_nblk, (M->V + 127) / 128) * HEAD_PART * 4);
  A((void**)&s->seed_dev, 8);
  A((void**)&s->counters, NV_CTR_COUNT * 8);
  A((void**)&s->status, 4);
  A((void**)&s->dec_ctr, ((size_t)B * M->H + 2) * 4);
  if (st != NV_OK) {
    nv_state_destroy(s);
    return st;
  }
  cudaMemset(s->counters, 0, NV_CTR_COUNT * 8);
  cudaMemset(s->tile_counters, 0, (size_t)kTileCounters * 4);
  if (s->lt_sync) cudaMemset(s->lt_sync, 0, (size_t)M->L * s->lt_sync_ints * 4);
  cudaMemset(s->nstop, 0, (size_t)NV_MAX_EXITS * 4);
  cudaMemcpy(s->d_B, &B, 4, cudaMemcpyHostToDevice);
  s->tc_head = M->bf16 && M->gemm_kind == GEMM_TC && B >= 16 && M->V % 128 == 0 && M->d % 64 == 0;
  if (!s->tc_head && !head_sample_fits(B, M->d, M->esz)) {
    set_error("nv_state_create: the exit-head sampler has no shared-memory plan for this batch and d_model");
    nv_state_destroy(s);
    return NV_ERR_UNSUPPORTED;
  }
  {
    // the MMA decode attention reads the pool through a tensor map: rows of
    // 128 bytes, boxes of 64 positions, row coordinates within int32
    const uint64_t rows = (uint64_t)M->L * s->kv_layer_stride / 64;
    if (mma_attention_enabled() && s->dec_attn && M->bf16 && M->hd == 64 && rows < (1ull << 31))
      s->kv_map_ok = encode_rows128_map(s->kv, rows, 64, &s->kv_map) == NV_OK;
    if (s->kv_map_ok && dec_pc_attention_enabled())
      s->kv_map32_ok = encode_rows128_map(s->kv, rows, 32, &s->kv_map32) == NV_OK;
    // enough (sequence, head, split) CTAs for two waves of three per SM, each
    // split keeping at least two 64-key tiles
    const int pairs = B * M->H, target = 2 * 3 * 148;
    int sp = (target + pairs - 1) / pairs;
    const int max_sp = std::max(1, (s->max_seq / 64) / 2);
    sp = std::min(sp, std::min(max_sp, s->kv_splits));
    s->dec_splits = std::max(1, sp);
  }
  cudaMemset(s->status, 0, 4);
  cudaMemset(s->dec_ctr, 0, ((size_t)B * M->H + 2) * 4);
  cudaMemset(s->nrows, 0, 4);
  cudaMemset(s->lens, 0, (size_t)B * M->L * 4);
  cudaMemset(s->t, 0, (size_t)B * 4);
  cudaMemset(s->page_table, 0xff, s->h_page_table.size() * 4);
  cudaError_t e = cudaHostAlloc((void**)&s->h_pt_pinned, s->h_page_table.size() * 4, cudaHostAllocDefault);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s->pt_done, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&s->cap_stream, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&s->cap_stream2, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    set_error(std::string("nv_state_create: ") + cudaGetErrorString(e));
    nv_state_destroy(s);
    return NV_ERR_CUDA;
  }
  s->h_t.assign(B, 0);
  *out = s;
  return NV_OK;
}

nv_status nv_state_destroy(nv_state* s) {
  if (!s) return NV_ERR_INVALID_ARG;
  cudaDeviceSynchronize();
  if (s->graph) cudaGraphExecDestroy(s->graph);
  if (s->cap_stream) cudaStreamDestroy(s->cap_stream);
  if (s->cap_stream2) cudaStreamDestroy(s->cap_stream2);
  for (void* p : s->allocs) cudaFree(p);
  for (Buf* b : {&s->pf_rows, &s->pf_h, &s->pf_act, &s->pf_u, &s->pf_q, &s->pf_o, &s->pf_Y, &s->pf_ctr}) b->release();
  if (s->h_pt_pinned) cudaFreeHost(s->h_pt_pinned);
  if (s->pt_done) cudaEventDestroy(s->pt_done);
  delete s;
  return NV_OK;
}

nv_status nv_prefill(nv_state* s, const int32_t* tokens, const int32_t* lens, void* stream) {
  if (!s || !tokens || !lens) {
    set_error("null argument");
    return NV_ERR_INVALID_ARG;
  }
  nv_model* M = s->m;
  cudaStream_t st = (cudaStream_t)stream;
  const int B = s->B;
  size_t total = 0;
  for (int b = 0; b < B; ++b) {
    if (lens[b] < 1 || lens[b] >= s->max_seq) {
      set_error("prompt length must be in [1, max_seq)");
      return NV_ERR_INVALID_ARG;
    }
    total += lens[b];
  }
  std::vector<int> htok(total);
  {
    cudaPointerAttributes pa{};
    const bool on_device = cudaPointerGetAttributes(&pa, tokens) == cudaSuccess &&
                           (pa.type == cudaMemoryTypeDevice || pa.type == cudaMemoryTypeManaged);
    cudaGetLastError();
    if (on_device) {
      NV_CUDA_TRY(cudaMemcpyAsync(htok.data(), tokens, total * 4, cudaMemcpyDeviceToHost, st));
      NV_CUDA_TRY(cudaStreamSynchronize(st));
    } else {
      std::memcpy(htok.data(), tokens, total * 4);
    }
  }
  for (size_t i = 0; i < total; ++i)
    if (htok[i] < 0 || htok[i] >= M->V) {
      set_error("token id out of range");
      return NV_ERR_INVALID_ARG;
    }
  // pages for every prompt position and the first decode position
  std::fill(s->h_page_table.begin(), s->h_page_table.end(), -1);
  s->next_free_page = 0;
  bool changed = false;
  for (int b = 0; b < B; ++b) NV_TRY(ensure_pages(s, b, lens[b], &changed));
  NV_TRY(upload_page_table(s, st));
  // rows: positions 0..P_b-2, in chunks of at most `chunk` rows (a sequence
  // may straddle chunks: a chunk's rows see the earlier chunks' KV at every
  // layer because chunks run through all layers in order)
  const int chunk = 8192;
  std::vector<int> rb, rp, rtok;
  std::vector<size_t> offs(B + 1, 0);
  for (int b = 0; b < B; ++b) offs[b + 1] = offs[b] + lens[b];
  for (int b = 0; b < B; ++b)
    for (int p = 0; p + 1 < lens[b]; ++p) {
      rb.push_back(b);
      rp.push_back(p);
      rtok.push_back(htok[offs[b] + p]);
    }
  const int R = (int)rb.size();
  const size_t wide = M->d > M->F ? M->d : M->F;
  // per-chunk buffers: h, act, q, o, Y, attention partials, row arrays
  const int cr = R < chunk ? (R > 0 ? R : 1) : chunk;
  Buf &h = s->pf_h, &act = s->pf_act, &u = s->pf_u, &q = s->pf_q, &o = s->pf_o, &Y = s->pf_Y, &rows = s->pf_rows,
      &ctr = s->pf_ctr;
  nv_status stt = NV_OK;
  if ((stt = u.need((size_t)cr * M->F * M->esz)) != NV_OK) return stt;
  if ((stt = ctr.need((size_t)kTileCounters * 4)) != NV_OK) return stt;
  NV_CUDA_TRY(cudaMemsetAsync(ctr.p, 0, (size_t)kTileCounters * 4, st));
  if ((stt = h.need((size_t)cr * M->d * 4)) != NV_OK) return stt;
  if ((stt = act.need((size_t)cr * wide * M->esz)) != NV_OK) return stt;
  if ((stt = q.need((size_t)cr * M->HQ * M->esz)) != NV_OK) return stt;
  if ((stt = o.need((size_t)cr * M->HQ * M->esz)) != NV_OK) return stt;
  if ((stt = Y.need(gemm_workspace_elems(M->gemm_kind, cr, 3 * M->HQ > 2 * M->F ? 3 * M->HQ : 2 * M->F) * 4)) != NV_OK)
    return stt;
  if ((stt = rows.need(((size_t)cr * 5 + B + 2) * 4)) != NV_OK) return stt;
  int* d_b = rows.as<int>();
  int* d_pos = d_b + cr;
  int* d_hrow = d_pos + cr;
  int* d_tok = d_hrow + cr;
  int* d_seq = d_tok + cr;
  int* d_n = d_seq + (B + 1);
  std::vector<int> hrow(cr), seq(B + 1);
  for (int i = 0; i < cr; ++i) hrow[i] = i;
  for (int c0 = 0; c0 < R; c0 += chunk) {
    const int n = std::min(chunk, R - c0);
    std::fill(seq.begin(), seq.end(), 0);
    for (int i = 0; i < n; ++i) seq[rb[c0 + i] + 1]++;
    for (int b = 0; b < B; ++b) seq[b + 1] += seq[b];
    NV_CUDA_TRY(cudaMemcpyAsync(d_b, rb.data() + c0, n * 4, cudaMemcpyHostToDevice, st));
    NV_CUDA_TRY(cudaMemcpyAsync(d_pos, rp.data() + c0, n * 4, cudaMemcpyHostToDevice, st));
    NV_CUDA_TRY(cudaMemcpyAsync(d_hrow, hrow.data(), n * 4, cudaMemcpyHostToDevice, st));
    NV_CUDA_TRY(cudaMemcpyAsync(d_tok, rtok.data() + c0, n * 4, cudaMemcpyHostToDevice, st));
    NV_CUDA_TRY(cudaMemcpyAsync(d_seq, seq.data(), (B + 1) * 4, cudaMemcpyHostToDevice, st));
    NV_CUDA_TRY(cudaMemcpyAsync(d_n, &n, 4, cudaMemcpyHostToDevice, st));
    LayerIO io{};
    io.rs = RowSet{d_n, d_b, d_pos, d_hrow, d_seq, h.as<float>(), cr, B};
    io.kv = state_kv(s);
    io.kv_map = s->kv_map_ok ? &s->kv_map : nullptr;
    io.act = act.p;
    io.u = u.p;
    io.tile_counters = ctr.as<int>();
    io.q = q.p;
    io.o = o.p;
    io.Y = Y.as<float>();
    io.attn_part = nullptr;
    io.kv_splits = 1;
    int maxrows_seq = 0;
    for (int b = 0; b < B; ++b) maxrows_seq = std::max(maxrows_seq, seq[b + 1] - seq[b]);
    io.row_groups = (maxrows_seq + ATTN_RPC - 1) / ATTN_RPC;
    io.lens = nullptr;
    io.L = M->L;
    io.epi_grid = 2048;
    launch_embed_rows(M->bf16, M->tok_emb, d_tok, io.rs, M->d, st);
    for (int layer = 0; layer < M->L; ++layer) {
      launch_rmsnorm_rows(M->bf16, io.rs, M->layers[layer].attn_norm, io.act, M->d, M->cfg.rms_eps, st);
      NV_TRY(layer_body(M, layer, io, st));
    }
    NV_CUDA_TRY(cudaStreamSynchronize(st));  // the host row arrays are reused by the next chunk
  }
  if (s->lt_sync) NV_CUDA_TRY(cudaMemsetAsync(s->lt_sync, 0, (size_t)M->L * s->lt_sync_ints * 4, st));
  // decode state after the prompt
  std::vector<int> t0(B), tk(B), ln((size_t)B * M->L);
  for (int b = 0; b < B; ++b) {
    t0[b] = lens[b] - 1;
    tk[b] = htok[offs[b] + lens[b] - 1];
    for (int m = 0; m < M->L; ++m) ln[(size_t)b * M->L + m] = lens[b] - 1;
  }
  NV_CUDA_TRY(cudaMemcpyAsync(s->t, t0.data(), B * 4, cudaMemcpyHostToDevice, st));
  NV_CUDA_TRY(cudaMemcpyAsync(s->tok, tk.data(), B * 4, cudaMemcpyHostToDevice, st));
  NV_CUDA_TRY(cudaMemcpyAsync(s->lens, ln.data(), ln.size() * 4, cudaMemcpyHostToDevice, st));
  NV_CUDA_TRY(cudaMemcpyAsync(s->prompt_len, t0.data(), B * 4, cudaMemcpyHostToDevice, st));
  NV_CUDA_TRY(cudaMemcpyAsync(s->prompt_last, tk.data(), B * 4, cudaMemcpyHostToDevice, st));
  NV_CUDA_TRY(cudaStreamSynchronize(st));
  s->h_prompt_len.assign(lens, lens + B);
  s->h_t = t0;
  s->prefilled = true;
  s->stepped = false;
  return check_status(s);
}

nv_status nv_rewind(nv_state* s, void* stream) {
  if (!s) return NV_ERR_INVALID_ARG;
  if (!s->prefilled) {
    set_error("nv_rewind before nv_prefill");
    return NV_ERR_STATE;
  }
  cudaStream_t st = (cudaStream_t)stream;
  const int B = s->B, L = s->m->L;
  std::vector<int> t0(B), ln((size_t)B * L);
  for (int b = 0; b < B; ++b) {
    t0[b] = s->h_prompt_len[b] - 1;
    for (int m = 0; m < L; ++m) ln[(size_t)b * L + m] = t0[b];
  }
  // counters of the persistent layer kernel start from zero (they are zero
  // after every completed launch; this also clears what an aborted one left)
  if (s->lt_sync) NV_CUDA_TRY(cudaMemsetAsync(s->lt_sync, 0, (size_t)L * s->lt_sync_ints * 4, st));
  NV_CUDA_TRY(cudaMemcpyAsync(s->t, s->prompt_len, B * 4, cudaMemcpyDeviceToDevice, st));
  NV_CUDA_TRY(cudaMemcpyAsync(s->tok, s->prompt_last, B * 4, cudaMemcpyDeviceToDevice, st));
  // lens[b][m] = prompt_len[b] for all m
  NV_CUDA_TRY(cudaMemcpyAsync(s->lens, ln.data(), ln.size() * 4, cudaMemcpyHostToDevice, st));
  NV_CUDA_TRY(cudaStreamSynchronize(st));
  s->h_t = t0;
  s->stepped = false;
  return NV_OK;
}

}  // extern "C"

namespace {
nv_status decode_step_impl(nv_state* s, uint64_t seed, int32_t* tokens_out, int32_t* exits_out, float* logp_out,
                           cudaStream_t st, Prof* prof) {
  if (!s || !tokens_out || !exits_out) {
    set_error("null argument");
    return NV_ERR_INVALID_ARG;
  }
  if (!s->prefilled) {
    set_error("nv_decode_step before nv_prefill");
    return NV_ERR_STATE;
  }
  nv_model* M = s->m;
  // pages for the positions this step writes (every sequence advances by one)
  bool changed = false;
  for (int b = 0; b < s->B; ++b) {
    if (s->h_t[b] + 1 >= s->max_seq) {
      set_error("sequence reached max_seq");
      return NV_ERR_CAPACITY;
    }
    NV_TRY(ensure_pages(s, b, s->h_t[b] + 1, &changed));
  }
  if (changed) NV_TRY(upload_page_table(s, st));
  StepArgs sa{};
  sa.B = s->B;
  sa.L = M->L;
  sa.cap = s->cap;
  sa.d = M->d;
  sa.n_exits = M->NE;
  sa.t = s->t;
  sa.tok = s->tok;
  sa.active = s->active;
  sa.exit_id = s->exit_id;
  sa.force = s->force;
  sa.stop = s->stop;
  sa.nstop = s->nstop;
  sa.router_p = s->router_p;
  sa.lens = s->lens;
  sa.hbuf = s->hbuf;
  sa.emb = M->tok_emb;
  sa.seed_dev = s->seed_dev;
  sa.seed = seed;
  sa.counters = s->counters;
  timed(prof, nullptr, 1, NV_K_STEP, (long long)s->B * M->d * (4 + (long long)M->esz), 0,
        [&] { launch_step_begin(M->bf16, sa, st); });
  if (prof) {
    NV_TRY(record_step(s, st, prof));
  } else {
    if (!s->graph) {
      cudaGraph_t g = nullptr;
      // Conditional blocks pay off when a step may leave an exit block
      // unreached; with 32 or more sequences every block runs in practice
      // (the chance that no token passes an exit is the product of the
      // sequences' stop probabilities), so the step is one flat graph, which
      // saves the conditional nodes' launch latency.  NVIUM_COND_GRAPH=1 / 0
      // forces either form.
      const char* cg = std::getenv("NVIUM_COND_GRAPH");
      const bool want_cond = cg ? cg[0] != '0' : s->B < 32;
      const bool try_cond = want_cond && M->NE > 1;
      if (!try_cond || build_conditional_step_graph(s, &g) != NV_OK) {
        // one flat graph of every layer (conditional nodes unavailable or disabled)
        g = nullptr;
        NV_CUDA_TRY(cudaStreamBeginCapture(s->cap_stream, cudaStreamCaptureModeThreadLocal));
        nv_status rs = record_step(s, s->cap_stream);
        cudaError_t e = cudaStreamEndCapture(s->cap_stream, &g);
        if (rs != NV_OK) {
          if (g) cudaGraphDestroy(g);
          return rs;
        }
        if (e != cudaSuccess) {
          set_error(std::string("capturing the decode step: ") + cudaGetErrorString(e));
          return NV_ERR_CUDA;
        }
        s->cond_graph = false;
      } else {
        s->cond_graph = true;
      }
      cudaError_t e = cudaGraphInstantiate(&s->graph, g, 0);
      cudaGraphDestroy(g);
      if (e != cudaSuccess) {
        set_error(std::string("instantiating the decode step: ") + cudaGetErrorString(e));
        s->graph = nullptr;
        return NV_ERR_CUDA;
      }
    }
    NV_CUDA_TRY(cudaGraphLaunch(s->graph, st));
  }
  s->launches_total += s->launches_per_step;
  NV_CUDA_TRY(cudaMemcpyAsync(tokens_out, s->out_tok, s->B * 4, cudaMemcpyDefault, st));
  NV_CUDA_TRY(cudaMemcpyAsync(exits_out, s->out_exit, s->B * 4, cudaMemcpyDefault, st));
  if (logp_out) NV_CUDA_TRY(cudaMemcpyAsync(logp_out, s->logp, s->B * 4, cudaMemcpyDefault, st));
  for (int b = 0; b < s->B; ++b) s->h_t[b] += 1;
  s->stepped = true;
  return NV_OK;
}
}  // namespace

extern "C" {

nv_status nv_decode_step(nv_state* s, uint64_t seed, int32_t* tokens_out, int32_t* exits_out, float* logp_out,
                         void* stream) {
  return decode_step_impl(s, seed, tokens_out, exits_out, logp_out, (cudaStream_t)stream, nullptr);
}

nv_status nv_decode_step_profiled(nv_state* s, uint64_t seed, int32_t* tokens_out, int32_t* exits_out,
                                  nv_kernel_stat* stats, void* stream) {
  if (!stats) {
    set_error("null argument");
    return NV_ERR_INVALID_ARG;
  }
  Prof prof;
  prof.st = (cudaStream_t)stream;
  NV_TRY(decode_step_impl(s, seed, tokens_out, exits_out, nullptr, prof.st, &prof));
  NV_CUDA_TRY(cudaStreamSynchronize(prof.st));
  for (const Prof::Rec& r : prof.recs) {
    float ms = 0.f;
    NV_CUDA_TRY(cudaEventElapsedTime(&ms, r.a, r.b));
    nv_kernel_stat& k = stats[r.kind];
    k.ms += ms;
    k.launches += 1;
    k.kernels += r.kernels;
    k.bytes += r.bytes;
    k.flops += r.flops;
  }
  return NV_OK;
}

nv_status nv_flush_deferred(nv_state* s, void* stream) {
  if (!s) return NV_ERR_INVALID_ARG;
  if (!s->prefilled) {
    set_error("nv_flush_deferred before nv_prefill");
    return NV_ERR_STATE;
  }
  nv_model* M = s->m;
  cudaStream_t st = (cudaStream_t)stream;
  LayerIO io = state_io(s);
  long long launches = 0;
  for (int layer = M->cfg.exit_layers[0]; layer < M->L; ++layer) {
    if (layer == M->cfg.exit_layers[0] || M->exit_at[layer - 1] >= 0) {
      PlanArgs p = state_plan(s, layer, 1);
      p.nlayers = block_layers(M, layer);
      launch_plan_norm(M->bf16, p, M->layers[layer].attn_norm, s->act, M->d, M->cfg.rms_eps, plan_grid(s), st);
      ++launches;
    }
    const bool block_start = layer == M->cfg.exit_layers[0] || M->exit_at[layer - 1] >= 0;
    NV_TRY(layer_body(M, layer, io, st, nullptr, &launches, next_norm_in_block(M, layer), !block_start));
  }
  s->launches_total += launches;
  NV_CUDA_TRY(cudaGetLastError());
  return NV_OK;
}

nv_status nv_read_kv(nv_state* s, int b, int layer, void* k_out, void* v_out, int* len_out, void* stream) {
  if (!s || !k_out || !v_out || !len_out) {
    set_error("null argument");
    return NV_ERR_INVALID_ARG;
  }
  nv_model* M = s->m;
  if (b < 0 || b >= s->B || layer < 0 || layer >= M->L) {
    set_error("b or layer out of range");
    return NV_ERR_INVALID_ARG;
  }
  cudaStream_t st = (cudaStream_t)stream;
  NV_CUDA_TRY(cudaStreamSynchronize(st));
  int len = 0;
  NV_CUDA_TRY(cudaMemcpy(&len, s->lens + (size_t)b * M->L + layer, 4, cudaMemcpyDeviceToHost));
  *len_out = len;
  const size_t row = (size_t)M->hd * M->esz;
  for (int pos = 0; pos < len; pos += s->ps) {
    const int page = s->h_page_table[(size_t)b * s->pps + pos / s->ps];
    if (page < 0) {
      set_error("KV position without a page");
      return NV_ERR_STATE;
    }
    const int n = std::min(s->ps, len - pos);
    for (int kv = 0; kv < 2; ++kv)
      for (int h = 0; h < M->H; ++h) {
        const unsigned char* src = (const unsigned char*)s->kv +
                                   ((size_t)layer * s->kv_layer_stride +
                                    (((size_t)page * 2 + kv) * M->H + h) * (size_t)s->ps * M->hd) *
                                       M->esz;
        unsigned char* dst = (unsigned char*)(kv ? v_out : k_out) + ((size_t)pos * M->H + h) * row;
        // n positions of one head: source stride hd, destination stride H*hd
        NV_CUDA_TRY(cudaMemcpy2DAsync(dst, (size_t)M->H * row, src, row, row, n, cudaMemcpyDefault, st));
      }
  }
  NV_CUDA_TRY(cudaStreamSynchronize(st));
  return NV_OK;
}

nv_status nv_read_router_probs(nv_state* s, float* w_out, void* stream) {
  if (!s || !w_out) {
    set_error("null argument");
    return NV_ERR_INVALID_ARG;
  }
  if (!s->stepped) {
    set_error("nv_read_router_probs before the first decode step");
    return NV_ERR_STATE;
  }
  const int n = (s->m->NE - 1) * s->B;
  if (n == 0) return NV_OK;
  cudaStream_t st = (cudaStream_t)stream;
  NV_CUDA_TRY(cudaMemcpyAsync(w_out, s->router_p, (size_t)n * 4, cudaMemcpyDeviceToHost, st));
  NV_CUDA_TRY(cudaStreamSynchronize(st));
  return NV_OK;
}

nv_status nv_read_counters(nv_state* s, int64_t* out, int n) {
  if (!s || !out || n < 1) {
    set_error("null argument");
    return NV_ERR_INVALID_ARG;
  }
  if (n > NV_CTR_COUNT) n = NV_CTR_COUNT;
  NV_CUDA_TRY(cudaDeviceSynchronize());
  NV_CUDA_TRY(cudaMemcpy(out, s->counters, (size_t)n * 8, cudaMemcpyDeviceToHost));
  // launches: the host's count plus the conditional blocks counted on the device
  if (n > NV_CTR_LAUNCHES) out[NV_CTR_LAUNCHES] += s->launches_total;
  return NV_OK;
}

nv_status nv_reset_counters(nv_state* s) {
  if (!s) return NV_ERR_INVALID_ARG;
  NV_CUDA_TRY(cudaDeviceSynchronize());
  NV_CUDA_TRY(cudaMemset(s->counters, 0, NV_CTR_COUNT * 8));
  s->launches_total = 0;
  return NV_OK;
}

nv_status nv_philox4x32_10(uint64_t seed, const uint32_t* ctr, int n, uint32_t* out, void* stream) {
  if (!ctr || !out || n < 1) {
    set_error("null argument");
    return NV_ERR_INVALID_ARG;
  }
  cudaStream_t st = (cudaStream_t)stream;
  void* d = nullptr;
  NV_TRY(dalloc_bytes(&d, (size_t)n * 32));
  unsigned char* din = (unsigned char*)d;
  unsigned char* dout = din + (size_t)n * 16;
  cudaError_t e = cudaMemcpyAsync(din, ctr, (size_t)n * 16, cudaMemcpyDefault, st);
  if (e == cudaSuccess) {
    launch_philox(seed, din, n, dout, st);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaMemcpyAsync(out, dout, (size_t)n * 16, cudaMemcpyDefault, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  cudaFree(d);
  if (e != cudaSuccess) {
    set_error(std::string("nv_philox4x32_10: ") + cudaGetErrorString(e));
    return NV_ERR_CUDA;
  }
  return NV_OK;
}

nv_status nv_sync_status(nv_state* s) {
  if (!s) return NV_ERR_INVALID_ARG;
  NV_CUDA_TRY(cudaDeviceSynchronize());
  return check_status(s);
}

}  // extern "C"

namespace {
nv_status score_impl(nv_model* M, const int32_t* tokens, int B, int S, float* logp, float* mean_nll, cudaStream_t st,
                     Prof* prof, float* depth = nullptr, float* mean_depth = nullptr) {
  if (!M || !tokens || !logp) {
    set_error("null argument");
    return NV_ERR_INVALID_ARG;
  }
  if (B < 1 || S < 2 || S > M->cfg.max_seq) {
    set_error("need B >= 1 and 2 <= S <= max_seq");
    return NV_ERR_INVALID_ARG;
  }
  const int Sm = S - 1;               // positions 0..S-2 predict tokens 1..S-1
  const long long R64 = (long long)B * Sm;
  if (R64 > (1LL << 26)) {
    set_error("B*(S-1) too large");
    return NV_ERR_CAPACITY;
  }
  const int R = (int)R64, NE = M->NE;
  std::vector<int> htok((size_t)B * S);
  NV_CUDA_TRY(cudaMemcpy(htok.data(), tokens, htok.size() * 4, cudaMemcpyDefault));
  for (int v : htok)
    if (v < 0 || v >= M->V) {
      set_error("token id out of range");
      return NV_ERR_INVALID_ARG;
    }
  const int ps = ATTN_KT;
  const int pps = (S + ps - 1) / ps;
  const size_t wide = M->d > M->F ? M->d : M->F;
  const int head_chunk = std::min(R, 4096);
  const int AH = M->cfg.adapter_hidden;
  const size_t y_layers = gemm_workspace_elems(
      M->gemm_kind, R, std::max<size_t>(3 * M->HQ > 2 * M->F ? 3 * M->HQ : 2 * M->F, (size_t)AH));
  // tcgen05 engine: the head GEMM's epilogue reduces the logits of each
  // 128-token tile to (max, sum exp) and picks the target logit, so logits
  // never reach memory; the SIMT engine writes one chunk of logits at a time
  const bool fused_lse = M->gemm_kind == GEMM_TC && M->V % 128 == 0;
  const int lse_nblk = M->V / 128;
  const size_t y_head = fused_lse ? 0 : gemm_workspace_elems(M->gemm_kind, head_chunk, M->V);
  if (fused_lse) {
    NV_TRY(M->sc_lse_part.need((size_t)R * lse_nblk * sizeof(float2)));
    NV_TRY(M->sc_lse_tgt.need((size_t)R * 4));
  }
  NV_TRY(M->sc_h.need((size_t)R * M->d * 4));
  NV_TRY(M->sc_act.need((size_t)R * wide * M->esz));
  NV_TRY(M->sc_u.need((size_t)R * std::max<size_t>(M->F, (size_t)AH) * M->esz));
  if (!M->sc_ctr.p) {
    NV_TRY(M->sc_ctr.need((size_t)kTileCounters * 4));
    NV_CUDA_TRY(cudaMemset(M->sc_ctr.p, 0, (size_t)kTileCounters * 4));
  }
  NV_TRY(M->sc_q.need((size_t)R * M->HQ * M->esz));
  NV_TRY(M->sc_o.need((size_t)R * M->HQ * M->esz));
  NV_TRY(M->sc_Y.need(std::max(y_layers, y_head) * 4));
  NV_TRY(M->sc_kv.need((size_t)B * pps * 2 * M->HQ * ps * M->esz));
  NV_TRY(M->sc_z.need((size_t)R * (NE > 1 ? NE - 1 : 1) * 4));
  NV_TRY(M->sc_logpi.need((size_t)R * NE * 4));
  NV_TRY(M->sc_logp.need((size_t)R * 4));
  NV_TRY(M->sc_nll.need(4));
  if (depth || mean_depth) {
    NV_TRY(M->sc_depth.need((size_t)R * 4));
    NV_TRY(M->sc_mdepth.need(4));
  }
  const int nchunks = (R + head_chunk - 1) / head_chunk;
  NV_TRY(M->sc_i32.need(((size_t)R * 5 + B + 2 + (size_t)B * pps + nchunks) * 4));
  int* d_b = M->sc_i32.as<int>();
  int* d_pos = d_b + R;
  int* d_hrow = d_pos + R;
  int* d_tok = d_hrow + R;
  int* d_tgt = d_tok + R;
  int* d_seq = d_tgt + R;
  int* d_n = d_seq + (B + 1);
  int* d_pt = d_n + 1;
  int* d_chunk = d_pt + (size_t)B * pps;
  {
    std::vector<int> hb(R), hp(R), hr(R), ht(R), hg(R), hs(B + 1), hpt((size_t)B * pps), hc(nchunks);
    for (int b = 0; b < B; ++b) {
      hs[b] = b * Sm;
      for (int p = 0; p < Sm; ++p) {
        const int r = b * Sm + p;
        hb[r] = b;
        hp[r] = p;
        hr[r] = r;
        ht[r] = htok[(size_t)b * S + p];
        hg[r] = htok[(size_t)b * S + p + 1];
      }
      for (int i = 0; i < pps; ++i) hpt[(size_t)b * pps + i] = b * pps + i;
    }
    hs[B] = R;
    for (int c = 0; c < nchunks; ++c) hc[c] = std::min(head_chunk, R - c * head_chunk);
    NV_CUDA_TRY(cudaMemcpyAsync(d_b, hb.data(), R * 4, cudaMemcpyHostToDevice, st));
    NV_CUDA_TRY(cudaMemcpyAsync(d_pos, hp.data(), R * 4, cudaMemcpyHostToDevice, st));
    NV_CUDA_TRY(cudaMemcpyAsync(d_hrow, hr.data(), R * 4, cudaMemcpyHostToDevice, st));
    NV_CUDA_TRY(cudaMemcpyAsync(d_tok, ht.data(), R * 4, cudaMemcpyHostToDevice, st));
    NV_CUDA_TRY(cudaMemcpyAsync(d_tgt, hg.data(), R * 4, cudaMemcpyHostToDevice, st));
    NV_CUDA_TRY(cudaMemcpyAsync(d_seq, hs.data(), (B + 1) * 4, cudaMemcpyHostToDevice, st));
    NV_CUDA_TRY(cudaMemcpyAsync(d_n, &R, 4, cudaMemcpyHostToDevice, st));
    NV_CUDA_TRY(cudaMemcpyAsync(d_pt, hpt.data(), hpt.size() * 4, cudaMemcpyHostToDevice, st));
    NV_CUDA_TRY(cudaMemcpyAsync(d_chunk, hc.data(), nchunks * 4, cudaMemcpyHostToDevice, st));
    NV_CUDA_TRY(cudaStreamSynchronize(st));  // host vectors go out of scope
  }
  LayerIO io{};
  io.rs = RowSet{d_n, d_b, d_pos, d_hrow, d_seq, M->sc_h.as<float>(), R, B};
  io.kv.base = M->sc_kv.p;
  io.kv.layer_stride = 0;  // one layer's KV at a time
  io.kv.page_table = d_pt;
  io.kv.pages_per_seq = pps;
  io.kv.page_size = ps;
  io.kv.H = M->H;
  io.kv.hd = M->hd;
  CUtensorMap sc_map;
  {
    const uint64_t rows = (uint64_t)B * pps * 2 * M->HQ * ps / 64;
    if (mma_attention_enabled() && M->bf16 && M->hd == 64 && ps % 64 == 0 && rows < (1ull << 31) &&
        encode_rows128_map(M->sc_kv.p, rows, 64, &sc_map) == NV_OK)
      io.kv_map = &sc_map;
  }
  io.act = M->sc_act.p;
  io.u = M->sc_u.p;
  io.tile_counters = M->sc_ctr.as<int>();
  io.q = M->sc_q.p;
  io.o = M->sc_o.p;
  io.Y = M->sc_Y.as<float>();
  io.attn_part = nullptr;
  io.kv_splits = 1;
  io.row_groups = (Sm + ATTN_RPC - 1) / ATTN_RPC;
  io.lens = nullptr;
  io.L = M->L;
  io.epi_grid = 4096;
  const long long es = (long long)M->esz;
  if (prof) {
    prof->R = R;
    // causal attention: row p reads K and V of positions 0..p
    prof->kv_read = (long long)B * Sm * (Sm + 1) / 2 * 2 * M->HQ * es;
  }
  timed(prof, nullptr, 1, NV_K_STEP, 0, 0, [&] { launch_embed_rows(M->bf16, M->tok_emb, d_tok, io.rs, M->d, st); });
  for (int layer = 0; layer < M->L; ++layer) {
    timed(prof, nullptr, 1, NV_K_NORM, (long long)R * M->d * (4 + es), 0, [&] {
      launch_rmsnorm_rows(M->bf16, io.rs, M->layers[layer].attn_norm, io.act, M->d, M->cfg.rms_eps, st);
    });
    NV_TRY(layer_body(M, layer, io, st, prof, nullptr));
    const int k = M->exit_at[layer];
    if (k < 0) continue;
    timed(prof, nullptr, 1, NV_K_JUNCTION, (long long)R * M->d * (4 + es), 0, [&] {
      launch_exit_rows(M->bf16, io.rs, M->exits[k], M->cfg.router_hidden, k, NE, io.act,
                       M->sc_z.as<float>(), M->d, M->cfg.rms_eps, st);
    });
    if (AH && k < NE - 1) {
      // exit adapter before the shared head: hidden = silu(n_k W1^T), then
      // act = final RMSNorm of h + hidden W2^T
      nv_status ast = NV_OK;
      timed(prof, nullptr, gemm_launch_count(M->gemm_kind, M->bf16, false, nullptr) * 2 + 2, NV_K_HEAD,
            2LL * AH * M->d * es, 4LL * R * AH * M->d, [&] {
              ast = gemm_run(M->gemm_plans, M->gemm_kind, M->bf16, io.act, M->d, M->exits[k].adapter_w1, AH, M->d,
                             io.rs.nrows, io.rs.max_rows, io.Y, false, nullptr, io.tile_counters, io.epi_grid,
                             nullptr, 0, st);
              if (ast != NV_OK) return;
              launch_silu_rows(M->bf16, io.rs.nrows, io.Y, AH, io.u, io.rs.max_rows, st);
              ast = gemm_run(M->gemm_plans, M->gemm_kind, M->bf16, io.u, AH, M->exits[k].adapter_w2, M->d, AH,
                             io.rs.nrows, io.rs.max_rows, io.Y, false, nullptr, io.tile_counters, io.epi_grid,
                             nullptr, 0, st);
              if (ast != NV_OK) return;
              launch_adapter_norm_rows(M->bf16, io.rs, io.Y, M->exits[NE - 1].norm, io.act, M->d, M->cfg.rms_eps,
                                       st);
            });
      NV_TRY(ast);
    }
    if (fused_lse) {
      EpiArgs le{};
      le.mode = EPI_LSE;
      le.lse_target = d_tgt;
      le.lse_part = M->sc_lse_part.as<float2>();
      le.lse_tgt = M->sc_lse_tgt.as<float>();
      le.nblk = lse_nblk;
      nv_status hst = NV_OK;
      timed(prof, nullptr, 2, NV_K_HEAD, (long long)M->V * M->d * es + (long long)R * M->d * es,
            2LL * R * M->V * M->d, [&] {
              hst = gemm_run(M->gemm_plans, M->gemm_kind, M->bf16, io.act, M->d, M->exits[k].head, M->V, M->d,
                             io.rs.nrows, io.rs.max_rows, io.Y, false, &le, nullptr, 0, nullptr, 0, st);
              launch_lse_combine(le.lse_part, le.lse_tgt, R, lse_nblk, M->sc_logpi.as<float>(), k, NE, st);
            });
      NV_TRY(hst);
      continue;
    }
    for (int c = 0; c < nchunks; ++c) {
      const int r0 = c * head_chunk;
      const long long rc = std::min(head_chunk, R - r0);
      nv_status hst = NV_OK;
      timed(prof, nullptr, 2, NV_K_HEAD, (long long)M->V * M->d * es + rc * M->d * es + rc * M->V * 4,
            2 * rc * M->V * M->d, [&] {
              hst = gemm_run(M->gemm_plans, M->gemm_kind, M->bf16,
                             (const unsigned char*)io.act + (size_t)r0 * M->d * M->esz, M->d, M->exits[k].head, M->V,
                             M->d, d_chunk + c, head_chunk, io.Y, false, nullptr, nullptr, 0, nullptr, 0, st);
              launch_lse_target(io.Y, r0, (int)rc, M->V, d_tgt, M->sc_logpi.as<float>(), k, NE, st);
            });
      NV_TRY(hst);
    }
  }
  ExitFrac ef{};
  for (int k = 0; k < NE; ++k) ef.f[k] = (float)M->cfg.exit_layers[k] / (float)M->L;
  const bool want_depth = depth || mean_depth;
  const int mix_kernels = 1 + 1 + (want_depth ? 1 : 0);
  timed(prof, nullptr, mix_kernels, NV_K_STEP, 0, 0, [&] {
    launch_mixture(M->sc_z.as<float>(), M->sc_logpi.as<float>(), R, NE, M->cfg.router_mode, M->sc_logp.as<float>(),
                   M->sc_nll.as<float>(), want_depth ? M->sc_depth.as<float>() : nullptr,
                   want_depth ? M->sc_mdepth.as<float>() : nullptr, ef, st);
  });
  NV_CUDA_TRY(cudaMemcpyAsync(logp, M->sc_logp.p, (size_t)R * 4, cudaMemcpyDefault, st));
  if (mean_nll) NV_CUDA_TRY(cudaMemcpyAsync(mean_nll, M->sc_nll.p, 4, cudaMemcpyDefault, st));
  if (depth) NV_CUDA_TRY(cudaMemcpyAsync(depth, M->sc_depth.p, (size_t)R * 4, cudaMemcpyDefault, st));
  if (mean_depth) NV_CUDA_TRY(cudaMemcpyAsync(mean_depth, M->sc_mdepth.p, 4, cudaMemcpyDefault, st));
  NV_CUDA_TRY(cudaGetLastError());
  return NV_OK;
}
}  // namespace

extern "C" {

nv_status nv_score_mixture(nv_model* M, const int32_t* tokens, int B, int S, float* logp, float* mean_nll,
                           void* stream) {
  return score_impl(M, tokens, B, S, logp, mean_nll, (cudaStream_t)stream, nullptr);
}

nv_status nv_score_mixture_ex(nv_model* M, const int32_t* tokens, int B, int S, float* logp, float* mean_nll,
                              float* depth, float* mean_depth, void* stream) {
  return score_impl(M, tokens, B, S, logp, mean_nll, (cudaStream_t)stream, nullptr, depth, mean_depth);
}

nv_status nv_score_mixture_profiled(nv_model* M, const int32_t* tokens, int B, int S, float* logp, float* mean_nll,
                                    nv_kernel_stat* stats, void* stream) {
  if (!stats) {
    set_error("null argument");
    return NV_ERR_INVALID_ARG;
  }
  Prof prof;
  prof.st = (cudaStream_t)stream;
  NV_TRY(score_impl(M, tokens, B, S, logp, mean_nll, prof.st, &prof));
  NV_CUDA_TRY(cudaStreamSynchronize(prof.st));
  for (const Prof::Rec& r : prof.recs) {
    float ms = 0.f;
    NV_CUDA_TRY(cudaEventElapsedTime(&ms, r.a, r.b));
    nv_kernel_stat& k = stats[r.kind];
    k.ms += ms;
    k.launches += 1;
    k.kernels += r.kernels;
    k.bytes += r.bytes;
    k.flops += r.flops;
  }
  return NV_OK;
}

}  // extern "C"
