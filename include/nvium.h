/*
 * nvium.h -- C ABI of libnvium, a B200 (sm_100a) implementation of the
 * N-vium mixture-of-exits decode hot path.
 *
 * Source of the method: "N-vium: Mixture-of-Exits Transformer for
 * Accelerated Exact Generation" (Lorenc, Berdoz, Mathys, Wattenhofer;
 * arXiv 2605.13190), as summarised on gist.science (technical summary,
 * sections 1-5) and in the paper's abstract.
 *
 *   - Section 2 "Architektur": the L backbone layers are split into N_V
 *     blocks; after block k a router gives the stop probability w_k, the exit
 *     probability is p_k = w_k prod_{j<k}(1 - w_j) with w_{N_V} = 1, and the
 *     next-token law is the mixture pi_mix = sum_k p_k pi_k.
 *   - Section 2 "Inferenz: Piggybacking": a token exiting at node k defers
 *     its layers above the exit; later tokens that reach those depths carry
 *     the deferred rows in the same batched pass, so the KV cache ends
 *     complete and exact.
 *   - Section 3 and the abstract: sampling from the mixture is exact.
 *   - Section 5: zero routing mass on the intermediate heads recovers the
 *     standard transformer exactly.
 *
 * Conventions for every call:
 *   - Pointers marked "host or device" may point to either; the library
 *     copies through unified addressing.  Pointers marked "device" must be
 *     device memory of the current device.
 *   - The caller owns every buffer it passes; the library owns models,
 *     states, KV pools and packed weights.
 *   - Each call returns an nv_status.  Nothing throws or aborts across the
 *     ABI.  Argument errors are detected on the host before any launch and
 *     leave the object unchanged.  Errors a kernel detects (an index out of
 *     range, a bounded wait that ran out) are written to the state's device
 *     status word and returned by the next call on that state that
 *     synchronises, or by nv_sync_status.
 *   - nv_last_error() returns a thread-local message for the last failure.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     are asynchronous on that stream unless noted.
 *   - Results are deterministic: the same config, weights, inputs and seeds
 *     give bit-identical outputs (no float atomics; fixed reduction order).
 */
#ifndef NVIUM_H
#define NVIUM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define NV_MAX_EXITS 8
#define NV_MAX_LAYERS 256

typedef enum {
  NV_OK = 0,
  NV_ERR_INVALID_ARG = -1, /* bad pointer, size or config field            */
  NV_ERR_OOM = -2,         /* device allocation failed                     */
  NV_ERR_CUDA = -3,        /* a CUDA runtime call failed                   */
  NV_ERR_CAPACITY = -4,    /* batch, sequence or row capacity exceeded     */
  NV_ERR_TIMEOUT = -5,     /* a bounded device wait ran out                */
  NV_ERR_STATE = -6,       /* call not valid in the object's current state */
  NV_ERR_UNSUPPORTED = -7  /* shape the kernels do not cover               */
} nv_status;

enum { NV_F32 = 0, NV_BF16 = 1 };

/* Routing modes.  NV_ROUTER_FORCE_LAST sets w_1..w_{N_V-1} := 0 exactly
 * (section 5: the standard transformer is recovered exactly). */
enum { NV_ROUTER_NORMAL = 0, NV_ROUTER_FORCE_LAST = 1 };

/* Model and capacity description (section 2 "Architektur"; LLaMA-2 backbone,
 * section 4).  exit_layers[k] (1-based) is the layer after which exit k+1
 * reads the residual stream; strictly increasing, last == n_layers,
 * exit_layers[0] >= 1.  dtype is the element type of every weight tensor and
 * of the KV cache; NV_F32 models compute in fp32 throughout, NV_BF16 models
 * round every input of a product with a bf16 weight or cache to bf16 and
 * accumulate in fp32 (the residual stream is fp32).
 * max_seq bounds prompt + generated length per sequence; max_pending bounds
 * the deferred positions a sequence may hold (a sequence that reaches it has
 * its deferred rows completed early, which does not change any value).
 * page_size is the KV page length in tokens (a multiple of 64). */
typedef struct nv_config {
  int n_layers, d_model, n_heads, head_dim, d_ff, vocab, n_exits;
  int exit_layers[NV_MAX_EXITS];
  int dtype;
  float rms_eps;    /* RMSNorm epsilon, 1e-5 for LLaMA-2          */
  float rope_theta; /* RoPE base, 10000 for LLaMA-2               */
  int max_batch, max_seq, page_size, max_pending;
  int router_mode;
  /* 0: scalar router (router_w, router_b).  r in [1, 1024]: a router MLP of
   * hidden width r on the exit-normalised state (section 2 "Architektur":
   * "a router MLP"), z = router_w2 . silu(router_w1 n_k + router_b1) +
   * router_b; router_w is then unused. */
  int router_hidden;
  /* 0: every exit has its own norm and head.  a > 0: the exits share one LM
   * head, the last exit's (section 2 "Architektur": a shared head with light
   * adapter MLPs): exit k < N_V's head reads the final RMSNorm (the last
   * exit's norm) of m = h + adapter_w2 silu(adapter_w1 n_k), n_k still
   * feeding the router.  a in [1, 4096]; bf16 models need a % 128 == 0. */
  int adapter_hidden;
} nv_config;

/* One backbone layer.  Row-major, PyTorch "out x in" convention (y = x W^T).
 * wq, wk, wv: [n_heads*head_dim, d_model]; wo: [d_model, n_heads*head_dim];
 * wg, wu: [d_ff, d_model]; wd: [d_model, d_ff]; norms: [d_model].
 * Host or device pointers, element type = config dtype. */
typedef struct nv_layer_weights {
  const void *attn_norm, *wq, *wk, *wv, *wo;
  const void *mlp_norm, *wg, *wu, *wd;
} nv_layer_weights;

/* One exit: its RMSNorm gain [d_model], its linear head [vocab, d_model], and
 * for k < N_V its sigmoid router w_k = sigma(z) on the exit-normalised state
 * n_k: z = router_w . n_k + router_b (router_w [d_model]), or with
 * router_hidden = r > 0 the router MLP z = router_w2 . silu(router_w1 n_k +
 * router_b1) + router_b (router_w1 [r, d_model] in the model dtype,
 * router_b1 and router_w2 [r] float; silu(x) = x sigmoid(x)).  Router fields
 * are ignored for the last exit.  Giving every exit the same `head` pointer
 * shares one head. */
typedef struct nv_exit_weights {
  const void *norm, *head, *router_w;
  float router_b;
  const void *router_w1;
  const float *router_b1, *router_w2;
  /* adapter_hidden = a > 0, exits before the last: adapter_w1 [a, d_model],
   * adapter_w2 [d_model, a] (model dtype); `head` is then read from the last
   * exit only. */
  const void *adapter_w1, *adapter_w2;
} nv_exit_weights;

typedef struct nv_weights {
  const void *tok_emb;              /* [vocab, d_model]   */
  const nv_layer_weights *layers;   /* [n_layers]         */
  const nv_exit_weights *exits;     /* [n_exits]          */
} nv_weights;

typedef struct nv_model nv_model;
typedef struct nv_state nv_state;

/* Validate the config, copy and pack the weights onto the current device
 * (fused QKV, interleaved gate/up), and build the RoPE table.  The caller may
 * free its weight buffers when this returns.  Synchronous. */
nv_status nv_create(const nv_config *cfg, const nv_weights *w, nv_model **out);
nv_status nv_destroy(nv_model *m);

/* Mixture scoring (section 2: pi_mix, and the cross-entropy of pi_mix that
 * training minimises).  tokens [B, S] int32 row-major (host or device).
 * logp [B, S-1] float (host or device): logp[b][t] = log pi_mix(x_{t+1} |
 * x_{<=t}) = logsumexp_k(log p_k + log pi_k(x_{t+1})).  mean_nll (host or
 * device, may be NULL) = -mean(logp).  S >= 2, S <= max_seq, B >= 1.
 * Synchronous with respect to `stream` when an output is host memory. */
nv_status nv_score_mixture(nv_model *m, const int32_t *tokens, int B, int S,
                           float *logp, float *mean_nll, void *stream);

/* nv_score_mixture plus the forward of the compute penalty (section 2
 * "Training": L_compute is the expected normalised layer depth).  depth
 * [B, S-1] float (host or device, may be NULL): depth[b][t] = sum_k p_k *
 * exit_layers[k] / n_layers with the exit probabilities p_k of position t
 * (those used by logp[b][t]); mean_depth (host or device, may be NULL) =
 * mean(depth).  Other arguments, results and errors as nv_score_mixture. */
nv_status nv_score_mixture_ex(nv_model *m, const int32_t *tokens, int B, int S,
                              float *logp, float *mean_nll, float *depth,
                              float *mean_depth, void *stream);

/* A decode state for B sequences (B <= max_batch): paged KV cache with its own
 * length per (sequence, layer), deferred-row store, work lists, CUDA graph.
 * *out (host) receives the state, owned by the caller until nv_state_destroy.
 * NV_ERR_INVALID_ARG for a null argument or B outside [1, max_batch];
 * NV_ERR_OOM / NV_ERR_CUDA when device memory or a CUDA call fails;
 * NV_ERR_UNSUPPORTED when the small-batch exit-head sampler has no
 * shared-memory plan for B and d_model (not reached by any configuration
 * nv_create accepts).  On error *out is NULL. */
nv_status nv_state_create(nv_model *m, int B, nv_state **out);
nv_status nv_state_destroy(nv_state *s);

/* Prefill: for sequence b with prompt length P_b >= 1 (lens, host [B]),
 * positions 0..P_b-2 run at full depth and fill every layer's KV; position
 * P_b-1 becomes the first decode input.  tokens: the prompts packed back to
 * back, sum(P_b) int32 (host or device).  P_b + generated tokens must stay
 * <= max_seq. */
nv_status nv_prefill(nv_state *s, const int32_t *tokens, const int32_t *lens,
                     void *stream);

/* Return the state to what nv_prefill left (the prompt KV is kept; decode
 * writes only beyond it).  Lets one prompt be decoded many times. */
nv_status nv_rewind(nv_state *s, void *stream);

/* One decode step for every sequence (section 2 "Inferenz: Piggybacking";
 * section 3 "exact sampling").  Each sequence's input token runs layer by
 * layer; at exit k its router gives w_k and the step stops there iff
 * u_k < w_k (u_k = Philox4x32-10 uniform, key = philox_seed, counter =
 * (b, t, 0, (k-1)/4), lane (k-1)%4); the token is then
 * argmax_v(logit_k[v] + Gumbel(U_v)), U_v from counter (b, t, 1, v/4), lane
 * v%4, ties to the lowest id.  Layers above the exit are deferred; at each
 * layer the deferred rows of a sequence whose new token reaches that layer
 * run in the same packed pass.  With adapter_hidden > 0 the logits come
 * from the shared head applied to the exit's adapter output.  Outputs (host
 * or device, [B]): tokens_out = sampled ids, exits_out = exit used (1..N_V),
 * logp_out (may be NULL) = log pi_exit(token). */
nv_status nv_decode_step(nv_state *s, uint64_t philox_seed, int32_t *tokens_out,
                         int32_t *exits_out, float *logp_out, void *stream);

/* Run every deferred row through the layers it still owes, so that every
 * layer's KV covers all positions (section 2: complete KV recovery). */
nv_status nv_flush_deferred(nv_state *s, void *stream);

/* Copy sequence b's layer `layer` (0-based) K and V cache, positions
 * [0, len), as [len][n_heads][head_dim] of the config dtype into k_out/v_out
 * (host or device, each max_seq*n_heads*head_dim elements), and the length
 * into *len_out (host).  Synchronous. */
nv_status nv_read_kv(nv_state *s, int b, int layer, void *k_out, void *v_out,
                     int *len_out, void *stream);

/* Test hook: the router probabilities of the last decode step (section 2
 * "Architektur": w_k of exit k's router).  w_out (host, (n_exits-1) x B
 * float, exit-major): w_out[(k-1)*B + b] = the w_k that sequence b's token
 * compared its uniform u_k against at junction k, as the kernel computed it
 * (0 under NV_ROUTER_FORCE_LAST), or NaN when that token stopped before
 * junction k.  Lets a caller check every stop decision against the device's
 * own w_k (stop iff u_k < w_k) and measure |w_k - w_k(reference)|.
 * Returns NV_ERR_STATE before the first decode step.  Synchronous. */
nv_status nv_read_router_probs(nv_state *s, float *w_out, void *stream);

/* Per-state counters, int64, accumulated since nv_state_create or the last
 * nv_reset_counters (synchronous).  Indices: see NV_CTR_*. */
enum {
  NV_CTR_STEPS = 0,          /* decode steps                               */
  NV_CTR_ROWS = 1,           /* layer-rows computed (decode + flush)       */
  NV_CTR_LAYERS_RUN = 2,     /* layers with at least one row               */
  NV_CTR_WEIGHT_BYTES = 3,   /* layer weight bytes read, once per layer run */
  NV_CTR_KV_READ_BYTES = 4,  /* KV bytes attention must read               */
  NV_CTR_KV_WRITE_BYTES = 5, /* KV bytes written                           */
  NV_CTR_HEAD_BYTES = 6,     /* exit-head weight bytes read                */
  NV_CTR_FORCED = 7,         /* sequence-steps with an early completion    */
  NV_CTR_LAUNCHES = 8,       /* kernels launched by decode steps and flush */
  NV_CTR_EXIT0 = 16,         /* 16..16+N_V-1: exits taken, per exit        */
  NV_CTR_COUNT = 24
};
nv_status nv_read_counters(nv_state *s, int64_t *out, int n);
nv_status nv_reset_counters(nv_state *s);

/* Test hook for the counter-based generator that every random draw above
 * uses: out[i] = Philox4x32-10(counter = ctr[i][0..3], key = (seed low 32
 * bits, seed high 32 bits)) (Salmon et al., "Parallel Random Numbers: As Easy
 * as 1, 2, 3", SC'11).  ctr, out: n x 4 uint32 (host or device).
 * Synchronous. */
nv_status nv_philox4x32_10(uint64_t seed, const uint32_t *ctr, int n,
                           uint32_t *out, void *stream);

/* The same generator as nv_philox4x32_10, for callers that cannot allocate
 * device memory.  The paper has no counterpart: this is a service of the
 * library, not a step of the method.
 *
 * Some callers cannot call cudaMalloc: a host framework whose caching
 * allocator already holds the device's memory (a fresh allocation fails or
 * fragments it), or a latency-critical loop that cannot afford the
 * device-wide synchronisation cudaMalloc / cudaFree may imply.
 * nv_philox4x32_10 allocates a staging buffer on every call; this entry
 * point allocates nothing.  It stages counters and results through a fixed
 * array of 2 * NV_PHILOX_NOALLOC_MAX * 16 bytes (1 MiB) in device global
 * memory, which every GPU that loads the library holds until the process
 * exits.
 *
 * ctr, out: n x 4 uint32 (host or device); 1 <= n <= NV_PHILOX_NOALLOC_MAX,
 * larger n returns NV_ERR_INVALID_ARG with a message.  The first call on a
 * device looks up the array's device address once, with that device
 * current, and keeps it for the life of the process.  A cudaDeviceReset (or
 * any reset of the primary context) unloads the array, so the kept address
 * is no longer valid: do not call this entry point on that device again
 * after such a reset.  All calls share the array and it keeps the last
 * call's contents, so calls that overlap on the GPU (other streams, other
 * host threads) race; serialise them.  Synchronous: the call waits for its
 * stream, so it cannot be recorded into a stream capture. */
#define NV_PHILOX_NOALLOC_MAX 32768
nv_status nv_philox4x32_10_noalloc(uint64_t seed, const uint32_t *ctr, int n,
                                   uint32_t *out, void *stream);

/* Self-test of the bounded-wait rule that every wait in the library's
 * kernels follows (a wait on an mbarrier or flag gives up after a time
 * limit, records a timeout in the device status word and returns, leaving
 * the CUDA context usable).  One thread waits on a shared-memory mbarrier
 * that nothing completes, for at most limit_us microseconds (1 ..
 * 1000000; else NV_ERR_INVALID_ARG), and *expired_out is set to 1 when the
 * wait gave up (the expected outcome), 0 otherwise.  No copy is in flight
 * while it waits.  Synchronous on `stream`.  The paper has no counterpart:
 * it is failure-detection test infrastructure. */
nv_status nv_selftest_bounded_wait(int limit_us, int *expired_out, void *stream);

/* Per-kernel timing of one decode step (a measurement hook, not a second
 * code path): the step's kernels are launched directly on `stream`, each
 * call bracketed by CUDA events, instead of as one graph replay; the step's
 * results are identical.  stats[kind] accumulates, for NV_K_* kinds, the
 * summed event time, the calls (`launches`: one GEMM with its split-K sum
 * epilogue is one call), the kernels those calls launched (`kernels`), and
 * the algorithmic bytes (the bytes the kernel must move: weights once, K/V
 * of the attended positions once, activations in and out) and flops of those
 * calls.  Synchronous. */
typedef struct nv_kernel_stat {
  double ms;
  int64_t launches;
  int64_t bytes;
  int64_t flops;
  int64_t kernels;
} nv_kernel_stat;
enum {
  NV_K_PLAN_NORM = 0, /* work-list planner + attention RMSNorm    */
  NV_K_GEMM = 1,      /* packed-row GEMMs (tcgen05 or SIMT)       */
  NV_K_EPILOGUE = 2,  /* RoPE/KV write, residual, SwiGLU          */
  NV_K_ATTENTION = 3, /* paged attention (+ split combine)        */
  NV_K_NORM = 4,      /* MLP RMSNorm                              */
  NV_K_JUNCTION = 5,  /* exit norm, router, stop draw             */
  NV_K_HEAD = 6,      /* exit-head sampler (+ reduce)             */
  NV_K_STEP = 7,      /* step begin / end                         */
  NV_K_COUNT = 8
};
nv_status nv_decode_step_profiled(nv_state *s, uint64_t philox_seed,
                                  int32_t *tokens_out, int32_t *exits_out,
                                  nv_kernel_stat *stats, void *stream);

/* nv_score_mixture with the same per-kernel timing (NV_K_GEMM: the layer
 * GEMMs with their fused epilogues, NV_K_HEAD: exit-head GEMM + log-sum-exp,
 * NV_K_ATTENTION: causal attention, ...); flops are the GEMMs' 2*rows*N*K.
 * Results are those of nv_score_mixture.  Synchronous. */
nv_status nv_score_mixture_profiled(nv_model *m, const int32_t *tokens, int B,
                                    int S, float *logp, float *mean_nll,
                                    nv_kernel_stat *stats, void *stream);

/* Synchronise the state's work and return any device-detected error. */
nv_status nv_sync_status(nv_state *s);

/* The calling thread's most recent error message (thread-local): every failing
 * call records one, except a null-handle rejection, which only returns
 * NV_ERR_INVALID_ARG.  The pointer stays valid until that thread records the
 * next message; never NULL. */
const char *nv_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* NVIUM_H */
