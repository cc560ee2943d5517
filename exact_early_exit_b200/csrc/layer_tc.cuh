// Persistent decode-layer kernel (sm_100a): everything of one backbone layer
// after its attention, for the packed rows of a decode step or a flush, in
// one launch of one CTA per SM.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"

namespace nv {

// Which parts a launch runs.
enum LayerTcFlags : int {
  LT_MLP = 1,    // output projection + residual + MLP norm, gate/up + SwiGLU, down projection
  LT_NORM2 = 2,  // after the down projection: residual + the next layer's attention norm (else residual only)
  LT_QKV = 4,    // QKV projection of `qkv` (RoPE, q out, K/V into the cache of kv_layer)
};

// Integers of device scratch one launch site needs (counters and per-tile
// ready flags); zero between launches.
size_t layer_tc_sync_ints(int max_rows, int F);
// floats of the gate/up split-slice buffer (gate/up splits only when all
// rows fit one 256-row tile)
size_t layer_tc_gu_floats(int F);

struct LayerTcRun {
  // weights (bf16): this layer's O, gate/up, down and norm gains; the QKV
  // weight of the layer whose projection LT_QKV runs
  const void *w_o, *w_gu, *w_d, *mlp_norm;
  const void *w_qkv, *norm2;
  int kv_layer;
  // row set and buffers of the state
  RowSet rs;
  KVView kv;
  const float2* rope;
  void *o, *act, *u, *q;
  float* Y;
  float* Ygu;  // gate/up split slices: layer_tc_gu_floats(F) floats
  int* sync;
  int* status;
  int d, HQ, H, hd, F;
  float eps;
  int flags;
};

// True when the model's shapes fit the kernel (bf16, head_dim 64, d and
// H*head_dim multiples of 128, d <= 2048, F a multiple of 64).
bool layer_tc_supported(int d, int HQ, int hd, int F, bool bf16);
nv_status layer_tc_prepare();
nv_status layer_tc_launch(TcPlanCache* plans, const LayerTcRun& r, cudaStream_t st);

}  // namespace nv
