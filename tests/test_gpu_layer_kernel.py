"""The persistent decode-layer kernel (one launch per layer after attention:
output projection, residual and MLP norm, gate/up with SwiGLU, down
projection, residual and the next layer's norm and QKV) against the
per-kernel path it replaces (NVIUM_LAYER_KERNEL=0): same split counts,
reduction orders and per-element arithmetic, so every sampled token, exit,
log-probability and every KV entry after the flush must be bit-identical.

Cases: the small bf16 model (ragged batch), the 1.5B shapes cut to 4 layers
(d 1536, F 4096, B 64), and flushes whose deferred rows exceed one 256-row
tile (several row tiles, no split)."""
import dataclasses
import os

import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu

nv = pytest.importorskip("exact_early_exit_b200")


def _decode(cfg, weights, prompts, steps, layer_kernel, max_pending=256, seed=77):
    os.environ["NVIUM_LAYER_KERNEL"] = "1" if layer_kernel else "0"
    try:
        lens = np.array([len(p) for p in prompts], np.int32)
        max_seq = int(lens.max()) + steps + 8
        model = nv.Model(cfg, weights, max_batch=len(prompts), max_seq=max_seq, max_pending=max_pending)
    finally:
        os.environ.pop("NVIUM_LAYER_KERNEL", None)
    B = len(prompts)
    st = nv.State(model, B)
    st.prefill(np.concatenate(prompts).astype(np.int32), lens)
    tok, ex, lp = np.zeros(B, np.int32), np.zeros(B, np.int32), np.zeros(B, np.float32)
    out = []
    for s in range(steps):
        st.decode_step(seed + s, tok, ex, lp)
        out.append((tok.copy(), ex.copy(), lp.copy()))
    st.flush()
    st.sync_status()
    kv = {}
    for b in range(B):
        for m in range(cfg.n_layers):
            K, V, n = st.read_kv(b, m, max_seq)
            kv[b, m] = (K.copy(), V.copy(), n)
    c = st.counters()
    st.close()
    model.close()
    return out, kv, c


def _same(a, b):
    out1, kv1, c1 = a
    out2, kv2, c2 = b
    for s, ((t1, e1, l1), (t2, e2, l2)) in enumerate(zip(out1, out2)):
        np.testing.assert_array_equal(e1, e2, err_msg=f"exits, step {s}")
        np.testing.assert_array_equal(t1, t2, err_msg=f"tokens, step {s}")
        np.testing.assert_array_equal(l1.view(np.uint32), l2.view(np.uint32), err_msg=f"log-probs, step {s}")
    assert kv1.keys() == kv2.keys()
    for key in kv1:
        K1, V1, n1 = kv1[key]
        K2, V2, n2 = kv2[key]
        assert n1 == n2, key
        np.testing.assert_array_equal(K1, K2, err_msg=f"K {key}")
        np.testing.assert_array_equal(V1, V2, err_msg=f"V {key}")
    assert c1[nv.CTR["rows"]] == c2[nv.CTR["rows"]]
    # the persistent path launches fewer kernels for the same work
    assert c1[nv.CTR["launches"]] < c2[nv.CTR["launches"]]


def test_small_model_ragged_batch_bit_identical():
    cfg = W.SMALL
    w = W.make_weights(cfg, seed=0)
    wl = W.WORKLOADS["S"]
    prompts = [p[:n] for p, n in zip(W.make_prompts(wl, seed=9), (64, 3, 130, 17, 1, 90, 257, 40))]
    _same(_decode(cfg, w, prompts, 20, True), _decode(cfg, w, prompts, 20, False))


def test_15b_shapes_4_layers_b64_bit_identical():
    cfg = dataclasses.replace(W.X15B, name="x15b-4layers", n_layers=4, exit_layers=(1, 2, 3, 4))
    w = W.make_weights(cfg, seed=0)
    rng = np.random.default_rng(3)
    lens = rng.integers(8, 96, size=64)
    prompts = W.make_prompts(W.WORKLOADS["X64"], lengths=lens)
    _same(_decode(cfg, w, prompts, 6, True), _decode(cfg, w, prompts, 6, False))


def test_flush_of_more_than_one_row_tile_bit_identical():
    """Every token stops at the first exit (router bias +30), so each sequence
    owes the upper layers for all its decoded positions: the flush then runs
    8 x 40 = 320 rows per layer, two row tiles of the persistent kernel."""
    cfg = W.SMALL
    w = W.make_weights(cfg, seed=0, router_bias=[30.0, 0.0, 0.0])
    wl = W.WORKLOADS["S"]
    prompts = [p[:n] for p, n in zip(W.make_prompts(wl, seed=2), (20, 5, 33, 64, 7, 12, 50, 2))]
    a = _decode(cfg, w, prompts, 40, True)
    assert all((e == 1).all() for _, e, _ in a[0])
    _same(a, _decode(cfg, w, prompts, 40, False))
