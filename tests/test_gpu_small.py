"""GPU parity on the small bf16 model (12 layers, d=768, 12 heads, vocab
32000, exits after layers 3/6/9/12), tcgen05 GEMM path.  Tolerance 2e-2."""
import os

import numpy as np
import pytest

import workloads as W
from oracle import nvium_oracle as O
from tests.nvium_testlib import run_decode_parity, tolerance

pytestmark = pytest.mark.gpu

nv = pytest.importorskip("exact_early_exit_b200")
CFG = W.SMALL


@pytest.fixture(scope="module")
def weights():
    return W.make_weights(CFG, seed=0)


def test_scoring_matches_oracle(weights):
    wl = W.WORKLOADS["S"]
    toks = np.stack([W.make_prompts(wl, seed=s)[0][:96] for s in (1, 2)]).astype(np.int32)
    model = nv.Model(CFG, weights, max_batch=1, max_seq=128)
    logp = np.zeros((2, 95), np.float32)
    nll = np.zeros(1, np.float32)
    depth = np.zeros((2, 95), np.float32)
    mean_depth = np.zeros(1, np.float32)
    model.score_mixture_ex(toks, logp, nll, depth, mean_depth)
    ref, ref_nll, ref_depth, ref_mean_depth = O.score_mixture_with_depth(O.OracleModel(CFG, weights), toks)
    np.testing.assert_allclose(logp, ref, atol=2e-2, rtol=0)
    assert abs(nll[0] - ref_nll) <= 2e-2
    np.testing.assert_allclose(depth, ref_depth, atol=2e-2, rtol=0)
    assert abs(mean_depth[0] - ref_mean_depth) <= 2e-2


def test_decode_parity_b4(weights):
    wl = W.WORKLOADS["S"]
    prompts = [p[:n] for p, n in zip(W.make_prompts(wl), (64, 33, 100, 7))]
    chk, state, dec, _ = run_decode_parity(nv, CFG, weights, prompts, 24)
    chk.report("B=4")
    # every stop decision followed the device's own w_k; a tie needs u_k to
    # fall between the two w_k, which happens with probability |dw|
    assert chk.exit_ties <= 2 + 4 * chk.expected_exit_ties
    c = state.counters()
    assert c[nv.CTR["steps"]] == 24


def test_simt_and_tcgen05_engines_agree(weights):
    toks = np.stack([W.make_prompts(W.WORKLOADS["S"], seed=5)[0][:80]]).astype(np.int32)
    out = {}
    for eng in ("simt", "tc"):
        os.environ["NVIUM_GEMM"] = eng
        try:
            m = nv.Model(CFG, weights, max_batch=1, max_seq=128)
        finally:
            os.environ.pop("NVIUM_GEMM", None)
        lp = np.zeros((1, 79), np.float32)
        m.score_mixture(toks, lp)
        out[eng] = lp
        m.close()
    np.testing.assert_allclose(out["simt"], out["tc"], atol=5e-3, rtol=0)



def test_prefill_kv_matches_oracle(weights):
    """Every layer's K and V right after prefill (full-depth rows, before any
    decode step) against the oracle's prefill caches."""
    from tests.nvium_testlib import gpu_kv, kv_close
    wl = W.WORKLOADS["S"]
    prompts = [p[:n] for p, n in zip(W.make_prompts(wl, seed=4), (70, 5, 129))]
    lens = np.array([len(p) for p in prompts], np.int32)
    model = nv.Model(CFG, weights, max_batch=3, max_seq=160)
    st = nv.State(model, 3)
    st.prefill(np.concatenate(prompts), lens)
    dec = O.OracleDecoder(O.OracleModel(CFG, weights), prompts, 4)
    for b in range(3):
        for m in range(CFG.n_layers):
            K, V, n = gpu_kv(st, b, m, 160, CFG)
            assert n == lens[b] - 1
            kv_close(K, dec.caches[b].K[m][:n], CFG)
            kv_close(V, dec.caches[b].V[m][:n], CFG)


def test_decode_parity_b16_tensor_core_head(weights):
    """16 sequences: the exit heads run as tcgen05 GEMMs with the sampling
    epilogue (Gumbel-max and log-sum-exp per 128-token tile)."""
    wl = W.WORKLOADS["S"]
    rng = np.random.default_rng(12)
    prompts = [p[:int(n)] for p, n in zip(W.make_prompts(wl, seed=6), rng.integers(3, 40, size=16))]
    chk, state, dec, _ = run_decode_parity(nv, CFG, weights, prompts, 8)
    chk.report("B=16")
    assert chk.exit_ties <= 2 + 4 * chk.expected_exit_ties
    assert chk.steps == 8


def test_sampler_chi_square_bf16_tensor_core_head():
    """Exact sampling through the tensor-core head: 4096 copies of one
    context on a 2-layer bf16 model (vocab 1024), 50 seeds; joint (exit,
    token) frequencies against p_k * pi_k(v) from the oracle."""
    from tests.nvium_testlib import chisq_pvalue
    mini = W.ModelConfig("mini-bf16", 2, 256, 4, 64, 512, 1024, (1, 2), W.BF16)
    w = W.make_weights(mini, seed=3, router_bias=[0.3])
    prompt = W.zipf_ids(6, mini.vocab, np.random.default_rng(2))
    B = 4096
    model = nv.Model(mini, w, max_batch=B, max_seq=16, max_pending=4)
    st = nv.State(model, B)
    st.prefill(np.tile(prompt, B).astype(np.int32), np.full(B, len(prompt), np.int32))
    counts = np.zeros((2, mini.vocab))
    tok = np.zeros(B, np.int32)
    ex = np.zeros(B, np.int32)
    for s in range(50):
        st.decode_step(2000 + s, tok, ex)
        np.add.at(counts, (ex - 1, tok), 1)
        st.rewind()
    om = O.OracleModel(mini, w)
    _, states, _ = om.forward_sequence(prompt)
    t = len(prompt) - 1
    p, pi = O.step_distribution(om, [states[k][t:t + 1] for k in range(2)])
    n = counts.sum()
    assert chisq_pvalue(counts, p[:, None] * pi * n) > 0.01
    assert chisq_pvalue(counts.sum(1), p * n) > 0.01


def test_mma_and_simt_decode_attention_agree(weights):
    """The warp-MMA decode attention (bf16 P as a hi/lo pair) and the SIMT one
    give the same step outputs on ragged prompts spanning several 128-key
    chunks, with deferred rows (several rows per sequence and layer)."""
    wl = W.WORKLOADS["S"]
    lens = np.array([300, 129, 64, 517], np.int64)
    prompts = [p[:n] for p, n in zip(W.make_prompts(wl, lengths=[600] * 4), lens)]
    out = {}
    for eng in ("simt", "mma"):
        if eng == "simt":
            os.environ["NVIUM_ATTN"] = "simt"
        try:
            m = nv.Model(CFG, weights, max_batch=4, max_seq=640)
            st = nv.State(m, 4)
        finally:
            os.environ.pop("NVIUM_ATTN", None)
        st.prefill(np.concatenate(prompts).astype(np.int32), lens)
        toks, exs, lps = [], [], []
        tok, ex, lp = np.zeros(4, np.int32), np.zeros(4, np.int32), np.zeros(4, np.float32)
        for s in range(24):
            st.decode_step(1000 + s, tok, ex, lp)
            toks.append(tok.copy()); exs.append(ex.copy()); lps.append(lp.copy())
        st.flush()
        st.sync_status()
        out[eng] = (np.array(toks), np.array(exs), np.array(lps))
        st.close()
        m.close()
    (t0, e0, l0), (t1, e1, l1) = out["simt"], out["mma"]
    # a near tie could flip one draw and then the rest of that sequence
    same = np.cumprod((t0 == t1) & (e0 == e1), axis=0).astype(bool)
    assert same.mean() >= 0.9, same.mean()
    # different fp32 summation orders flip bf16 roundings of attention outputs,
    # which propagate through the layers: the bound is the path's tolerance
    np.testing.assert_allclose(l0[same], l1[same], atol=tolerance(CFG), rtol=0)


def _decode_run(cfg, w, prompts, steps, max_seq, env):
    """Decode `steps` steps and flush with the environment `env` set while the
    model is built; returns tokens, exits, log-probs and every layer's KV."""
    for k, v in env.items():
        os.environ[k] = v
    try:
        m = nv.Model(cfg, w, max_batch=len(prompts), max_seq=max_seq)
        st = nv.State(m, len(prompts))
    finally:
        for k in env:
            os.environ.pop(k, None)
    B = len(prompts)
    st.prefill(np.concatenate(prompts).astype(np.int32), np.array([len(p) for p in prompts], np.int32))
    toks, exs, lps = [], [], []
    tok, ex, lp = np.zeros(B, np.int32), np.zeros(B, np.int32), np.zeros(B, np.float32)
    for s in range(steps):
        st.decode_step(1000 + s, tok, ex, lp)
        toks.append(tok.copy()); exs.append(ex.copy()); lps.append(lp.copy())
    st.flush()
    st.sync_status()
    kv = {(b, l): st.read_kv(b, l, max_seq) for b in range(B) for l in range(cfg.n_layers)}
    st.close()
    m.close()
    return np.array(toks), np.array(exs), np.array(lps), kv


def test_persistent_and_per_head_decode_attention_agree(weights):
    """Decode attention on persistent warps (items of 16 rows x a key chunk,
    taken from a counter, chunks merged by the last arrival) against one CTA
    per (sequence, head): ragged prompts spanning several chunks, 64 sequences
    (several items per warp), then a flush
    whose sequences owe 40 deferred rows each (three 16-row passes), every
    token having stopped at the first exit."""
    wl = W.WORKLOADS["S"]
    lens = np.array([300, 129, 64, 517], np.int64)
    prompts = [p[:n] for p, n in zip(W.make_prompts(wl, lengths=[600] * 4), lens)]
    a = _decode_run(CFG, weights, prompts, 24, 640, {})
    b = _decode_run(CFG, weights, prompts, 24, 640, {"NVIUM_DEC_ATTN": "pc"})
    same = np.cumprod((a[0] == b[0]) & (a[1] == b[1]), axis=0).astype(bool)
    assert same.mean() >= 0.9, same.mean()
    np.testing.assert_allclose(a[2][same], b[2][same], atol=tolerance(CFG), rtol=0)

    # 64 sequences: several items per warp, so each warp's ring streams
    # across item boundaries
    lens = np.random.default_rng(4).integers(200, 600, size=64)
    prompts = W.make_prompts(wl, lengths=lens)
    a = _decode_run(CFG, weights, prompts, 6, 640, {})
    b = _decode_run(CFG, weights, prompts, 6, 640, {"NVIUM_DEC_ATTN": "pc"})
    same = np.cumprod((a[0] == b[0]) & (a[1] == b[1]), axis=0).astype(bool)
    assert same.mean() >= 0.9, same.mean()
    np.testing.assert_allclose(a[2][same], b[2][same], atol=tolerance(CFG), rtol=0)

    w30 = W.make_weights(CFG, seed=0, router_bias=[30.0, 0.0, 0.0])
    prompts = [p[:n] for p, n in zip(W.make_prompts(wl, seed=2), (20, 5, 33, 64))]
    a = _decode_run(CFG, w30, prompts, 40, 128, {})
    b = _decode_run(CFG, w30, prompts, 40, 128, {"NVIUM_DEC_ATTN": "pc"})
    assert (a[1] == 1).all() and (b[1] == 1).all()
    # a near tie may flip a draw (different summation orders): compare each
    # sequence's cache up to its first differing token
    diff = a[0] != b[0]
    assert diff.mean() <= 0.05, diff.mean()
    first = np.where(diff.any(0), diff.argmax(0), 40)
    for (bq, layer), (K1, V1, n1) in a[3].items():
        K2, V2, n2 = b[3][bq, layer]
        assert n1 == n2, (bq, layer)
        n = n1 if first[bq] == 40 else len(prompts[bq]) + first[bq] - 1
        np.testing.assert_allclose(W.as_f32(K1[:n]), W.as_f32(K2[:n]), atol=2e-2, rtol=2 ** -7, err_msg=str((bq, layer)))
        np.testing.assert_allclose(W.as_f32(V1[:n]), W.as_f32(V2[:n]), atol=2e-2, rtol=2 ** -7, err_msg=str((bq, layer)))


def test_mma_and_simt_scoring_attention_agree(weights):
    """Flash-style MMA attention (64-row query tiles, 64-key tiles, online
    softmax) and the SIMT row-group kernel score the same sequences alike:
    several query and key tiles, ragged tails (700 = 10 x 64 + 60)."""
    toks = np.stack([W.make_prompts(W.WORKLOADS["S"], seed=s, lengths=[701])[0] for s in (3, 4)]).astype(np.int32)
    out = {}
    for eng in ("simt", "mma"):
        if eng == "simt":
            os.environ["NVIUM_ATTN"] = "simt"
        try:
            m = nv.Model(CFG, weights, max_batch=1, max_seq=704)
        finally:
            os.environ.pop("NVIUM_ATTN", None)
        lp = np.zeros((2, 700), np.float32)
        m.score_mixture(toks, lp)
        out[eng] = lp
        m.close()
    assert np.all(np.isfinite(out["mma"]))
    np.testing.assert_allclose(out["mma"], out["simt"], atol=tolerance(CFG), rtol=0)


def test_sampler_many_rows_at_one_exit_bf16():
    """Twelve sequences that all stop at the first exit (router bias +30): the
    small-batch sampler takes twelve stopped rows in one pass, its Gumbel
    draws in two rounds over a warp's lanes (four lanes per row).  Tokens,
    exits and log-probs against the oracle, then every cache after the flush."""
    w = W.make_weights(CFG, seed=0, router_bias=[30.0, 0.0, 0.0])
    wl = W.WORKLOADS["S"]
    prompts = [p[:n] for p, n in zip(W.make_prompts(wl, seed=5, lengths=[40] * 12), range(5, 41, 3))]
    chk, state, dec, _ = run_decode_parity(nv, CFG, w, prompts, 6, max_pending=8)
    chk.report("B=12, every row at exit 1")
    assert chk.steps == 6


def test_decode_parity_bf16_degenerate_and_ragged_prompts(weights):
    """A one-token prompt (no prefill rows), one ending a 64-row query tile
    plus one row, and one spanning several key tiles, through the MMA
    attention kernels."""
    wl = W.WORKLOADS["S"]
    prompts = [p[:n] for p, n in zip(W.make_prompts(wl), (1, 65, 130))]
    chk, state, dec, _ = run_decode_parity(nv, CFG, weights, prompts, 12)
    assert chk.steps == 12


def test_router_mlp_bf16_scoring_and_decode_match_oracle():
    """Router MLP of width 64 on the bf16 model: scoring and decode parity."""
    import dataclasses
    cfg = dataclasses.replace(CFG, router_hidden=64)
    w = W.make_weights(cfg, seed=0)
    wl = W.WORKLOADS["S"]
    toks = np.stack([W.make_prompts(wl, seed=s)[0][:80] for s in (1, 2)]).astype(np.int32)
    model = nv.Model(cfg, w, max_batch=1, max_seq=128)
    logp = np.zeros((2, 79), np.float32)
    model.score_mixture(toks, logp)
    ref, _ = O.score_mixture(O.OracleModel(cfg, w), toks)
    np.testing.assert_allclose(logp, ref, atol=tolerance(cfg), rtol=0)
    model.close()
    prompts = [p[:n] for p, n in zip(W.make_prompts(wl), (40, 9, 70))]
    chk, *_ = run_decode_parity(nv, cfg, w, prompts, 12)
    assert chk.steps == 12


@pytest.mark.parametrize("batch", [3, 16])
def test_shared_head_with_adapters_bf16_matches_oracle(batch):
    """Shared head behind adapters of width 128 on the bf16 model: scoring
    (tcgen05 GEMMs for the adapters) and decode, with the SIMT head (B=3) and
    the tensor-core head (B=16)."""
    import dataclasses
    cfg = dataclasses.replace(CFG, adapter_hidden=128)
    w = W.make_weights(cfg, seed=0)
    wl = W.WORKLOADS["S"]
    if batch == 3:
        toks = np.stack([W.make_prompts(wl, seed=s)[0][:80] for s in (1, 2)]).astype(np.int32)
        model = nv.Model(cfg, w, max_batch=1, max_seq=128)
        logp = np.zeros((2, 79), np.float32)
        model.score_mixture(toks, logp)
        ref, _ = O.score_mixture(O.OracleModel(cfg, w), toks)
        np.testing.assert_allclose(logp, ref, atol=tolerance(cfg), rtol=0)
        model.close()
    prompts = [p[:n] for p, n in zip(W.make_prompts(wl, seed=4, lengths=[70] * batch),
                                     np.random.default_rng(1).integers(1, 70, size=batch))]
    chk, *_ = run_decode_parity(nv, cfg, w, prompts, 8, check_kv=batch == 3)
    assert chk.steps == 8


def test_cta_pair_and_single_cta_gemm_agree(weights):
    """The CTA-pair GEMM (tcgen05.mma cta_group::2, 256 x 256 tiles; launches
    with 1024 rows or more and one K slice) against the one-CTA kernel, on
    scoring rows whose last pair tile is ragged (5 x 257 = 1285 rows) and on a
    ragged prefill: every epilogue (RoPE + KV write, residual, SwiGLU, exit
    log-sum-exp) runs on both."""
    toks = np.stack([W.make_prompts(W.WORKLOADS["S"], seed=s)[0][:257] for s in range(5)]).astype(np.int32)
    lens = np.array([300, 257, 129, 64, 517], np.int32)
    prompts = [p[:n] for p, n in zip(W.make_prompts(W.WORKLOADS["S"], lengths=[600] * 5), lens)]
    out = {}
    for eng in ("single", "pair"):
        if eng == "single":
            os.environ["NVIUM_GEMM_PAIR"] = "0"
        try:
            m = nv.Model(CFG, weights, max_batch=5, max_seq=640)
        finally:
            os.environ.pop("NVIUM_GEMM_PAIR", None)
        lp = np.zeros((5, 256), np.float32)
        m.score_mixture(toks, lp)
        st = nv.State(m, 5)
        st.prefill(np.concatenate(prompts), lens)
        st.sync_status()
        kv = [st.read_kv(b, l, 640) for b in range(5) for l in (0, 11)]
        out[eng] = (lp, kv)
        st.close()
        m.close()
    np.testing.assert_allclose(out["single"][0], out["pair"][0], atol=5e-3, rtol=0)
    for (K1, V1, n1), (K2, V2, n2) in zip(out["single"][1], out["pair"][1]):
        assert n1 == n2
        np.testing.assert_allclose(W.as_f32(K1), W.as_f32(K2), atol=2e-2, rtol=2 ** -7)
        np.testing.assert_allclose(W.as_f32(V1), W.as_f32(V2), atol=2e-2, rtol=2 ** -7)


def test_tcgen05_and_mma_flash_attention_agree(weights):
    """Scoring and prefill attention on the tcgen05 kernel (128-row query
    tiles, scores and P V in TMEM) against the warp-MMA kernel, on sequences
    of ragged lengths spanning several query and key tiles."""
    toks = np.stack([W.make_prompts(W.WORKLOADS["S"], seed=s)[0][:300] for s in (7, 8)]).astype(np.int32)
    out = {}
    for eng in ("mma", "tc"):
        if eng == "mma":
            os.environ["NVIUM_ATTN"] = "mma"
        try:
            m = nv.Model(CFG, weights, max_batch=3, max_seq=320)
        finally:
            os.environ.pop("NVIUM_ATTN", None)
        lp = np.zeros((2, 299), np.float32)
        m.score_mixture(toks, lp)
        # prefill of ragged prompts: every layer's KV depends on the attention outputs
        lens = np.array([300, 129, 64], np.int32)
        st = nv.State(m, 3)
        st.prefill(np.concatenate([toks[0], toks[1][:129], toks[0][:64]]), lens)
        kv = [st.read_kv(b, 11, 320) for b in range(3)]
        out[eng] = (lp, kv)
        st.close()
        m.close()
    np.testing.assert_allclose(out["mma"][0], out["tc"][0], atol=5e-3, rtol=0)
    for (K1, V1, n1), (K2, V2, n2) in zip(out["mma"][1], out["tc"][1]):
        assert n1 == n2
        np.testing.assert_allclose(W.as_f32(K1), W.as_f32(K2), atol=2e-2, rtol=2 ** -7)
        np.testing.assert_allclose(W.as_f32(V1), W.as_f32(V2), atol=2e-2, rtol=2 ** -7)
