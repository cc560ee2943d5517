"""GPU parity on the tiny fp32 model (4 layers, d=64, 2 heads, vocab 256,
exits after layers 1/2/3/4): the CUDA path against the CPU oracle on the same
seeded inputs, through the C ABI.  Tolerance 1e-4 (fp32)."""
import numpy as np
import pytest

import workloads as W
from oracle import nvium_oracle as O
from tests.nvium_testlib import chisq_pvalue, run_decode_parity

pytestmark = pytest.mark.gpu

nv = pytest.importorskip("exact_early_exit_b200")
CFG = W.TINY


@pytest.fixture(scope="module")
def weights():
    return W.make_weights(CFG, seed=0)


def test_philox_matches_oracle():
    rng = np.random.default_rng(0)
    ctr = rng.integers(0, 2**32, size=(4096, 4), dtype=np.uint64).astype(np.uint32)
    ctr[0] = 0
    ctr[1] = 0xFFFFFFFF
    for seed in (0, 1234, 0xFFFFFFFFFFFFFFFF, 0xA409382229F31D0):
        out = nv.philox4x32_10(seed, ctr)
        ref = O.philox4x32_10([ctr[:, i] for i in range(4)], (seed & 0xFFFFFFFF, seed >> 32))
        np.testing.assert_array_equal(out, np.stack([r.astype(np.uint32) for r in ref], 1))


@pytest.mark.parametrize("mode", [O.ROUTER_NORMAL, O.ROUTER_FORCE_LAST])
def test_scoring_matches_oracle(weights, mode):
    wl = W.WORKLOADS["T"]
    toks = np.stack([W.make_prompts(wl, seed=s)[0] for s in (1, 2, 3)]).astype(np.int32)   # [3, 32]
    model = nv.Model(CFG, weights, max_batch=1, max_seq=64, router_mode=mode)
    logp = np.zeros((3, 31), np.float32)
    nll = np.zeros(1, np.float32)
    depth = np.zeros((3, 31), np.float32)
    mean_depth = np.zeros(1, np.float32)
    model.score_mixture_ex(toks, logp, nll, depth, mean_depth)
    ref, ref_nll, ref_depth, ref_mean_depth = O.score_mixture_with_depth(O.OracleModel(CFG, weights, mode), toks)
    np.testing.assert_allclose(logp, ref, atol=1e-4, rtol=0)
    assert abs(nll[0] - ref_nll) <= 1e-4
    # the compute-penalty forward: expected normalised depth per position
    np.testing.assert_allclose(depth, ref_depth, atol=1e-4, rtol=0)
    assert abs(mean_depth[0] - ref_mean_depth) <= 1e-4
    logp2 = np.zeros((3, 31), np.float32)
    model.score_mixture(toks, logp2)
    np.testing.assert_array_equal(logp2, logp)
    if mode == O.ROUTER_FORCE_LAST:
        dense = O.dense_logprobs(O.OracleModel(CFG, weights, mode), toks[0, :-1])
        np.testing.assert_allclose(logp[0], dense[np.arange(31), toks[0, 1:]], atol=1e-4, rtol=0)


def test_decode_parity_prompt32_steps32(weights):
    prompts = W.make_prompts(W.WORKLOADS["T"])
    chk, state, dec, _ = run_decode_parity(nv, CFG, weights, prompts, 32)
    assert chk.steps == 32
    # fp32: no near-ties expected, and the device's router probabilities
    # agree with the oracle's to fp32 rounding
    assert chk.exit_ties == 0 and chk.token_ties == 0
    assert chk.junctions > 0 and chk.max_dw < 1e-5
    c = state.counters()
    assert c[nv.CTR["steps"]] == 32
    assert c[nv.CTR["exit0"]:nv.CTR["exit0"] + 4].sum() == 32


def test_decode_parity_batch_ragged(weights):
    prompts = [W.make_prompts(W.WORKLOADS["T"], seed=s)[0][:n] for s, n in ((1, 5), (2, 1), (3, 17), (4, 64 + 3))]
    chk, *_ = run_decode_parity(nv, CFG, weights, prompts, 20, max_seq=128)
    assert chk.steps == 20


def test_force_last_decode_is_the_dense_model(weights):
    prompts = W.make_prompts(W.WORKLOADS["T"])
    chk, state, dec, _ = run_decode_parity(nv, CFG, weights, prompts, 16, router_mode=O.ROUTER_FORCE_LAST)
    c = state.counters()
    assert c[nv.CTR["exit0"] + 3] == 16 and c[nv.CTR["exit0"]:nv.CTR["exit0"] + 3].sum() == 0


@pytest.mark.parametrize("bias", [30.0, -30.0])
def test_extreme_routing_and_overflowing_deferred_store(bias):
    """All tokens exit at the first junction (bias +30) so rows pile up until
    the deferred store (max_pending = 4) forces early completion; or none
    exit early (bias -30)."""
    w = W.make_weights(CFG, seed=0, router_bias=[bias, bias, bias])
    prompts = [W.make_prompts(W.WORKLOADS["T"], seed=s)[0][:n] for s, n in ((1, 9), (2, 3))]
    chk, state, dec, _ = run_decode_parity(nv, CFG, w, prompts, 24, max_pending=4)
    c = state.counters()
    if bias > 0:
        assert c[nv.CTR["exit0"]] == 48
        assert c[nv.CTR["forced"]] > 0
    else:
        assert c[nv.CTR["exit0"] + 3] == 48


def test_rewind_replays_identically(weights):
    prompts = W.make_prompts(W.WORKLOADS["T"])
    model = nv.Model(CFG, weights, max_batch=1, max_seq=80)
    st = nv.State(model, 1)
    st.prefill(prompts[0], [32])
    outs = []
    for rep in range(2):
        seq = []
        tok = np.zeros(1, np.int32)
        ex = np.zeros(1, np.int32)
        for s in range(12):
            st.decode_step(77 + s, tok, ex)
            seq.append((int(tok[0]), int(ex[0])))
        outs.append(seq)
        st.rewind()
    assert outs[0] == outs[1]


def test_sampler_chi_square():
    """Exact sampling on the GPU: 4096 copies of one context, 50 seeds, joint
    (exit, token) frequencies against p_k * pi_k(v) from the oracle."""
    w = W.make_weights(CFG, seed=0, router_bias=[-0.3, 0.2, 0.0])
    prompt = W.make_prompts(W.WORKLOADS["T"])[0][:8]
    B = 4096
    model = nv.Model(CFG, w, max_batch=B, max_seq=16, max_pending=4)
    st = nv.State(model, B)
    st.prefill(np.tile(prompt, B).astype(np.int32), np.full(B, 8, np.int32))
    counts = np.zeros((4, CFG.vocab))
    tok = np.zeros(B, np.int32)
    ex = np.zeros(B, np.int32)
    for s in range(50):
        st.decode_step(1000 + s, tok, ex)
        np.add.at(counts, (ex - 1, tok), 1)
        st.rewind()
    om = O.OracleModel(CFG, w)
    _, states, _ = om.forward_sequence(prompt)
    p, pi = O.step_distribution(om, [states[k][7:8] for k in range(4)])
    n = counts.sum()
    assert chisq_pvalue(counts, p[:, None] * pi * n) > 0.01
    assert chisq_pvalue(counts.sum(1), p * n) > 0.01
    assert chisq_pvalue(counts.sum(0), (p[:, None] * pi).sum(0) * n) > 0.01


def test_decode_parity_contexts_spanning_many_chunks(weights):
    """Contexts of 130..400 positions: several 128-key attention chunks,
    a ragged last chunk and a chunk that ends exactly on a page."""
    rng = np.random.default_rng(9)
    prompts = [rng.integers(0, CFG.vocab, size=n).astype(np.int32) for n in (129, 256, 383)]
    chk, *_ = run_decode_parity(nv, CFG, weights, prompts, 12, max_seq=420)
    assert chk.steps == 12


@pytest.mark.parametrize("cfg_name", ["tiny", "mini-bf16"])
def test_conditional_and_flat_step_graphs_agree(cfg_name):
    """The decode-step graph skips the layer blocks no token reaches
    (conditional nodes); the flat graph launches every layer.  Outputs and
    caches are bit-identical."""
    import os
    if cfg_name == "tiny":
        cfg, w = CFG, W.make_weights(CFG, seed=0)
    else:
        cfg = W.ModelConfig("mini-bf16", 4, 256, 4, 64, 512, 1024, (1, 2, 3, 4), W.BF16)
        w = W.make_weights(cfg, seed=3, router_bias=[0.5, 0.0, -0.5])
    rng = np.random.default_rng(3)
    prompts = [rng.integers(0, cfg.vocab, size=n).astype(np.int32) for n in (12, 30, 7)]
    lens = np.array([len(p) for p in prompts], np.int32)
    outs = {}
    for mode in ("1", "0"):
        os.environ["NVIUM_COND_GRAPH"] = mode
        try:
            m = nv.Model(cfg, w, max_batch=3, max_seq=64, max_pending=8)
            st = nv.State(m, 3)
            st.prefill(np.concatenate(prompts), lens)
            tok, ex, lp = np.zeros(3, np.int32), np.zeros(3, np.int32), np.zeros(3, np.float32)
            seq = []
            for s in range(16):
                st.decode_step(77 + s, tok, ex, lp)
                seq.append(np.concatenate([tok, ex, lp.view(np.int32)]))
            st.flush()
            kv = [st.read_kv(b, cfg.n_layers - 1, 64) for b in range(3)]
            outs[mode] = (np.stack(seq), kv, st.counters())
            st.close()
            m.close()
        finally:
            os.environ.pop("NVIUM_COND_GRAPH", None)
    np.testing.assert_array_equal(outs["1"][0], outs["0"][0])
    for a, b in zip(outs["1"][1], outs["0"][1]):
        np.testing.assert_array_equal(a[0], b[0])
        np.testing.assert_array_equal(a[1], b[1])
    # the conditional graph launches no more kernels than the flat one
    assert outs["1"][2][nv.CTR["launches"]] <= outs["0"][2][nv.CTR["launches"]]


def test_decode_parity_batch_wider_than_one_planner_block(weights):
    """300 sequences: the planner's 256 threads each take two sequences; the
    attention and junction grids span several waves."""
    rng = np.random.default_rng(5)
    lens = rng.integers(1, 13, size=300)
    prompts = [W.make_prompts(W.WORKLOADS["T"], seed=10 + i)[0][:n] for i, n in enumerate(lens)]
    chk, state, dec, _ = run_decode_parity(nv, CFG, weights, prompts, 4, max_seq=32)
    assert chk.steps == 4 and chk.exit_ties == 0 and chk.token_ties == 0


def test_host_argument_and_capacity_errors(weights):
    """Argument and state errors come back as statuses, and a sequence that
    reaches max_seq stops with NV_ERR_CAPACITY; the state stays usable."""
    prompt = W.make_prompts(W.WORKLOADS["T"])[0][:10]
    model = nv.Model(CFG, weights, max_batch=2, max_seq=16)
    st = nv.State(model, 1)
    tok, ex = np.zeros(1, np.int32), np.zeros(1, np.int32)
    with pytest.raises(nv.NviumError) as e:
        st.decode_step(1, tok, ex)
    assert e.value.status == nv.NV_ERR_STATE
    with pytest.raises(nv.NviumError) as e:
        st.prefill(prompt, [0])
    assert e.value.status == nv.NV_ERR_INVALID_ARG
    bad = prompt.copy()
    bad[3] = CFG.vocab
    with pytest.raises(nv.NviumError) as e:
        st.prefill(bad, [10])
    assert e.value.status == nv.NV_ERR_INVALID_ARG
    st.prefill(prompt, [10])
    n = 0
    with pytest.raises(nv.NviumError) as e:
        for s in range(16):
            st.decode_step(5 + s, tok, ex)
            n += 1
    assert e.value.status == nv.NV_ERR_CAPACITY
    # steps at positions 9 .. 14 sample tokens for 10 .. 15; the next would
    # sample position 16 = max_seq
    assert n == 16 - 10
    st.sync_status()
    st.rewind()
    st.decode_step(5, tok, ex)
    st.sync_status()
    st.close()
    model.close()


def test_bounded_wait_gives_up_and_leaves_the_context_usable():
    """Failure detection without a GPU fault: a wait that nothing completes
    gives up after its limit and reports it; the next launches still work."""
    assert nv.selftest_bounded_wait(20000)
    ctr = np.arange(64, dtype=np.uint32).reshape(16, 4)
    out = nv.philox4x32_10(7, ctr)
    ref = O.philox4x32_10([ctr[:, i] for i in range(4)], (7, 0))
    np.testing.assert_array_equal(out, np.stack([r.astype(np.uint32) for r in ref], 1))


def test_router_mlp_scoring_and_decode_match_oracle():
    """Router MLP (width 8) instead of the scalar router: mixture scoring and
    teacher-forced decode against the oracle, fp32 tolerance."""
    import dataclasses
    cfg = dataclasses.replace(CFG, router_hidden=8)
    w = W.make_weights(cfg, seed=0)
    toks = np.stack([W.make_prompts(W.WORKLOADS["T"], seed=s)[0] for s in (1, 2)]).astype(np.int32)
    model = nv.Model(cfg, w, max_batch=1, max_seq=64)
    logp = np.zeros((2, 31), np.float32)
    depth = np.zeros((2, 31), np.float32)
    model.score_mixture_ex(toks, logp, None, depth)
    ref, _, ref_depth, _ = O.score_mixture_with_depth(O.OracleModel(cfg, w), toks)
    np.testing.assert_allclose(logp, ref, atol=1e-4, rtol=0)
    np.testing.assert_allclose(depth, ref_depth, atol=1e-4, rtol=0)
    model.close()
    prompts = [W.make_prompts(W.WORKLOADS["T"], seed=s)[0][:n] for s, n in ((1, 7), (2, 20), (3, 1))]
    chk, state, dec, _ = run_decode_parity(nv, cfg, w, prompts, 16)
    assert chk.steps == 16 and chk.exit_ties == 0 and chk.token_ties == 0
    c = state.counters()
    assert c[nv.CTR["exit0"]:nv.CTR["exit0"] + 4].sum() == 48


def test_shared_head_with_adapters_matches_oracle():
    """Exits share the last exit's head behind adapters of width 32: scoring
    and teacher-forced decode against the oracle (fp32)."""
    import dataclasses
    cfg = dataclasses.replace(CFG, adapter_hidden=32)
    w = W.make_weights(cfg, seed=0)
    for k in range(cfg.n_exits - 1):
        del w["exits"][k]["head"]  # only the last exit's head is read
    toks = np.stack([W.make_prompts(W.WORKLOADS["T"], seed=s)[0] for s in (1, 2)]).astype(np.int32)
    model = nv.Model(cfg, w, max_batch=1, max_seq=64)
    logp = np.zeros((2, 31), np.float32)
    model.score_mixture(toks, logp)
    ref, _ = O.score_mixture(O.OracleModel(cfg, w), toks)
    np.testing.assert_allclose(logp, ref, atol=1e-4, rtol=0)
    model.close()
    prompts = [W.make_prompts(W.WORKLOADS["T"], seed=s)[0][:n] for s, n in ((1, 9), (2, 1), (3, 30))]
    chk, *_ = run_decode_parity(nv, cfg, w, prompts, 16)
    assert chk.steps == 16 and chk.exit_ties == 0 and chk.token_ties == 0
