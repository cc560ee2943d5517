"""Pins for the CPU oracle, each against something other than the oracle itself.

* Philox4x32-10 against the published known-answer vectors (tests/golden).
* bf16 rounding against torch's float32 -> bfloat16 conversion.
* Stick-breaking exit probabilities (gist.science summary, section 2, equation
  for p_k with w_{N_V} = 1) against the closed form sum_k p_k = 1.
* The mixture (section 2, equation for pi_mix) sums to one over the vocabulary.
* The backbone against an independent LLaMA implementation
  (transformers.LlamaForCausalLM, float64): the dense model is the special case
  of zero intermediate routing mass (section 5), and every intermediate exit is
  checked through the same model's hidden states.
* The piggybacked decode (section 2, "Inferenz: Piggybacking") against an
  undeferred full-depth forward: KV caches equal after the flush.
* Exact sampling: chi-square of (exit, token) draws against p_k * pi_k(v).
"""
import os

import numpy as np
import pytest
import torch

import workloads as W
from oracle import nvium_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def tiny_model(mode=O.ROUTER_NORMAL, random_gains=True, seed=0):
    w = W.make_weights(W.TINY, seed=seed, random_gains=random_gains)
    return O.OracleModel(W.TINY, w, mode), w


# --------------------------------------------------------------------------
def test_philox_known_answers():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) if not l.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        v = [int(x, 16) for x in r]
        out = O.philox4x32_10(v[:4], v[4:6])
        assert [int(o) for o in out] == v[6:]


def test_philox_vectorised_matches_scalar():
    rng = np.random.default_rng(5)
    ctr = rng.integers(0, 2**32, size=(4, 64), dtype=np.uint64)
    key = rng.integers(0, 2**32, size=(2, 64), dtype=np.uint64)
    vec = O.philox4x32_10(list(ctr), list(key))
    for i in range(0, 64, 13):
        one = O.philox4x32_10([int(c[i]) for c in ctr], [int(k[i]) for k in key])
        assert [int(x[i]) for x in vec] == [int(x) for x in one]


def test_uniform_is_exact_in_fp32_and_open_interval():
    x = np.array([0, 1, 511, 512, 2**31, 2**32 - 1, 0xDEADBEEF], dtype=np.uint64)
    u = O.uniform01(x)
    assert np.all(u > 0) and np.all(u < 1)
    assert np.array_equal(u.astype(np.float32).astype(np.float64), u)
    assert u[0] == 2.0 ** -24 and u[-2] == 1 - 2.0 ** -24


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(100000) * 3,
                        rng.standard_normal(1000) * 1e-3,
                        # exact ties between two bf16 neighbours
                        (np.arange(1, 200) * 2 + 1) * 2.0 ** -8 + 1.0]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.bf16_round(x.astype(np.float64)), ref)


# --------------------------------------------------------------------------
def test_stick_breaking_sums_to_one():
    rng = np.random.default_rng(2)
    for n in (1, 2, 3, 7):
        w = rng.random((1000, n))
        p = O.exit_probs(w)
        assert np.all(p >= 0)
        np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-12)
        # log-space form agrees with the direct product
        z = np.log(w) - np.log1p(-w)
        np.testing.assert_allclose(np.exp(O.log_exit_probs(z)), p, rtol=1e-10, atol=1e-14)
    # p_1 = w_1 and p_k for a hand example
    p = O.exit_probs(np.array([0.5, 0.5, 0.5]))
    np.testing.assert_allclose(p, [0.5, 0.25, 0.125, 0.125])


def test_force_last_log_exit_probs():
    lp = O.log_exit_probs(np.array([[3.0, -2.0, 0.1]]), O.ROUTER_FORCE_LAST)
    assert np.all(np.isneginf(lp[0, :3])) and lp[0, 3] == 0.0


def test_mixture_logprob_logspace_vs_direct():
    rng = np.random.default_rng(3)
    z = rng.standard_normal((50, 3)) * 2
    logpi = np.log(rng.dirichlet(np.ones(6), size=(50, 4)))[..., 0]
    direct = np.log(np.sum(O.exit_probs(1 / (1 + np.exp(-z))) * np.exp(logpi), axis=-1))
    np.testing.assert_allclose(O.mixture_logprob(O.log_exit_probs(z), logpi), direct, rtol=1e-12)


def test_mixture_sums_to_one_on_tiny_vocab():
    model, _ = tiny_model()
    prompt = W.make_prompts(W.WORKLOADS["T"])[0][:12]
    _, states, _ = model.forward_sequence(prompt)
    for pos in (0, 5, 11):
        p, pi = O.step_distribution(model, [states[k][pos:pos + 1] for k in range(4)])
        np.testing.assert_allclose(p.sum(), 1.0, atol=1e-12)
        mix = (p[:, None] * pi).sum(0)
        np.testing.assert_allclose(mix.sum(), 1.0, atol=1e-12)
        assert 0.0 < p[0] < 1.0


def test_rope_relative_position_and_identity():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 2, 32))
    k = rng.standard_normal((1, 2, 32))
    np.testing.assert_allclose(O.rope(q, np.array([0]), 1e4), q)
    d1 = np.einsum("nhd,nhd->nh", O.rope(q, np.array([17]), 1e4), O.rope(k, np.array([5]), 1e4))
    d2 = np.einsum("nhd,nhd->nh", O.rope(q, np.array([112]), 1e4), O.rope(k, np.array([100]), 1e4))
    np.testing.assert_allclose(d1, d2, rtol=1e-10)


@pytest.mark.parametrize("rows_per_block", [256, 7])
def test_causal_attention_against_torch_sdpa(rows_per_block):
    """The oracle's attention (per row, and as masked blocks of rows) against
    torch's scaled_dot_product_attention with a causal mask in float64: rows
    at positions 300..599 of one sequence attend to keys 0..their position."""
    rng = np.random.default_rng(9)
    H, hd, P = 3, 32, 600
    q = rng.standard_normal((P, H, hd))
    K = rng.standard_normal((P, H, hd))
    V = rng.standard_normal((P, H, hd))
    scale = 1.0 / np.sqrt(hd)
    tq = torch.from_numpy(q.transpose(1, 0, 2))[None]
    tk = torch.from_numpy(K.transpose(1, 0, 2))[None]
    tv = torch.from_numpy(V.transpose(1, 0, 2))[None]
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)[0].numpy().transpose(1, 0, 2)
    pos = np.arange(300, P)
    blk = O.causal_attention_rows(q[pos], K, V, pos, scale, rows_per_block=rows_per_block)
    np.testing.assert_allclose(blk, ref[pos], rtol=0, atol=1e-12)
    for p in (300, 301, 450, 599):
        np.testing.assert_allclose(O.attention_row(q[p], K, V, p, scale), ref[p], rtol=0, atol=1e-12)
    # a ragged subset of positions (the deferred rows of a decode step)
    sub = np.array([3, 4, 5, 77, 78, 599])
    np.testing.assert_allclose(O.causal_attention_rows(q[sub], K, V, sub, scale, rows_per_block), ref[sub],
                               rtol=0, atol=1e-12)


def test_block_and_row_attention_give_the_same_forward():
    """A full-depth forward with block attention equals the row-at-a-time one."""
    om, _ = tiny_model()
    toks = W.make_prompts(W.WORKLOADS["T"])[0]
    h1, s1, c1 = om.forward_sequence(toks)
    om.block_attention = False
    h2, s2, c2 = om.forward_sequence(toks)
    np.testing.assert_allclose(h1, h2, rtol=0, atol=1e-12)
    for m in range(W.TINY.n_layers):
        np.testing.assert_allclose(c1.K[m], c2.K[m], rtol=0, atol=1e-12)
        np.testing.assert_allclose(c1.V[m], c2.V[m], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# independent LLaMA (transformers, float64)
# --------------------------------------------------------------------------

def _hf_llama(cfg, w):
    from transformers import LlamaConfig, LlamaForCausalLM
    hc = LlamaConfig(vocab_size=cfg.vocab, hidden_size=cfg.d_model, intermediate_size=cfg.d_ff,
                     num_hidden_layers=cfg.n_layers, num_attention_heads=cfg.n_heads,
                     num_key_value_heads=cfg.n_heads, head_dim=cfg.head_dim,
                     rms_norm_eps=cfg.rms_eps, rope_theta=cfg.rope_theta,
                     max_position_embeddings=4096, tie_word_embeddings=False,
                     attention_bias=False, mlp_bias=False, hidden_act="silu")
    hc._attn_implementation = "eager"
    torch.manual_seed(0)
    m = LlamaForCausalLM(hc).to(torch.float64).eval()
    t = lambda a: torch.from_numpy(W.as_f32(a).astype(np.float64))
    with torch.no_grad():
        m.model.embed_tokens.weight.copy_(t(w["tok_emb"]))
        for i, L in enumerate(w["layers"]):
            ly = m.model.layers[i]
            ly.input_layernorm.weight.copy_(t(L["attn_norm"]))
            ly.self_attn.q_proj.weight.copy_(t(L["wq"]))
            ly.self_attn.k_proj.weight.copy_(t(L["wk"]))
            ly.self_attn.v_proj.weight.copy_(t(L["wv"]))
            ly.self_attn.o_proj.weight.copy_(t(L["wo"]))
            ly.post_attention_layernorm.weight.copy_(t(L["mlp_norm"]))
            ly.mlp.gate_proj.weight.copy_(t(L["wg"]))
            ly.mlp.up_proj.weight.copy_(t(L["wu"]))
            ly.mlp.down_proj.weight.copy_(t(L["wd"]))
        m.model.norm.weight.copy_(t(w["exits"][-1]["norm"]))
        m.lm_head.weight.copy_(t(w["exits"][-1]["head"]))
    return m


HF_TOL = 2e-6


@pytest.fixture(scope="module")
def hf_tiny():
    model, w = tiny_model(random_gains=True)
    return model, w, _hf_llama(W.TINY, w)


def test_dense_equals_hf_llama(hf_tiny):
    model, w, hf = hf_tiny
    toks = W.make_prompts(W.WORKLOADS["T"])[0]
    ours = O.dense_logprobs(model, toks)
    with torch.no_grad():
        ref = torch.log_softmax(hf(torch.from_numpy(toks.astype(np.int64))[None]).logits[0], -1).numpy()
    # transformers computes RMSNorm and the RoPE tables in float32 internally,
    # so agreement is at the 1e-7 level; a wrong sign, index or term is >1e-3.
    np.testing.assert_allclose(ours, ref, atol=HF_TOL, rtol=0)


def test_mixture_scoring_against_hf_hidden_states(hf_tiny):
    """Every exit's head, the routers and the mixture, recomputed from the
    independent model's per-layer hidden states with torch routines."""
    model, w, hf = hf_tiny
    cfg = W.TINY
    toks = W.make_prompts(W.WORKLOADS["T"])[0][None, :24]
    logp, nll = O.score_mixture(model, toks)
    with torch.no_grad():
        out = hf(torch.from_numpy(toks[:, :-1].astype(np.int64)), output_hidden_states=True)
    tgt = torch.from_numpy(toks[0, 1:].astype(np.int64))
    t = lambda a: torch.from_numpy(W.as_f32(a).astype(np.float64))
    probs = torch.zeros(toks.shape[1] - 1, dtype=torch.float64)
    surv = torch.ones(toks.shape[1] - 1, dtype=torch.float64)
    for k, layer in enumerate(cfg.exit_layers):
        hs = out.hidden_states[layer][0]          # residual after `layer` layers
        if layer == cfg.n_layers:
            # the last exit is the model's own final norm + LM head
            pik = torch.softmax(out.logits[0], -1)
        else:
            nk = torch.nn.functional.rms_norm(hs, (cfg.d_model,), t(w["exits"][k]["norm"]), cfg.rms_eps)
            pik = torch.softmax(nk @ t(w["exits"][k]["head"]).T, -1)
        if k < cfg.n_exits - 1:
            wk = torch.sigmoid(nk @ t(w["exits"][k]["router_w"]) + w["exits"][k]["router_b"])
            pk = wk * surv
            surv = surv * (1 - wk)
        else:
            pk = surv
        probs += pk * pik[torch.arange(len(tgt)), tgt]
    np.testing.assert_allclose(logp[0], torch.log(probs).numpy(), atol=HF_TOL, rtol=0)
    assert abs(nll + float(torch.log(probs).mean())) < HF_TOL


def test_force_last_scoring_equals_dense():
    model, _ = tiny_model(O.ROUTER_FORCE_LAST)
    toks = W.make_prompts(W.WORKLOADS["T"])[0][None, :20]
    logp, _ = O.score_mixture(model, toks)
    dense = O.dense_logprobs(model, toks[0, :-1])
    np.testing.assert_array_equal(logp[0], dense[np.arange(19), toks[0, 1:]])


def test_bf16_model_matches_hf_in_fp64_when_rounding_off():
    """The bf16 code path minus its rounding points is the plain LLaMA; with
    the rounding points the change is at the bf16 scale, not more."""
    cfg = W.ModelConfig("mini-bf16", 2, 64, 4, 16, 128, 512, (1, 2), W.BF16)
    w = W.make_weights(cfg, seed=3, random_gains=True)
    model = O.OracleModel(cfg, w, O.ROUTER_FORCE_LAST)
    toks = W.zipf_ids(16, cfg.vocab, np.random.default_rng(0))
    hf = _hf_llama(cfg, w)
    with torch.no_grad():
        ref = torch.log_softmax(hf(torch.from_numpy(toks.astype(np.int64))[None]).logits[0], -1).numpy()
    model.bf16 = False
    np.testing.assert_allclose(O.dense_logprobs(model, toks), ref, atol=HF_TOL, rtol=0)
    model.bf16 = True
    d = np.abs(O.dense_logprobs(model, toks) - ref).max()
    assert 1e-6 < d < 5e-2


# --------------------------------------------------------------------------
# piggybacked decode == undeferred full depth
# --------------------------------------------------------------------------

def _check_invariants(dec, b):
    cfg = dec.model.cfg
    lens = dec.caches[b].lens
    t = dec.t[b]
    # len non-increasing in m, every layer up to the first exit complete
    assert all(lens[i] >= lens[i + 1] for i in range(cfg.n_layers - 1))
    assert all(lens[i] == t for i in range(cfg.exit_layers[0]))
    # pending set = suffix [len_L, t)
    assert sorted(dec.pending[b]) == list(range(lens[-1], t))


@pytest.mark.parametrize("pattern", ["all1", "alternate", "random", "routed", "last"])
def test_deferred_kv_equals_full_depth(pattern):
    cfg = W.TINY
    model, _ = tiny_model()
    prompts = [W.make_prompts(W.WORKLOADS["T"])[0][:9], W.make_prompts(W.WORKLOADS["T"], seed=7)[0][:14]]
    steps = 20
    dec = O.OracleDecoder(model, prompts, steps)
    rng = np.random.default_rng(11)
    for s in range(steps):
        if pattern == "all1":
            ex = [1, 1]
        elif pattern == "alternate":
            ex = [1 + (s % 2) * 3, 4 - (s % 2) * 2]
        elif pattern == "random":
            ex = list(rng.integers(1, 5, size=2))
        elif pattern == "last":
            ex = [4, 4]
        else:
            ex = None
        dec.step(1234, forced_exits=ex)
        for b in range(2):
            _check_invariants(dec, b)
    dec.flush()
    for b in range(2):
        t = dec.t[b]
        assert dec.caches[b].lens == [t] * cfg.n_layers
        _, _, full = model.forward_sequence(dec.tokens[b][:t])
        for m in range(cfg.n_layers):
            np.testing.assert_allclose(dec.caches[b].K[m][:t], full.K[m][:t], rtol=1e-10, atol=1e-13)
            np.testing.assert_allclose(dec.caches[b].V[m][:t], full.V[m][:t], rtol=1e-10, atol=1e-13)


@pytest.mark.parametrize("pattern", ["routed", "all1"])
def test_early_completion_changes_nothing(pattern):
    """Reading r7: completing a sequence's deferred rows before the lazy rule
    would run them (what the GPU does when a sequence's deferred store is
    full) changes no value.  A decoder that flushes part-way takes the same
    exits and tokens with the same log-probabilities and junction draws as
    the lazy one, and both end with the same caches."""
    cfg = W.TINY
    model, _ = tiny_model()
    prompts = [W.make_prompts(W.WORKLOADS["T"])[0][:9], W.make_prompts(W.WORKLOADS["T"], seed=7)[0][:14]]
    steps = 16
    lazy = O.OracleDecoder(model, prompts, steps)
    eager = O.OracleDecoder(model, prompts, steps)
    completed = 0
    for s in range(steps):
        ex = [1, 1] if pattern == "all1" else None
        if s in (4, 9):
            completed += sum(eager.deferred_rows(b) for b in range(2))
            eager.flush()
        ra = lazy.step(1234, forced_exits=ex)
        rb = eager.step(1234, forced_exits=ex)
        for a, b in zip(ra, rb):
            assert (a.exit, a.token) == (b.exit, b.token)
            np.testing.assert_allclose(b.logp, a.logp, rtol=1e-10, atol=1e-12)
            assert len(a.junctions) == len(b.junctions)
            for (ka, ua, wa), (kb, ub, wb) in zip(a.junctions, b.junctions):
                assert (ka, ua) == (kb, ub)
                np.testing.assert_allclose(wb, wa, rtol=1e-10)
    assert completed > 0, "nothing was deferred when the early completion ran"
    lazy.flush()
    eager.flush()
    for b in range(2):
        t = lazy.t[b]
        assert eager.t[b] == t and lazy.caches[b].lens == eager.caches[b].lens == [t] * cfg.n_layers
        # both against an undeferred full-depth forward of the same tokens
        _, _, full = model.forward_sequence(lazy.tokens[b][:t])
        for m in range(cfg.n_layers):
            for dec in (lazy, eager):
                np.testing.assert_allclose(dec.caches[b].K[m][:t], full.K[m][:t], rtol=1e-10, atol=1e-13)
                np.testing.assert_allclose(dec.caches[b].V[m][:t], full.V[m][:t], rtol=1e-10, atol=1e-13)


def test_decode_step_law_matches_full_depth_states():
    """The h a new token reaches each junction with, under deferral, is the
    full-depth forward's h: the step's (u, w) and scores use it."""
    model, _ = tiny_model()
    p = W.make_prompts(W.WORKLOADS["T"])[0][:10]
    dec = O.OracleDecoder(model, [p], 8)
    for s in range(6):
        dec.step(99, forced_exits=[1 + (s % 3)])
    t = dec.t[0]
    rec = dec.step_seq(0, 4321, forced_exit=4)
    _, states, _ = model.forward_sequence(dec.tokens[0][: t + 1])
    for (k, u, w) in rec.junctions:
        np.testing.assert_allclose(w, model.router_prob(k - 1, states[k - 1][t]).item(), rtol=1e-10)
        assert u == float(O.exit_uniform(4321, 0, t, k))
    lg = model.head_logits(3, states[3][t:t + 1])[0]
    np.testing.assert_allclose(rec.scores, lg + O.gumbel_noise(4321, 0, t, W.TINY.vocab), rtol=1e-10)


# --------------------------------------------------------------------------
# exact sampling
# --------------------------------------------------------------------------

def _chisq_merged(counts, expected):
    from tests.nvium_testlib import chisq_pvalue
    return chisq_pvalue(counts, expected)


def test_sequential_stop_frequencies_match_pk():
    w = np.array([0.3, 0.5, 0.2])
    seeds = np.arange(200000, dtype=np.uint64)
    u = np.stack([O.exit_uniform(seeds, 0, 7, k) for k in (1, 2, 3)], -1)
    ex = O.sample_exit(u, w)
    counts = np.bincount(ex, minlength=5)[1:]
    assert _chisq_merged(counts, O.exit_probs(w) * len(seeds)) > 0.01


def test_exact_sampler_joint_frequencies():
    """(exit, token) from sequential stopping + Gumbel-max, 2e5 seeds, against
    p_k * pi_k(v); the token marginal against pi_mix."""
    model, _ = tiny_model()
    cfg = W.TINY
    prompt = W.make_prompts(W.WORKLOADS["T"])[0][:16]
    _, states, _ = model.forward_sequence(prompt)
    t = len(prompt) - 1
    js = [states[k][t:t + 1] for k in range(4)]
    p, pi = O.step_distribution(model, js)
    w = np.array([model.router_prob(k, js[k]).item() for k in range(3)])
    logits = np.stack([model.head_logits(k, js[k])[0] for k in range(4)])
    N, chunk = 200000, 25000
    joint = np.zeros((4, cfg.vocab))
    for c0 in range(0, N, chunk):
        seeds = np.arange(c0, c0 + chunk, dtype=np.uint64) + np.uint64(10**6)
        u = np.stack([O.exit_uniform(seeds, 0, t, k) for k in (1, 2, 3)], -1)
        ex = O.sample_exit(u, w) - 1
        tok = O.gumbel_argmax(logits[ex], O.gumbel_noise(seeds, 0, t, cfg.vocab))
        np.add.at(joint, (ex, tok), 1)
    assert _chisq_merged(joint, p[:, None] * pi * N) > 0.01
    assert _chisq_merged(joint.sum(0), (p[:, None] * pi).sum(0) * N) > 0.01
    assert _chisq_merged(joint.sum(1), p * N) > 0.01


def test_decoder_step_uses_the_vectorised_sampler():
    model, _ = tiny_model()
    prompt = W.make_prompts(W.WORKLOADS["T"])[0][:16]
    _, states, _ = model.forward_sequence(prompt)
    t = len(prompt) - 1
    js = [states[k][t:t + 1] for k in range(4)]
    w = np.array([model.router_prob(k, js[k]).item() for k in range(3)])
    logits = np.stack([model.head_logits(k, js[k])[0] for k in range(4)])
    for seed in (1, 2, 3, 1234, 2**40 + 5):
        dec = O.OracleDecoder(model, [prompt], 1)
        rec = dec.step(seed)[0]
        u = np.array([float(O.exit_uniform(seed, 0, t, k)) for k in (1, 2, 3)])
        ex = int(O.sample_exit(u, w))
        tok = int(O.gumbel_argmax(logits[ex - 1], O.gumbel_noise(seed, 0, t, W.TINY.vocab)))
        assert (rec.exit, rec.token) == (ex, tok)


def test_gumbel_argmax_ties_to_lowest_id():
    assert int(O.gumbel_argmax(np.array([1.0, 3.0, 3.0, 2.0]), np.zeros(4))) == 1


# ---------------------------------------------------------------------------
# compute-penalty forward: expected normalised layer depth
# ---------------------------------------------------------------------------
def test_expected_depth_closed_forms():
    """Zero intermediate mass: every token runs all L layers (depth 1). A
    router that always stops at the first node: depth l_1 / L."""
    z = np.random.default_rng(3).normal(size=(50, 3))
    exits, L = (3, 6, 9, 12), 12
    d_last = O.expected_depth(O.log_exit_probs(z, O.ROUTER_FORCE_LAST), exits, L)
    np.testing.assert_array_equal(d_last, np.ones(50))
    d_first = O.expected_depth(O.log_exit_probs(np.full((4, 3), 60.0)), exits, L)
    np.testing.assert_allclose(d_first, 3 / 12, rtol=0, atol=1e-12)
    d_never = O.expected_depth(O.log_exit_probs(np.full((4, 3), -60.0)), exits, L)
    np.testing.assert_allclose(d_never, 1.0, rtol=0, atol=1e-12)


def test_expected_depth_matches_sampled_exits():
    """E[depth] equals the mean depth of exits drawn by the sequential
    stop/continue sampler (itself pinned to p_k above): 2e5 draws, 5 sigma."""
    w = np.array([0.35, 0.4, 0.55])
    z = np.log(w / (1 - w))
    exits, L = (2, 5, 7, 11), 11
    want = float(O.expected_depth(O.log_exit_probs(z[None, :]), exits, L)[0])
    seeds = np.arange(200000, dtype=np.uint64)
    u = np.stack([O.exit_uniform(seeds, 0, 3, k) for k in (1, 2, 3)], -1)
    depth = np.asarray(exits, dtype=np.float64)[O.sample_exit(u, w) - 1] / L
    assert abs(depth.mean() - want) < 5 * depth.std() / np.sqrt(len(depth))


def test_scoring_depth_uses_the_scoring_exit_probabilities():
    """score_mixture_with_depth returns score_mixture's values plus the depth
    of the same log p_k (its definition on the tiny model)."""
    model, _ = tiny_model()
    toks = np.stack([W.make_prompts(W.WORKLOADS["T"], seed=s)[0][:12] for s in (1, 2)])
    lp, nll = O.score_mixture(model, toks)
    lp2, nll2, depth, mean_depth = O.score_mixture_with_depth(model, toks)
    np.testing.assert_array_equal(lp, lp2)
    assert nll == nll2
    assert depth.shape == lp.shape and abs(mean_depth - depth.mean()) < 1e-15
    assert np.all(depth >= model.cfg.exit_layers[0] / model.cfg.n_layers - 1e-12) and np.all(depth <= 1 + 1e-12)


# ---------------------------------------------------------------------------
# router MLP (section 2 "Architektur": a router MLP maps h at node k to w_k)
# ---------------------------------------------------------------------------
def _mlp_router_model(U_of, c_of, v_of, mode=O.ROUTER_NORMAL):
    import dataclasses
    model, w = tiny_model(mode)
    r = U_of(w["exits"][0]).shape[0]
    cfg = dataclasses.replace(W.TINY, router_hidden=r)
    w2 = {**w, "exits": [dict(e) for e in w["exits"]]}
    for k in range(cfg.n_exits - 1):
        e = w2["exits"][k]
        e["router_w1"], e["router_b1"], e["router_w2"] = U_of(e), c_of(e), v_of(e)
    return O.OracleModel(cfg, w2, mode), model


def test_router_mlp_reduces_to_the_scalar_router():
    """silu(x) - silu(-x) = x, so hidden units U = [r; -r], c = 0, v = [1, -1]
    give z = r . n + b: mixture scoring equals the (pinned) scalar router's."""
    mlp, scalar = _mlp_router_model(lambda e: np.stack([e["router_w"], -e["router_w"]]),
                                    lambda e: np.zeros(2, np.float32), lambda e: np.array([1.0, -1.0], np.float32))
    toks = np.stack([W.make_prompts(W.WORKLOADS["T"], seed=s)[0][:16] for s in (1, 2)])
    a, _ = O.score_mixture(mlp, toks)
    b, _ = O.score_mixture(scalar, toks)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_router_mlp_hidden_unit_is_torch_silu():
    """One hidden unit: z = silu(r . n + c) + b, against torch's SiLU; a second
    unit with output weight 0 changes nothing."""
    import torch
    c0 = np.float32(0.37)
    mlp, scalar = _mlp_router_model(lambda e: e["router_w"][None, :], lambda e: np.array([c0], np.float32),
                                    lambda e: np.array([1.0], np.float32))
    rng = np.random.default_rng(2)
    n = rng.normal(size=(32, W.TINY.d_model))
    for k in range(W.TINY.n_exits - 1):
        pre = n @ O.widen(scalar.exits[k]["router_w"]) + float(c0)
        want = torch.nn.functional.silu(torch.from_numpy(pre)).numpy() + scalar.exits[k]["router_b"]
        np.testing.assert_allclose(mlp.router_logit(k, n), want, rtol=0, atol=1e-13)
    wide, _ = _mlp_router_model(lambda e: np.stack([e["router_w"], e["router_w"] * 3]),
                                lambda e: np.array([c0, 1.0], np.float32), lambda e: np.array([1.0, 0.0], np.float32))
    for k in range(W.TINY.n_exits - 1):
        np.testing.assert_allclose(wide.router_logit(k, n), mlp.router_logit(k, n), rtol=0, atol=1e-13)


# ---------------------------------------------------------------------------
# shared head + exit adapters (section 2 "Architektur": all exits share the
# final LM head; light adapter MLPs map intermediate states to its geometry)
# ---------------------------------------------------------------------------
def _adapter_model(W1_of, W2_of, same_norms=False, mode=O.ROUTER_NORMAL):
    import dataclasses
    _, w = tiny_model(mode)
    a = W1_of(w["exits"][0]).shape[0]
    cfg = dataclasses.replace(W.TINY, adapter_hidden=a)
    w2 = {**w, "exits": [dict(e) for e in w["exits"]]}
    last = w2["exits"][-1]
    for k in range(cfg.n_exits - 1):
        e = w2["exits"][k]
        e["adapter_w1"], e["adapter_w2"] = W1_of(e), W2_of(e)
        if same_norms:
            e["norm"] = last["norm"]
    return O.OracleModel(cfg, w2, mode), w2


def test_adapters_with_zero_output_are_the_shared_head_model():
    """W2 = 0 and every exit norm equal to the final norm: the adapter model is
    the per-exit-head model whose heads are all the final LM head (pinned
    through the independent LLaMA above)."""
    d = W.TINY.d_model
    rng = np.random.default_rng(4)
    ad, w2 = _adapter_model(lambda e: rng.normal(size=(32, d)).astype(np.float32),
                            lambda e: np.zeros((d, 32), np.float32), same_norms=True)
    per = {**w2, "exits": [dict(e, head=w2["exits"][-1]["head"]) for e in w2["exits"]]}
    ref = O.OracleModel(W.TINY, per)
    toks = np.stack([W.make_prompts(W.WORKLOADS["T"], seed=s)[0][:16] for s in (1, 2)])
    np.testing.assert_allclose(O.score_mixture(ad, toks)[0], O.score_mixture(ref, toks)[0], rtol=0, atol=1e-12)


def test_adapter_head_input_against_torch():
    """One exit's head input, m = h + W2 silu(W1 n_k) then the final RMSNorm,
    against torch's silu and rms_norm in float64 (fp32 model: no rounding)."""
    import torch
    import torch.nn.functional as F
    d = W.TINY.d_model
    rng = np.random.default_rng(6)
    ad, w2 = _adapter_model(lambda e: (rng.normal(size=(16, d)) / np.sqrt(d)).astype(np.float32),
                            lambda e: (rng.normal(size=(d, 16)) * 0.3).astype(np.float32))
    h = rng.normal(size=(8, d))
    for k in range(W.TINY.n_exits - 1):
        e = w2["exits"][k]
        n = F.rms_norm(torch.from_numpy(h), (d,), torch.from_numpy(e["norm"].astype(np.float64)), 1e-5)
        m = torch.from_numpy(h) + F.silu(n @ torch.from_numpy(e["adapter_w1"].astype(np.float64)).T) @ \
            torch.from_numpy(e["adapter_w2"].astype(np.float64)).T
        want = F.rms_norm(m, (d,), torch.from_numpy(w2["exits"][-1]["norm"].astype(np.float64)), 1e-5).numpy()
        np.testing.assert_allclose(ad.head_input(k, h), want, rtol=0, atol=1e-12)
    # the last exit reads its own state, adapters or not
    np.testing.assert_array_equal(ad.head_input(3, h), ad.exit_state(3, h))


@pytest.mark.parametrize("pattern", ["random", "all1", "last"])
def test_layers_of_an_exit_block_keep_equal_cache_lengths(pattern):
    """Exits happen only after a block's last layer, so at every step the
    layers between two exits have equal cache lengths and hence run the same
    rows: the GPU plans each block once.  Checked on a 6-layer model with
    blocks of two layers, under forced exit patterns, and after the flush."""
    cfg = W.ModelConfig("blocks-of-two", 6, 64, 2, 32, 172, 256, (2, 4, 6), W.F32)
    model = O.OracleModel(cfg, W.make_weights(cfg, seed=1))
    prompts = [W.make_prompts(W.WORKLOADS["T"], seed=s)[0][:n] for s, n in ((1, 5), (2, 11), (3, 1))]
    dec = O.OracleDecoder(model, prompts, 24)
    rng = np.random.default_rng(9)
    blocks = [(0, 2), (2, 4), (4, 6)]
    for s in range(24):
        ex = {"random": list(rng.integers(1, 4, size=3)), "all1": [1, 1, 1], "last": [3, 3, 3]}[pattern]
        dec.step(77 + s, forced_exits=ex)
        for b in range(3):
            lens = dec.caches[b].lens
            for l0, l1 in blocks:
                assert len(set(lens[l0:l1])) == 1, (s, b, lens)
    dec.flush()
    for b in range(3):
        assert len(set(dec.caches[b].lens)) == 1


def test_router_bias_calibration_hits_the_target_stop_rates():
    """The calibrated biases make E[sigmoid(b_k + eps)], eps ~ N(0, 0.02^2 d),
    the conditional stop rate of each junction (target exit mass
    0.4/0.25/0.2/0.15): checked by Monte Carlo, not by the quadrature used to
    solve for them, and the implied exit masses multiply back to the target."""
    d = 1536
    b = W.calibrate_router_biases(d)
    eps = np.random.default_rng(0).normal(0.0, 0.02 * np.sqrt(d), size=2_000_000)
    c = [float(np.mean(1.0 / (1.0 + np.exp(-(bk + eps))))) for bk in b]
    mass, left = [], 1.0
    for ck in c:
        mass.append(left * ck)
        left *= 1.0 - ck
    mass.append(left)
    np.testing.assert_allclose(mass, W.TARGET_EXIT_MASS, rtol=0, atol=2e-3)
