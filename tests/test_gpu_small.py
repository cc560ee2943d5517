"""GPU parity on the small bf16 model (12 layers, d=768, 12 heads, vocab
32000, exits after layers 3/6/9/12), tcgen05 GEMM path.  Tolerance 2e-2."""
import os

import numpy as np
import pytest

import workloads as W
from oracle import nvium_oracle as O
from tests.nvium_testlib import run_decode_parity

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
    model.score_mixture(toks, logp, nll)
    ref, ref_nll = O.score_mixture(O.OracleModel(CFG, weights), toks)
    np.testing.assert_allclose(logp, ref, atol=2e-2, rtol=0)
    assert abs(nll[0] - ref_nll) <= 2e-2


def test_decode_parity_b4(weights):
    wl = W.WORKLOADS["S"]
    prompts = [p[:n] for p, n in zip(W.make_prompts(wl), (64, 33, 100, 7))]
    chk, state, dec, _ = run_decode_parity(nv, CFG, weights, prompts, 24)
    print(f"near ties: exits {chk.exit_ties} tokens {chk.token_ties}, max logp err {chk.max_logp_err:.2e}")
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
