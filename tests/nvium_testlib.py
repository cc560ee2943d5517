"""Helpers shared by the GPU parity tests (not a test module)."""
import numpy as np

import workloads as W
from oracle import nvium_oracle as O


def tolerance(cfg) -> float:
    """Absolute tolerance on log-probabilities, router margins and Gumbel
    scores: 1e-4 for the fp32 model, 2e-2 for bf16 models."""
    return 1e-4 if cfg.dtype == W.F32 else 2e-2


def kv_close(gpu, ref, cfg):
    """KV entries: the tolerance, plus one bf16 step of the value for bf16
    caches (both sides store rounded values; a rounding flip moves one step)."""
    tol = tolerance(cfg)
    rtol = 2.0 ** -7 if cfg.dtype == W.BF16 else 0.0
    np.testing.assert_allclose(gpu, ref, atol=tol, rtol=rtol)


def kv_close_counted(gpu, ref, cfg, what="", max_frac=1e-5, hard_factor=1.5):
    """Full-depth (48-layer) bf16 caches: two pipelines that each round to
    bf16 at every layer drift apart slowly, so a rare element crosses the
    stated bound (the tolerance plus one bf16 step of the value).  Such
    elements are counted like near-ties: at most `max_frac` of the elements
    may exceed their bound, and no element may exceed `hard_factor` times its
    own bound.  Returns (fraction over, max |delta|, max |delta| / bound)."""
    tol = tolerance(cfg)
    rtol = 2.0 ** -7 if cfg.dtype == W.BF16 else 0.0
    d = np.abs(np.asarray(gpu, np.float64) - np.asarray(ref, np.float64))
    bound = tol + rtol * np.abs(np.asarray(ref, np.float64))
    ratio = d / bound
    over = float(np.mean(ratio > 1.0)) if d.size else 0.0
    mx = float(d.max()) if d.size else 0.0
    worst = float(ratio.max()) if d.size else 0.0
    print(f"kv {what}: {over:.2e} of {d.size} elements over their bound, max |delta| {mx:.4f}, "
          f"max |delta|/bound {worst:.3f}")
    assert over <= max_frac, (what, over, mx)
    assert worst <= hard_factor, (what, worst, mx)
    return over, mx, worst


def gpu_kv(state, b, layer, max_len, cfg):
    K, V, n = state.read_kv(b, layer, max_len)
    return W.as_f32(K).astype(np.float64), W.as_f32(V).astype(np.float64), n


class StepChecker:
    """Step-synchronous comparison with teacher forcing.

    Exits: with the device's own router probabilities (``w_gpu``, from
    State.router_probs) every stop decision must follow them exactly (stop at
    junction k iff u_k < w_k(gpu); u_k is the same Philox number on both
    sides), |w_k(gpu) - w_k(oracle)| must stay within tau, and an exit that
    differs from the oracle's is a near-tie only when u_k lies between the two
    w_k; such ties are counted, with their expected number sum |dw| (the
    chance that u falls between the two values).  Without ``w_gpu`` a
    mismatch is a near-tie iff |u_k - w_k(oracle)| <= tau.
    Tokens: a mismatch is a near-tie iff the oracle's perturbed scores of the
    two ids differ by <= tau; counted."""

    def __init__(self, cfg):
        self.cfg = cfg
        self.tau = tolerance(cfg)
        self.exit_ties = 0
        self.token_ties = 0
        self.steps = 0
        self.max_logp_err = 0.0
        self.max_dw = 0.0
        self.expected_exit_ties = 0.0
        self.junctions = 0

    def check(self, recs, tok, ex, lp, w_gpu=None):
        ne = self.cfg.n_exits
        for b, rec in enumerate(recs):
            ge, gt = int(ex[b]), int(tok[b])
            assert 1 <= ge <= ne
            if w_gpu is not None:
                seen = set()
                for (k, u, w) in rec.junctions:
                    wg = float(w_gpu[k - 1][b])
                    assert np.isfinite(wg), f"b={b}: junction {k} evaluated by the oracle, not by the GPU"
                    assert (u < wg) == (k == ge), f"b={b} junction {k}: GPU exit {ge} but u={u} w_gpu={wg}"
                    dw = abs(wg - w)
                    assert dw <= self.tau, f"b={b} junction {k}: |w_gpu - w_oracle| = {dw}"
                    self.max_dw = max(self.max_dw, dw)
                    self.expected_exit_ties += dw
                    self.junctions += 1
                    seen.add(k)
                for k in range(1, ne):
                    if k > ge:
                        assert np.isnan(w_gpu[k - 1][b]), f"b={b}: junction {k} beyond the exit was evaluated"
                    elif k not in seen:
                        assert False, f"b={b}: junction {k} evaluated by the GPU, not by the oracle"
            if ge != rec.oracle_exit:
                k = min(ge, rec.oracle_exit)
                uw = [(u, w) for (kk, u, w) in rec.junctions if kk == k]
                assert uw, (b, ge, rec.oracle_exit)
                u, w = uw[0]
                if w_gpu is not None:
                    wg = float(w_gpu[k - 1][b])
                    assert min(w, wg) <= u <= max(w, wg), f"exit mismatch b={b}: u={u} outside [{w}, {wg}]"
                else:
                    assert abs(u - w) <= self.tau, \
                        f"exit mismatch b={b}: gpu {ge} oracle {rec.oracle_exit} u={u} w={w}"
                self.exit_ties += 1
            if gt != rec.oracle_token:
                gap = abs(rec.scores[gt] - rec.scores[rec.oracle_token])
                assert gap <= self.tau, f"token mismatch b={b}: gpu {gt} oracle {rec.oracle_token} gap={gap}"
                self.token_ties += 1
            if lp is not None:
                err = abs(rec.logp - float(lp[b]))
                self.max_logp_err = max(self.max_logp_err, err)
                assert err <= self.tau, f"log-prob b={b}: gpu {lp[b]} oracle {rec.logp}"
        self.steps += 1

    def report(self, what=""):
        msg = (f"{what} near ties: exits {self.exit_ties} (expected {self.expected_exit_ties:.3f} from "
               f"{self.junctions} junctions, max |dw| {self.max_dw:.2e}), tokens {self.token_ties}, "
               f"max |dlogp| {self.max_logp_err:.2e}")
        print(msg)
        return msg


def run_decode_parity(nv, cfg, weights, prompts, steps, seed=1234, max_pending=256, router_mode=0,
                      max_seq=None, check_kv=True):
    """Decode `steps` steps on the GPU and in the oracle (teacher forced),
    flush both, compare the caches.  Returns (checker, state, oracle)."""
    B = len(prompts)
    lens = np.array([len(p) for p in prompts], dtype=np.int32)
    max_seq = max_seq or int(lens.max()) + steps + 8
    model = nv.Model(cfg, weights, max_batch=B, max_seq=max_seq, max_pending=max_pending,
                     router_mode=router_mode)
    state = nv.State(model, B)
    state.prefill(np.concatenate(prompts).astype(np.int32), lens)
    om = O.OracleModel(cfg, weights, router_mode)
    dec = O.OracleDecoder(om, prompts, steps)
    chk = StepChecker(cfg)
    tok = np.zeros(B, np.int32)
    ex = np.zeros(B, np.int32)
    lp = np.zeros(B, np.float32)
    for s in range(steps):
        state.decode_step(seed + s, tok, ex, lp)
        recs = dec.step(seed + s, forced_exits=ex, forced_tokens=tok)
        chk.check(recs, tok, ex, lp, state.router_probs())
    state.sync_status()
    if check_kv:
        state.flush()
        dec.flush()
        state.sync_status()
        for b in range(B):
            for m in range(cfg.n_layers):
                K, V, n = gpu_kv(state, b, m, max_seq, cfg)
                assert n == dec.t[b] == dec.caches[b].lens[m]
                kv_close(K, dec.caches[b].K[m][:n], cfg)
                kv_close(V, dec.caches[b].V[m][:n], cfg)
    return chk, state, dec, model


def chisq_pvalue(counts, expected, min_expected=5.0):
    """Chi-square p-value with the smallest-expectation cells merged until
    every cell expects at least `min_expected` draws."""
    from scipy import stats
    c = np.asarray(counts, dtype=np.float64).ravel()
    e = np.asarray(expected, dtype=np.float64).ravel()
    keep = e > 0
    assert c[~keep].sum() == 0, "draws in a cell of probability zero"
    c, e = c[keep], e[keep]
    order = np.argsort(e)
    c, e = c[order], e[order]
    cut = int(np.sum(e < min_expected))        # cells too small on their own
    if cut > 0:
        while cut < len(e) and e[:cut].sum() < min_expected:
            cut += 1
        c = np.concatenate([[c[:cut].sum()], c[cut:]])
        e = np.concatenate([[e[:cut].sum()], e[cut:]])
    assert np.all(e >= min_expected)
    return stats.chisquare(c, e * c.sum() / e.sum()).pvalue
