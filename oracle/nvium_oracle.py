"""Plain CPU oracle for the N-vium mixture-of-exits hot path (numpy, float64).

TEST INFRASTRUCTURE.  Only the tests, the package entry's smoke check and the
benchmark's CPU-baseline / reference leg may import or run anything under
``oracle/``.  The CUDA library never does, and the two share no code: the only
common module is ``workloads`` (seeded inputs, no arithmetic of the method).

What it follows, from "N-vium: Mixture-of-Exits Transformer for Accelerated
Exact Generation" (arXiv 2605.13190; gist.science technical summary and the
abstract):

* section 2 "Architektur": the L layers split into N_V blocks, a router at the
  end of each block gives w_k, the exit probability is the stick-breaking
  product p_k = w_k * prod_{j<k} (1 - w_j) with w_{N_V} = 1, and the next-token
  distribution is the mixture pi_mix = sum_k p_k pi_k;
* section 2 "Inferenz: Piggybacking": a token that exits at node k defers the
  layers above the exit; later tokens reaching those depths carry the deferred
  rows in the same batched pass, so every KV cache ends complete and exact;
* section 4 and the abstract: LLaMA-2 backbone (RMSNorm, SwiGLU, RoPE), exact
  sampling from the mixture, and exact recovery of the standard transformer
  when the intermediate exits get zero routing mass (section 5).

Readings where the pages are silent (all listed in the design notes): each exit
has its own RMSNorm and linear head; the router is a scalar sigmoid on the
exit-normalised state; an exit is drawn by sequential stop/continue
(stop at k iff u_k < w_k), then the token by Gumbel-max at temperature 1 with
ties to the lowest id; random numbers come from Philox4x32-10 with
key = (seed lo, seed hi) and counter = (b, t, stream, block);
U = ((x >> 9) + 0.5) * 2^-23; RMSNorm eps 1e-5, RoPE theta 1e4 with the
rotate-half pairing (i, i + head_dim/2); for bf16 models the inputs of every
product with a bf16 weight or cache (normed activations, q, k, v, attention
output, SwiGLU product, exit-normalised state) are rounded to bf16
(round-to-nearest-even) and everything else stays float64.

Parity status: every function here is pinned by a CPU test (closed forms,
library routines, an independent LLaMA implementation, known-answer vectors,
chi-square tests); the absolute log-probabilities of the random 1.5B model
have no printed value to pin them and are checked only against the GPU path.
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence

import numpy as np

import workloads as _wl

# --------------------------------------------------------------------------
# Philox4x32-10 (Salmon, Moraes, Dror, Shaw: "Parallel Random Numbers: As Easy
# as 1, 2, 3", SC'11, section 3.2): a 10-round counter-based generator; each
# round multiplies two counter words by fixed odd constants and mixes the high
# and low halves with the other two words and the round key; the key is bumped
# by the Weyl constants between rounds.
# --------------------------------------------------------------------------
_PHILOX_M0 = 0xD2511F53
_PHILOX_M1 = 0xCD9E8D57
_PHILOX_W0 = 0x9E3779B9
_PHILOX_W1 = 0xBB67AE85
_MASK32 = 0xFFFFFFFF


def philox4x32_10(ctr, key):
    """Philox4x32-10 on arrays.

    ctr: 4 arrays (or ints) of uint32 counter words c0..c3 (broadcastable);
    key: 2 arrays (or ints) k0, k1.  Returns 4 uint64 arrays holding 32-bit
    outputs.
    """
    c = [np.asarray(x, dtype=np.uint64) & np.uint64(_MASK32) for x in ctr]
    k0 = np.asarray(key[0], dtype=np.uint64) & np.uint64(_MASK32)
    k1 = np.asarray(key[1], dtype=np.uint64) & np.uint64(_MASK32)
    m0 = np.uint64(_PHILOX_M0)
    m1 = np.uint64(_PHILOX_M1)
    mask = np.uint64(_MASK32)
    s32 = np.uint64(32)
    for r in range(10):
        if r > 0:
            k0 = (k0 + np.uint64(_PHILOX_W0)) & mask
            k1 = (k1 + np.uint64(_PHILOX_W1)) & mask
        p0 = m0 * c[0]            # < 2^64, exact in uint64
        p1 = m1 * c[2]
        hi0, lo0 = p0 >> s32, p0 & mask
        hi1, lo1 = p1 >> s32, p1 & mask
        c = [hi1 ^ c[1] ^ k0, lo1, hi0 ^ c[3] ^ k1, lo0]
    return c


def uniform01(x) -> np.ndarray:
    """32-bit output -> U in (0, 1): ((x >> 9) + 0.5) * 2^-23 (exact in fp32)."""
    x = np.asarray(x, dtype=np.uint64)
    return ((x >> np.uint64(9)).astype(np.float64) + 0.5) * 2.0 ** -23


STREAM_EXIT = 0
STREAM_GUMBEL = 1


def _seed_key(seed):
    s = np.asarray(seed, dtype=np.uint64)
    return (s & np.uint64(_MASK32), s >> np.uint64(32))


def exit_uniform(seed, b: int, t: int, k: int) -> np.ndarray:
    """u_k for junction k (1-based, k < N_V): counter (b, t, 0, (k-1)//4), lane (k-1)%4."""
    blk, lane = (k - 1) // 4, (k - 1) % 4
    out = philox4x32_10((b, t, STREAM_EXIT, blk), _seed_key(seed))
    return uniform01(out[lane])


def gumbel_noise(seed, b: int, t: int, vocab: int) -> np.ndarray:
    """g_v = -log(-log U_v), U_v from counter (b, t, 1, v//4), lane v%4.

    ``seed`` may be an array of shape [n]; the result is then [n, vocab].
    """
    seed = np.asarray(seed, dtype=np.uint64)
    nblk = (vocab + 3) // 4
    blocks = np.arange(nblk, dtype=np.uint64)
    key = _seed_key(seed[..., None] if seed.ndim else seed)
    out = philox4x32_10((b, t, STREAM_GUMBEL, blocks), key)
    u = uniform01(np.stack(out, axis=-1).reshape(out[0].shape[:-1] + (nblk * 4,)))
    u = u[..., :vocab]
    return -np.log(-np.log(u))


# --------------------------------------------------------------------------
# numeric helpers
# --------------------------------------------------------------------------

def bf16_round(x: np.ndarray) -> np.ndarray:
    """Nearest bfloat16 value (8 significant bits, ties to even), as float64."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m * 2^e, |m| in [0.5, 1)
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def widen(a) -> np.ndarray:
    """A stored tensor (float32, or bf16 bits as uint16) as float64 values."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm (LLaMA-2): g * x / sqrt(mean(x^2) + eps) over the last axis."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * g


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotary embedding, rotate-half pairing: x [n, H, hd], pos [n].

    For i < hd/2 the pair (x_i, x_{i+hd/2}) is rotated by the angle
    pos * theta^(-2i/hd).
    """
    hd = x.shape[-1]
    half = hd // 2
    inv = theta ** (-2.0 * np.arange(half, dtype=np.float64) / hd)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]      # [n, half]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def attention_row(q: np.ndarray, K: np.ndarray, V: np.ndarray, p: int, scale: float) -> np.ndarray:
    """Causal softmax attention of one row at position p (LLaMA-2): q [H, hd]
    against the cached keys and values of positions 0..p (K, V [>= p+1, H, hd]);
    o_h = sum_j softmax_j(q_h . k_jh * scale) v_jh.  Returns [H, hd]."""
    Kc, Vc = K[: p + 1], V[: p + 1]
    s = np.einsum("hd,jhd->hj", q, Kc) * scale
    s = s - s.max(axis=1, keepdims=True)
    e = np.exp(s)
    a = e / e.sum(axis=1, keepdims=True)
    return np.einsum("hj,jhd->hd", a, Vc)


def causal_attention_rows(q: np.ndarray, K: np.ndarray, V: np.ndarray, pos: np.ndarray, scale: float,
                          rows_per_block: int = 256) -> np.ndarray:
    """attention_row for many rows of one sequence at once: q [n, H, hd],
    positions pos [n]; row i attends to positions 0..pos[i].  The same
    definition, evaluated as one score matrix per block of rows with the keys
    beyond each row's position masked out (they get weight exactly 0).
    Returns [n, H, hd]."""
    pos = np.asarray(pos, dtype=np.int64)
    n = q.shape[0]
    out = np.empty_like(q)
    for r0 in range(0, n, rows_per_block):
        r1 = min(n, r0 + rows_per_block)
        P = int(pos[r0:r1].max()) + 1
        qh = q[r0:r1].transpose(1, 0, 2)                       # [H, m, hd]
        s = np.matmul(qh, K[:P].transpose(1, 2, 0)) * scale     # [H, m, P]
        beyond = np.arange(P)[None, :] > pos[r0:r1, None]       # [m, P]
        s = np.where(beyond[None], -np.inf, s)
        s = s - s.max(axis=2, keepdims=True)
        e = np.exp(s)
        a = e / e.sum(axis=2, keepdims=True)
        out[r0:r1] = np.matmul(a, V[:P].transpose(1, 0, 2)).transpose(1, 0, 2)
    return out


def log_sigmoid(z):
    """log sigma(z) = -softplus(-z), computed stably."""
    z = np.asarray(z, dtype=np.float64)
    return -np.logaddexp(0.0, -z)


def logsumexp(a: np.ndarray, axis=-1) -> np.ndarray:
    m = np.max(a, axis=axis, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    return np.squeeze(m, axis=axis) + np.log(np.sum(np.exp(a - m), axis=axis))


# --------------------------------------------------------------------------
# mixture of exits: section 2 "Architektur" (equations for p_k and pi_mix)
# --------------------------------------------------------------------------

ROUTER_NORMAL = 0
ROUTER_FORCE_LAST = 1


def exit_probs(w: np.ndarray) -> np.ndarray:
    """Stick-breaking exit probabilities p_k = w_k prod_{j<k}(1 - w_j), w_{N_V} := 1.

    w: [..., N_V - 1] router probabilities of the intermediate exits.
    Returns [..., N_V].
    """
    w = np.asarray(w, dtype=np.float64)
    ones = np.ones(w.shape[:-1] + (1,))
    wf = np.concatenate([w, ones], axis=-1)
    surv = np.concatenate([ones, np.cumprod(1.0 - w, axis=-1)], axis=-1)
    return wf * surv


def log_exit_probs(z: np.ndarray, mode: int = ROUTER_NORMAL) -> np.ndarray:
    """log p_k from router logits z [..., N_V - 1]: log w_k = log sigma(z_k),
    log(1 - w_j) = log sigma(-z_j).  In the zero-intermediate-mass mode
    (section 5: the standard transformer is recovered exactly), w_k := 0."""
    z = np.asarray(z, dtype=np.float64)
    n = z.shape[-1] + 1
    out = np.empty(z.shape[:-1] + (n,))
    if mode == ROUTER_FORCE_LAST:
        out[...] = -np.inf
        out[..., -1] = 0.0
        return out
    lw = log_sigmoid(z)
    l1w = log_sigmoid(-z)
    acc = np.zeros(z.shape[:-1])
    for k in range(n - 1):
        out[..., k] = lw[..., k] + acc
        acc = acc + l1w[..., k]
    out[..., -1] = acc
    return out


def mixture_logprob(log_p: np.ndarray, log_pi: np.ndarray) -> np.ndarray:
    """log pi_mix(x) = log sum_k p_k pi_k(x), in log space: LSE_k(log p_k + log pi_k)."""
    return logsumexp(log_p + log_pi, axis=-1)


def expected_depth(log_p: np.ndarray, exit_layers: Sequence[int], n_layers: int) -> np.ndarray:
    """Expected normalised layer depth of a token (section 2 "Training": the
    compute penalty L_compute is the expected normalised depth): a token that
    exits at node k has run exit_layers[k] of the n_layers layers, so
    E[depth] = sum_k p_k * exit_layers[k] / n_layers."""
    frac = np.asarray(exit_layers, dtype=np.float64) / float(n_layers)
    return np.exp(np.asarray(log_p, dtype=np.float64)) @ frac


# --------------------------------------------------------------------------
# backbone (LLaMA-2, section 4) on rows of one sequence
# --------------------------------------------------------------------------

class SeqCache:
    """Per-sequence KV cache: one [capacity, H, hd] K and V array per layer,
    with its own length per layer (the piggybacking rule lets them differ)."""

    def __init__(self, n_layers: int, capacity: int, n_heads: int, head_dim: int):
        self.K = [np.zeros((capacity, n_heads, head_dim)) for _ in range(n_layers)]
        self.V = [np.zeros((capacity, n_heads, head_dim)) for _ in range(n_layers)]
        self.lens = [0] * n_layers   # len[m]: positions whose layer-m KV is present


class OracleModel:
    """Weights (float32 copies of the stored values; widened to float64 at use)."""

    def __init__(self, cfg, weights: dict, router_mode: int = ROUTER_NORMAL, cache_f64: Optional[bool] = None):
        self.cfg = cfg
        self.mode = router_mode
        self.bf16 = cfg.dtype == _wl.BF16
        # keep float64 copies of the weights when they fit comfortably
        self._f64 = {} if (cache_f64 if cache_f64 is not None else cfg.n_params() < 4e8) else None
        f = _wl.as_f32
        self.tok_emb = f(weights["tok_emb"])
        self.layers = [{k: f(v) for k, v in L.items()} for L in weights["layers"]]
        self.exits = []
        for k, E in enumerate(weights["exits"]):
            e = {"norm": f(E["norm"])}
            if "head" in E:  # with adapters only the last exit's head is read
                e["head"] = f(E["head"])
            if k < cfg.n_exits - 1:
                e["router_w"] = f(E["router_w"])
                e["router_b"] = float(E["router_b"])
                if getattr(cfg, "router_hidden", 0):
                    e["router_w1"] = f(E["router_w1"])
                    e["router_b1"] = np.asarray(E["router_b1"], dtype=np.float32)
                    e["router_w2"] = np.asarray(E["router_w2"], dtype=np.float32)
                if getattr(cfg, "adapter_hidden", 0):
                    e["adapter_w1"] = f(E["adapter_w1"])
                    e["adapter_w2"] = f(E["adapter_w2"])
            self.exits.append(e)
        self.adapters = bool(getattr(cfg, "adapter_hidden", 0))
        self.exit_at = {l: k for k, l in enumerate(cfg.exit_layers)}  # layer -> exit index (0-based)
        # rows of one sequence attend through one masked product per block of
        # rows (causal_attention_rows); False: one row at a time (attention_row)
        self.block_attention = True

    # rounding point of the bf16 numerics contract
    def rnd(self, x):
        return bf16_round(x) if self.bf16 else x

    def mm(self, x: np.ndarray, w32: np.ndarray) -> np.ndarray:
        """y = x W^T with x [n, in] float64 and W [out, in]."""
        if self._f64 is None:
            return x @ w32.astype(np.float64).T
        w = self._f64.get(id(w32))
        if w is None:
            w = self._f64[id(w32)] = w32.astype(np.float64)
        return x @ w.T

    def embed(self, tokens) -> np.ndarray:
        return self.tok_emb[np.asarray(tokens, dtype=np.int64)].astype(np.float64)

    def layer_rows(self, m: int, h: np.ndarray, pos: Sequence[int], cache: SeqCache) -> np.ndarray:
        """Layer m (0-based) on rows of one sequence at ascending positions ``pos``.

        Writes the rows' K and V into the cache at layer m, then lets row p
        attend causally to positions 0..p of layer m.  Returns the new residual.
        """
        return self.layer_rows_multi(m, h, pos, [cache] * len(pos))

    def layer_rows_multi(self, m: int, h: np.ndarray, pos: Sequence[int], caches: List[SeqCache]) -> np.ndarray:
        """Layer m on rows that may belong to several sequences: row i sits at
        position pos[i] of the sequence whose cache is caches[i]; each
        sequence's rows come in ascending position order.  The projections are
        per-row products (stacked into one matrix product); attention of row i
        reads only its own sequence's cache."""
        cfg, L = self.cfg, self.layers[m]
        H, hd = cfg.n_heads, cfg.head_dim
        pos = np.asarray(pos, dtype=np.int64)
        n = h.shape[0]
        # attention sub-block
        x = self.rnd(rmsnorm(h, widen(L["attn_norm"]), cfg.rms_eps))
        q = self.mm(x, L["wq"]).reshape(n, H, hd)
        k = self.mm(x, L["wk"]).reshape(n, H, hd)
        v = self.mm(x, L["wv"]).reshape(n, H, hd)
        q = self.rnd(rope(q, pos, cfg.rope_theta))
        k = self.rnd(rope(k, pos, cfg.rope_theta))
        v = self.rnd(v)
        for i in range(n):
            caches[i].K[m][pos[i]] = k[i]
            caches[i].V[m][pos[i]] = v[i]
        scale = 1.0 / math.sqrt(hd)
        one_seq = n > 1 and all(c is caches[0] for c in caches)
        if one_seq and self.block_attention:
            o = causal_attention_rows(q, caches[0].K[m], caches[0].V[m], pos, scale)
        else:
            o = np.empty((n, H, hd))
            for i in range(n):
                o[i] = attention_row(q[i], caches[i].K[m], caches[i].V[m], int(pos[i]), scale)
        o = self.rnd(o.reshape(n, H * hd))
        h = h + self.mm(o, L["wo"])
        # MLP sub-block (SwiGLU)
        x = self.rnd(rmsnorm(h, widen(L["mlp_norm"]), cfg.rms_eps))
        a = self.rnd(silu(self.mm(x, L["wg"])) * self.mm(x, L["wu"]))
        return h + self.mm(a, L["wd"])

    # ---- exits ----------------------------------------------------------
    def exit_state(self, k: int, h: np.ndarray) -> np.ndarray:
        """n_k = RMSNorm_k(h) (rounded to bf16 for bf16 models)."""
        return self.rnd(rmsnorm(h, widen(self.exits[k]["norm"]), self.cfg.rms_eps))

    def router_logit(self, k: int, nk: np.ndarray) -> np.ndarray:
        """z_k = r_k . n_k + b_k (k < N_V - 1, 0-based), or, with a router MLP
        (section 2 "Architektur": a router MLP maps the node's hidden state to
        w_k), z_k = v_k . silu(U_k n_k + c_k) + b_k, silu(x) = x sigmoid(x)."""
        e = self.exits[k]
        if "router_w1" in e:
            a = np.asarray(nk, dtype=np.float64) @ widen(e["router_w1"]).T + widen(e["router_b1"])
            return silu(a) @ widen(e["router_w2"]) + e["router_b"]
        return nk @ widen(e["router_w"]) + e["router_b"]

    def router_prob(self, k: int, nk: np.ndarray) -> np.ndarray:
        if self.mode == ROUTER_FORCE_LAST:
            return np.zeros(np.shape(nk)[:-1])
        z = self.router_logit(k, nk)
        return 1.0 / (1.0 + np.exp(-z))

    def head_input(self, k: int, h: np.ndarray) -> np.ndarray:
        """What exit k's head reads.  Per-exit heads: the exit state n_k.
        Shared head (section 2 "Architektur": all exits share the final LM
        head, light adapter MLPs map the intermediate states to the geometry
        the head expects): for k < N_V - 1, m = h + W2 silu(W1 n_k) and the
        head reads the final norm of m (the last exit's norm); the last exit
        reads its own state."""
        if not self.adapters or k == self.cfg.n_exits - 1:
            return self.exit_state(k, h)
        e = self.exits[k]
        nk = self.exit_state(k, h)
        hid = self.rnd(silu(self.mm(np.atleast_2d(nk), e["adapter_w1"])))
        m = np.atleast_2d(h) + self.mm(hid, e["adapter_w2"])
        last = self.cfg.n_exits - 1
        return self.rnd(rmsnorm(m, widen(self.exits[last]["norm"]), self.cfg.rms_eps)).reshape(np.shape(h))

    def head_logits(self, k: int, x: np.ndarray) -> np.ndarray:
        """Logits of exit k from its head input x (head_input): exit k's own
        head, or with adapters the one shared head (the last exit's)."""
        head = self.exits[-1]["head"] if self.adapters else self.exits[k]["head"]
        return self.mm(np.atleast_2d(x), head)

    # ---- full forward over whole sequences ------------------------------
    def forward_sequence(self, tokens: Sequence[int], cache: Optional[SeqCache] = None,
                         collect_exits: bool = True, with_heads: bool = False):
        """Standard full-depth forward over positions 0..n-1 of one sequence.

        Returns (h_final [n, d], exit states {k: n_k [n, d]}, cache), and with
        with_heads also {k: head input [n, d]} (head_input of each exit).
        """
        cfg = self.cfg
        n = len(tokens)
        if cache is None:
            cache = SeqCache(cfg.n_layers, n, cfg.n_heads, cfg.head_dim)
        h = self.embed(tokens)
        pos = np.arange(n)
        states, heads = {}, {}
        for m in range(cfg.n_layers):
            h = self.layer_rows(m, h, pos, cache)
            cache.lens[m] = n
            if collect_exits and (m + 1) in self.exit_at:
                k = self.exit_at[m + 1]
                states[k] = self.exit_state(k, h)
                if with_heads:
                    heads[k] = self.head_input(k, h)
        if with_heads:
            return h, states, cache, heads
        return h, states, cache


# --------------------------------------------------------------------------
# scoring: per-position mixture log-probabilities (the training objective's
# forward value, section 2 "Training": cross-entropy of pi_mix)
# --------------------------------------------------------------------------

def score_mixture(model: OracleModel, tokens: np.ndarray):
    """tokens [B, S] -> (logp [B, S-1], mean NLL).

    logp[b, t] = log pi_mix(x_{t+1} | x_{<=t}) = LSE_k(log p_k + log pi_k(x_{t+1})),
    with log p_k from the routers at position t and
    log pi_k(v) = logit_k[v] - LSE_v logit_k.
    """
    logp, nll, _, _ = score_mixture_with_depth(model, tokens)
    return logp, nll


def score_mixture_with_depth(model: OracleModel, tokens: np.ndarray):
    """score_mixture plus the compute-penalty forward: (logp [B, S-1], mean
    NLL, depth [B, S-1], mean depth), depth[b, t] = expected normalised layer
    depth of position t (expected_depth of its exit probabilities)."""
    cfg = model.cfg
    tokens = np.asarray(tokens)
    B, S = tokens.shape
    out = np.empty((B, S - 1))
    depth = np.empty((B, S - 1))
    for b in range(B):
        _, states, _, heads = model.forward_sequence(tokens[b, : S - 1], with_heads=True)
        tgt = tokens[b, 1:].astype(np.int64)
        z = np.zeros((S - 1, cfg.n_exits - 1))
        logpi = np.empty((S - 1, cfg.n_exits))
        for k in range(cfg.n_exits):
            nk = states[k]
            if k < cfg.n_exits - 1:
                z[:, k] = model.router_logit(k, nk)
            lg = model.head_logits(k, heads[k])
            logpi[:, k] = lg[np.arange(S - 1), tgt] - logsumexp(lg, axis=-1)
        lp = log_exit_probs(z, model.mode)
        out[b] = mixture_logprob(lp, logpi)
        depth[b] = expected_depth(lp, cfg.exit_layers, cfg.n_layers)
    return out, float(-out.mean()), depth, float(depth.mean())


def dense_logprobs(model: OracleModel, tokens: Sequence[int]) -> np.ndarray:
    """The plain L-layer transformer: log-softmax of the last exit's head at
    every position (final norm = exit N_V's norm).  [n, V]."""
    _, states, _ = model.forward_sequence(tokens)
    lg = model.head_logits(model.cfg.n_exits - 1, states[model.cfg.n_exits - 1])
    return lg - logsumexp(lg, axis=-1)[:, None]


# --------------------------------------------------------------------------
# exact sampling: exit by sequential stop/continue, token by Gumbel-max
# --------------------------------------------------------------------------

def sample_exit(u: np.ndarray, w: np.ndarray) -> np.ndarray:
    """First k with u_k < w_k (k < N_V); N_V (1-based) if none.

    u, w: [..., N_V - 1].  P(exit = k) = w_k prod_{j<k}(1 - w_j) = p_k.
    """
    stop = np.asarray(u) < np.asarray(w)
    n = stop.shape[-1] + 1
    first = np.where(stop.any(axis=-1), np.argmax(stop, axis=-1) + 1, n)
    return first


def gumbel_argmax(logits: np.ndarray, g: np.ndarray) -> np.ndarray:
    """argmax_v (logit_v + g_v); np.argmax returns the lowest id on ties."""
    return np.argmax(np.asarray(logits) + np.asarray(g), axis=-1)


# --------------------------------------------------------------------------
# deferred decode (section 2 "Inferenz: Piggybacking")
# --------------------------------------------------------------------------

class StepRecord:
    """What one decode step decided, with the margins a parity check needs."""

    def __init__(self):
        self.junctions = []   # (k 1-based, u_k, w_k) for every junction evaluated
        self.exit = None      # 1-based exit used
        self.oracle_exit = None
        self.token = None
        self.oracle_token = None
        self.scores = None    # logit + gumbel at the exit used, [V]
        self.logp = None      # log pi_exit(token)


class OracleDecoder:
    """Deferred (piggybacked) decode of B independent sequences.

    State per sequence b: the tokens so far, t_b = position of the next input
    token, per-layer KV caches with lengths len[b][m], and the residual h of
    every deferred position at its frontier (the number of layers computed).
    Lazy rule: the deferred rows at layer m run only when the sequence's new
    token reaches layer m (or at flush).
    """

    def __init__(self, model: OracleModel, prompts: List[np.ndarray], max_new: int):
        self.model = model
        cfg = model.cfg
        self.B = len(prompts)
        self.ids = list(range(self.B))   # sequence index b used in the Philox counters
        self.tokens = [list(map(int, p)) for p in prompts]
        self.caches = []
        self.pending = []   # per b: {pos: h}
        self.t = []
        for b, p in enumerate(prompts):
            P = len(p)
            cache = SeqCache(cfg.n_layers, P + max_new + 1, cfg.n_heads, cfg.head_dim)
            self.caches.append(cache)
            self.pending.append({})
            self.t.append(P - 1)
        self.prefill()

    def prefill(self):
        """Positions 0..P-2 at full depth; position P-1 is the first decode input."""
        m = self.model
        for b in range(self.B):
            P = len(self.tokens[b])
            cache = self.caches[b]
            if P > 1:
                h = m.embed(self.tokens[b][: P - 1])
                pos = np.arange(P - 1)
                for layer in range(m.cfg.n_layers):
                    h = m.layer_rows(layer, h, pos, cache)
            cache.lens = [P - 1] * m.cfg.n_layers

    def _run_layer(self, b: int, layer: int, positions: List[int]):
        if not positions:
            return
        pend = self.pending[b]
        h = np.stack([pend[p] for p in positions])
        h = self.model.layer_rows(layer, h, positions, self.caches[b])
        for i, p in enumerate(positions):
            pend[p] = h[i]
        self.caches[b].lens[layer] = positions[-1] + 1

    def step(self, seed: int, forced_exits=None, forced_tokens=None) -> List[StepRecord]:
        """One decode step of every sequence.  ``forced_exits`` /
        ``forced_tokens`` ([B]) make the oracle follow another
        implementation's choices (teacher forcing) while it still records its
        own decisions and their margins."""
        model, cfg = self.model, self.model.cfg
        B = self.B
        recs = [StepRecord() for _ in range(B)]
        active = [True] * B
        for b in range(B):
            self.pending[b][self.t[b]] = model.embed([self.tokens[b][self.t[b]]])[0]
        for layer in range(cfg.n_layers):
            rows = []          # (b, pos) in sequence order, ascending positions
            for b in range(B):
                if active[b]:
                    rows += [(b, p) for p in range(self.caches[b].lens[layer], self.t[b] + 1)]
            if not rows:
                break
            h = np.stack([self.pending[b][p] for b, p in rows])
            h = model.layer_rows_multi(layer, h, [p for _, p in rows], [self.caches[b] for b, _ in rows])
            for i, (b, p) in enumerate(rows):
                self.pending[b][p] = h[i]
                self.caches[b].lens[layer] = p + 1
            if (layer + 1) not in model.exit_at:
                continue
            k0 = model.exit_at[layer + 1]            # 0-based exit index
            for b in range(B):
                if not active[b]:
                    continue
                rec, t = recs[b], self.t[b]
                nk = model.exit_state(k0, self.pending[b][t])
                if k0 < cfg.n_exits - 1:
                    w = np.asarray(model.router_prob(k0, nk)).item()
                    u = np.asarray(exit_uniform(seed, self.ids[b], t, k0 + 1)).item()
                    rec.junctions.append((k0 + 1, u, w))
                    own_stop = u < w
                else:
                    own_stop = True
                if own_stop and rec.oracle_exit is None:
                    rec.oracle_exit = k0 + 1
                fe = None if forced_exits is None else int(forced_exits[b])
                if (own_stop if fe is None else fe == k0 + 1):
                    active[b] = False
                    hin = model.head_input(k0, self.pending[b][t]) if model.adapters else nk
                    lg = model.head_logits(k0, hin)[0]
                    sc = lg + gumbel_noise(seed, self.ids[b], t, cfg.vocab)
                    rec.scores = sc
                    rec.oracle_token = int(np.argmax(sc))
                    tok = rec.oracle_token if forced_tokens is None else int(forced_tokens[b])
                    rec.logp = float(lg[tok] - logsumexp(lg))
                    rec.token = tok
                    rec.exit = k0 + 1
        for b in range(B):
            rec = recs[b]
            if rec.oracle_exit is None:
                rec.oracle_exit = cfg.n_exits
            done = self.caches[b].lens[cfg.n_layers - 1]
            for p in [p for p in self.pending[b] if p < done]:
                del self.pending[b][p]
            self.tokens[b].append(rec.token)
            self.t[b] += 1
        return recs

    def step_seq(self, b: int, seed: int, forced_exit: Optional[int] = None,
                 forced_token: Optional[int] = None) -> StepRecord:
        """One decode step of sequence b alone (the others do not move)."""
        saved = self.B, self.tokens, self.caches, self.pending, self.t, self.ids
        try:
            self.B = 1
            self.tokens, self.caches = [saved[1][b]], [saved[2][b]]
            self.pending, self.t, self.ids = [saved[3][b]], [saved[4][b]], [saved[5][b]]
            rec = self.step(seed, None if forced_exit is None else [forced_exit],
                            None if forced_token is None else [forced_token])[0]
            saved[4][b] = self.t[0]
        finally:
            self.B, self.tokens, self.caches, self.pending, self.t, self.ids = saved
        return rec

    def flush(self):
        """Run every deferred row through the layers it still owes
        (layers above the first exit), so that len[b][m] = t_b for all m."""
        cfg = self.model.cfg
        for b in range(self.B):
            t = self.t[b]
            for layer in range(cfg.exit_layers[0], cfg.n_layers):
                rows = list(range(self.caches[b].lens[layer], t))
                self._run_layer(b, layer, rows)
                self.caches[b].lens[layer] = t
            self.pending[b].clear()

    def deferred_rows(self, b: int) -> int:
        """Positions still owing layers (pending at the last layer)."""
        return self.t[b] - self.caches[b].lens[self.model.cfg.n_layers - 1]


def step_distribution(model: OracleModel, junction_states: List[np.ndarray]):
    """Exact next-token law of one step from the exit states n_k of the new
    token: returns (p [N_V], pi [N_V, V]) with p the stick-breaking exit
    probabilities and pi_k = softmax(head_k n_k)."""
    cfg = model.cfg
    assert not model.adapters, "exit states are the head inputs only without adapters"
    w = np.array([np.asarray(model.router_prob(k, junction_states[k])).item() for k in range(cfg.n_exits - 1)])
    p = exit_probs(w)
    pi = np.empty((cfg.n_exits, cfg.vocab))
    for k in range(cfg.n_exits):
        lg = model.head_logits(k, junction_states[k])[0]
        pi[k] = np.exp(lg - logsumexp(lg))
    return p, pi
