"""Seeded synthetic workloads for the N-vium mixture-of-exits decoder.

This module only draws inputs: model configurations, random weights, prompt
token ids and prompt lengths.  It holds none of the method's arithmetic (no
norms, attention, routing or sampling), so both the CPU oracle and the CUDA
library's tests and benchmarks can take their inputs from it.

The pages describe a LLaMA-2-style decoder pretrained on C4 with the LLaMA-2
tokenizer ("N-vium: Mixture-of-Exits Transformer for Accelerated Exact
Generation", gist.science technical summary, section 4).  Neither the corpus
nor trained weights are available, so seeded stand-ins are drawn here:

* weights: every matrix N(0, 0.02^2), one independent PCG64 stream per tensor
  (SeedSequence(seed, spawn_key=(tensor_index,))), stored as float32 for the
  fp32 configuration and rounded to bfloat16 (round-to-nearest-even) for the
  bf16 configurations; norm gains 1.0 unless ``random_gains``;
* router biases: U(-1, 1) for the tiny configuration, otherwise calibrated so
  that the expected exit mass is about [0.4, 0.25, 0.2, 0.15]
  (see :func:`calibrate_router_biases`);
* prompts: uniform ids for the tiny configuration, truncated Zipf(s=1.1)
  ranks over the vocabulary (id = rank - 1) otherwise;
* ragged prompt lengths: U[lo, hi] inclusive.
"""
from __future__ import annotations

import concurrent.futures as _fut
import dataclasses
import os
from typing import Dict, List, Optional, Sequence

import numpy as np

F32 = 0
BF16 = 1


@dataclasses.dataclass(frozen=True)
class ModelConfig:
    """Shape of a mixture-of-exits LLaMA-style decoder.

    ``exit_layers`` are 1-based: exit k reads the residual stream after layer
    ``exit_layers[k-1]``; the last entry equals ``n_layers``.
    """

    name: str
    n_layers: int
    d_model: int
    n_heads: int
    head_dim: int
    d_ff: int
    vocab: int
    exit_layers: tuple
    dtype: int  # F32 or BF16
    rms_eps: float = 1e-5
    rope_theta: float = 10000.0
    # hidden width of the router MLP of every exit but the last; 0: scalar router
    router_hidden: int = 0
    # hidden width of the exit adapters in front of one shared LM head (the
    # last exit's head and norm); 0: every exit has its own head
    adapter_hidden: int = 0

    @property
    def n_exits(self) -> int:
        return len(self.exit_layers)

    def n_params(self) -> int:
        d, f, v = self.d_model, self.d_ff, self.vocab
        per_layer = 4 * d * self.n_heads * self.head_dim + 3 * d * f + 2 * d
        heads = self.n_exits * (v * d + d) + (self.n_exits - 1) * d
        return v * d + self.n_layers * per_layer + heads


@dataclasses.dataclass(frozen=True)
class Workload:
    """A model plus the run shape drawn on it."""

    name: str
    model: ModelConfig
    batch: int
    prompt_len: int            # fixed prompt length (or the upper bound when ragged)
    prompt_len_lo: int         # == prompt_len unless ragged
    steps: int                 # decode steps (0 for scoring)
    mode: str                  # "decode" or "score"
    zipf: bool                 # Zipf(1.1) ids (else uniform)
    philox_seed: int = 1234


TINY = ModelConfig("tiny-fp32", 4, 64, 2, 32, 172, 256, (1, 2, 3, 4), F32)
SMALL = ModelConfig("small-bf16", 12, 768, 12, 64, 2048, 32000, (3, 6, 9, 12), BF16)
X15B = ModelConfig("nvium-1.5b-bf16", 48, 1536, 24, 64, 4096, 32000, (12, 24, 36, 48), BF16)

WORKLOADS: Dict[str, Workload] = {
    "T": Workload("tiny-fp32-b1", TINY, 1, 32, 32, 32, "decode", False),
    "S": Workload("small-bf16-b8", SMALL, 8, 512, 512, 256, "decode", True),
    "X1": Workload("1.5b-bf16-b1-decode", X15B, 1, 2048, 2048, 512, "decode", True),
    "X64": Workload("1.5b-bf16-b64-decode", X15B, 64, 1024, 256, 256, "decode", True),
    "XS": Workload("1.5b-bf16-score-16x2048", X15B, 16, 2048, 2048, 0, "score", True),
}

# Exit mass the bf16 configurations aim for (exits 1..4).
TARGET_EXIT_MASS = (0.4, 0.25, 0.2, 0.15)


# --------------------------------------------------------------------------
# encodings of the stored inputs
# --------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16, round-to-nearest-even; uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def as_f32(arr: np.ndarray) -> np.ndarray:
    """Stored tensor (float32, or bf16 as uint16 bits) as float32 values."""
    if arr.dtype == np.uint16:
        return bf16_bits_to_f32(arr)
    return np.asarray(arr, dtype=np.float32)


# --------------------------------------------------------------------------
# router bias calibration
# --------------------------------------------------------------------------

def calibrate_router_biases(d_model: int, mass: Sequence[float] = TARGET_EXIT_MASS,
                            weight_std: float = 0.02) -> List[float]:
    """Biases b_k for which a scalar sigmoid router stops with the target mass.

    The stop probability at junction k, given that the token reached it, is
    c_k = mass_k / (1 - sum_{j<k} mass_j).  The router input is an RMS-
    normalised state (unit RMS) and the router weight is N(0, weight_std^2),
    so the router logit's token-to-token spread is about
    N(0, weight_std^2 * d_model).  b_k solves E[sigmoid(b_k + eps)] = c_k,
    the expectation by 64-point Gauss-Hermite quadrature, by bisection.
    """
    s = weight_std * np.sqrt(d_model)
    x, w = np.polynomial.hermite_e.hermegauss(64)
    w = w / w.sum()
    out = []
    remaining = 1.0
    for m in list(mass)[:-1]:
        c = m / remaining
        remaining -= m
        lo, hi = -30.0, 30.0
        for _ in range(200):
            mid = 0.5 * (lo + hi)
            e = float(np.sum(w / (1.0 + np.exp(-(mid + s * x)))))
            if e < c:
                lo = mid
            else:
                hi = mid
        out.append(0.5 * (lo + hi))
    return out


# --------------------------------------------------------------------------
# weights
# --------------------------------------------------------------------------

def _tensor_specs(cfg: ModelConfig):
    """(key path, shape, kind) in manifest order; kind in {normal, gain}."""
    d, hq, f, v = cfg.d_model, cfg.n_heads * cfg.head_dim, cfg.d_ff, cfg.vocab
    specs = [(("tok_emb",), (v, d), "normal")]
    for i in range(cfg.n_layers):
        specs += [
            (("layers", i, "attn_norm"), (d,), "gain"),
            (("layers", i, "wq"), (hq, d), "normal"),
            (("layers", i, "wk"), (hq, d), "normal"),
            (("layers", i, "wv"), (hq, d), "normal"),
            (("layers", i, "wo"), (d, hq), "normal"),
            (("layers", i, "mlp_norm"), (d,), "gain"),
            (("layers", i, "wg"), (f, d), "normal"),
            (("layers", i, "wu"), (f, d), "normal"),
            (("layers", i, "wd"), (d, f), "normal"),
        ]
    for k in range(cfg.n_exits):
        specs += [
            (("exits", k, "norm"), (d,), "gain"),
            (("exits", k, "head"), (v, d), "normal"),
        ]
        if k < cfg.n_exits - 1:
            specs.append((("exits", k, "router_w"), (d,), "normal"))
    return specs


def make_weights(cfg: ModelConfig, seed: int = 0, random_gains: bool = False,
                 router_bias: Optional[Sequence[float]] = None,
                 threads: Optional[int] = None) -> dict:
    """Draw the model's weights.

    Returns {"dtype", "tok_emb", "layers": [dict], "exits": [dict]}; tensors
    are float32 (F32 configs) or bf16 bits as uint16 (BF16 configs).  Each
    exit dict has "norm", "head", and for k < N_V "router_w" and the float
    "router_b"; with cfg.router_hidden = r > 0 also the router MLP's
    "router_w1" [r, d] (model dtype), "router_b1" [r] and "router_w2" [r]
    (float32); with cfg.adapter_hidden = a > 0 also the exit adapter's
    "adapter_w1" [a, d] and "adapter_w2" [d, a] (model dtype), and the exits
    then share the last exit's head and norm.
    """
    specs = _tensor_specs(cfg)

    def draw(i):
        path, shape, kind = specs[i]
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(i,))))
        if kind == "gain":
            if random_gains:
                a = rng.uniform(0.5, 1.5, size=shape).astype(np.float32)
            else:
                a = np.ones(shape, dtype=np.float32)
        else:
            a = rng.standard_normal(size=shape, dtype=np.float32)
            a *= np.float32(0.02)
        if cfg.dtype == BF16:
            a = f32_to_bf16_bits(a)
        return path, a

    nthreads = threads or min(16, os.cpu_count() or 1)
    with _fut.ThreadPoolExecutor(nthreads) as ex:
        results = list(ex.map(draw, range(len(specs))))

    w = {"dtype": cfg.dtype, "layers": [dict() for _ in range(cfg.n_layers)],
         "exits": [dict() for _ in range(cfg.n_exits)]}
    for path, a in results:
        if path[0] == "tok_emb":
            w["tok_emb"] = a
        else:
            w[path[0]][path[1]][path[2]] = a

    if router_bias is None:
        if cfg.vocab <= 4096:  # tiny configuration: U(-1, 1) from the same seed
            rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(len(specs),))))
            router_bias = rng.uniform(-1.0, 1.0, size=cfg.n_exits - 1).tolist()
        else:
            router_bias = calibrate_router_biases(cfg.d_model, TARGET_EXIT_MASS[:cfg.n_exits]
                                                  if cfg.n_exits == 4 else
                                                  [1.0 / cfg.n_exits] * cfg.n_exits)
    for k in range(cfg.n_exits - 1):
        w["exits"][k]["router_b"] = float(np.float32(router_bias[k]))
    if cfg.router_hidden:
        # router MLP z = v . silu(U n + c) + b: U ~ N(0, 1/d) (model dtype),
        # c ~ N(0, 0.1^2), v ~ N(0, 1/r) (float32); streams after the manifest's
        r, d = cfg.router_hidden, cfg.d_model
        for k in range(cfg.n_exits - 1):
            rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(len(specs) + 1 + k,))))
            U = rng.standard_normal(size=(r, d), dtype=np.float32) * np.float32(1.0 / np.sqrt(d))
            w["exits"][k]["router_w1"] = f32_to_bf16_bits(U) if cfg.dtype == BF16 else U
            w["exits"][k]["router_b1"] = (rng.standard_normal(size=r, dtype=np.float32) * np.float32(0.1))
            w["exits"][k]["router_w2"] = (rng.standard_normal(size=r, dtype=np.float32) *
                                          np.float32(1.0 / np.sqrt(r)))
    if cfg.adapter_hidden:
        # exit adapters m = h + W2 silu(W1 n_k): W1 ~ N(0, 1/d), W2 ~ N(0, 0.02^2)
        # (model dtype); streams after the router MLP's
        a, d = cfg.adapter_hidden, cfg.d_model
        for k in range(cfg.n_exits - 1):
            rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(len(specs) + 101 + k,))))
            W1 = rng.standard_normal(size=(a, d), dtype=np.float32) * np.float32(1.0 / np.sqrt(d))
            W2 = rng.standard_normal(size=(d, a), dtype=np.float32) * np.float32(0.02)
            w["exits"][k]["adapter_w1"] = f32_to_bf16_bits(W1) if cfg.dtype == BF16 else W1
            w["exits"][k]["adapter_w2"] = f32_to_bf16_bits(W2) if cfg.dtype == BF16 else W2
    return w


# --------------------------------------------------------------------------
# prompts
# --------------------------------------------------------------------------

def zipf_ids(n: int, vocab: int, rng: np.random.Generator, s: float = 1.1) -> np.ndarray:
    """Truncated Zipf(s) ranks 1..vocab by inverse CDF; returns id = rank - 1."""
    ranks = np.arange(1, vocab + 1, dtype=np.float64)
    p = ranks ** (-s)
    cdf = np.cumsum(p)
    cdf /= cdf[-1]
    u = rng.random(n)
    ids = np.searchsorted(cdf, u, side="right")
    return np.minimum(ids, vocab - 1).astype(np.int32)


def make_prompt_lengths(wl: Workload, seed: int = 2) -> np.ndarray:
    if wl.prompt_len_lo == wl.prompt_len:
        return np.full(wl.batch, wl.prompt_len, dtype=np.int32)
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(wl.prompt_len_lo, wl.prompt_len + 1, size=wl.batch).astype(np.int32)


def make_prompts(wl: Workload, seed: int = 1, lengths: Optional[np.ndarray] = None) -> List[np.ndarray]:
    """One int32 id array per sequence (lengths from :func:`make_prompt_lengths`)."""
    if lengths is None:
        lengths = make_prompt_lengths(wl)
    rng = np.random.Generator(np.random.PCG64(seed))
    out = []
    for n in lengths:
        if wl.zipf:
            out.append(zipf_ids(int(n), wl.model.vocab, rng))
        else:
            out.append(rng.integers(0, wl.model.vocab, size=int(n)).astype(np.int32))
    return out


def scaled(wl: Workload, **changes) -> Workload:
    """A copy of a workload with some fields replaced (smaller test cases)."""
    return dataclasses.replace(wl, **changes)
