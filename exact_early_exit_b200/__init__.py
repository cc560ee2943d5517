"""Python binding of libnvium, the B200 mixture-of-exits decode library.

Argument marshalling only: every step of the path runs in the CUDA kernels of
``libnvium.so`` (built in-tree by :mod:`exact_early_exit_b200.build`).  The
binding raises if the library is missing; there is no other implementation
behind it.  Buffers may be torch tensors (device or host) or numpy arrays
(host); the library copies through unified addressing.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# NVIUM_LIB points the binding at another build of the library (the same ABI)
LIB_PATH = os.environ.get("NVIUM_LIB") or os.path.join(_HERE, "libnvium.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "nvium.h")

NV_OK = 0
NV_ERR_INVALID_ARG = -1
NV_ERR_OOM = -2
NV_ERR_CUDA = -3
NV_ERR_CAPACITY = -4
NV_ERR_TIMEOUT = -5
NV_ERR_STATE = -6
NV_ERR_UNSUPPORTED = -7

NV_F32 = 0
NV_BF16 = 1
NV_ROUTER_NORMAL = 0
NV_ROUTER_FORCE_LAST = 1
NV_MAX_EXITS = 8
NV_PHILOX_NOALLOC_MAX = 32768

CTR = dict(steps=0, rows=1, layers_run=2, weight_bytes=3, kv_read_bytes=4, kv_write_bytes=5, head_bytes=6,
           forced=7, launches=8, exit0=16)
NV_CTR_COUNT = 24
KERNEL_KINDS = ("plan_norm", "gemm", "epilogue", "attention", "norm", "junction", "head", "step")


class KernelStat(ctypes.Structure):
    _fields_ = [("ms", ctypes.c_double), ("launches", ctypes.c_int64), ("bytes", ctypes.c_int64),
                ("flops", ctypes.c_int64), ("kernels", ctypes.c_int64)]


class NviumError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"libnvium status {status}: {msg}")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("d_model", ctypes.c_int), ("n_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("d_ff", ctypes.c_int), ("vocab", ctypes.c_int),
                ("n_exits", ctypes.c_int), ("exit_layers", ctypes.c_int * NV_MAX_EXITS), ("dtype", ctypes.c_int),
                ("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_float), ("max_batch", ctypes.c_int),
                ("max_seq", ctypes.c_int), ("page_size", ctypes.c_int), ("max_pending", ctypes.c_int),
                ("router_mode", ctypes.c_int), ("router_hidden", ctypes.c_int), ("adapter_hidden", ctypes.c_int)]


class LayerWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("attn_norm", "wq", "wk", "wv", "wo", "mlp_norm", "wg", "wu", "wd")]


class ExitWeights(ctypes.Structure):
    _fields_ = [("norm", ctypes.c_void_p), ("head", ctypes.c_void_p), ("router_w", ctypes.c_void_p),
                ("router_b", ctypes.c_float), ("router_w1", ctypes.c_void_p), ("router_b1", ctypes.c_void_p),
                ("router_w2", ctypes.c_void_p), ("adapter_w1", ctypes.c_void_p), ("adapter_w2", ctypes.c_void_p)]


class Weights(ctypes.Structure):
    _fields_ = [("tok_emb", ctypes.c_void_p), ("layers", ctypes.POINTER(LayerWeights)),
                ("exits", ctypes.POINTER(ExitWeights))]


_lib = None

# (name, restype, argtypes) of every exported entry point
_P = ctypes.c_void_p
_I = ctypes.c_int
_SIGS = [
    ("nv_create", _I, [ctypes.POINTER(Config), ctypes.POINTER(Weights), ctypes.POINTER(_P)]),
    ("nv_destroy", _I, [_P]),
    ("nv_score_mixture", _I, [_P, _P, _I, _I, _P, _P, _P]),
    ("nv_state_create", _I, [_P, _I, ctypes.POINTER(_P)]),
    ("nv_state_destroy", _I, [_P]),
    ("nv_prefill", _I, [_P, _P, _P, _P]),
    ("nv_rewind", _I, [_P, _P]),
    ("nv_decode_step", _I, [_P, ctypes.c_uint64, _P, _P, _P, _P]),
    ("nv_flush_deferred", _I, [_P, _P]),
    ("nv_read_kv", _I, [_P, _I, _I, _P, _P, ctypes.POINTER(_I), _P]),
    ("nv_read_router_probs", _I, [_P, _P, _P]),
    ("nv_read_counters", _I, [_P, _P, _I]),
    ("nv_reset_counters", _I, [_P]),
    ("nv_sync_status", _I, [_P]),
    ("nv_philox4x32_10", _I, [ctypes.c_uint64, _P, _I, _P, _P]),
    ("nv_decode_step_profiled", _I, [_P, ctypes.c_uint64, _P, _P, _P, _P]),
    ("nv_philox4x32_10_noalloc", _I, [ctypes.c_uint64, _P, _I, _P, _P]),
    ("nv_selftest_bounded_wait", _I, [_I, _P, _P]),
    ("nv_score_mixture_profiled", _I, [_P, _P, _I, _I, _P, _P, _P, _P]),
    ("nv_score_mixture_ex", _I, [_P, _P, _I, _I, _P, _P, _P, _P, _P]),
    ("nv_last_error", ctypes.c_char_p, []),
]


def lib():
    """Load libnvium.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m exact_early_exit_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, res, args in _SIGS:
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int):
    if status != NV_OK:
        raise NviumError(status, lib().nv_last_error().decode(errors="replace"))


def _ptr(x) -> Optional[int]:
    """Raw address of a torch tensor or numpy array (None passes NULL)."""
    if x is None:
        return None
    if hasattr(x, "data_ptr"):
        if not x.is_contiguous():
            raise ValueError("buffers must be contiguous")
        return x.data_ptr()
    if isinstance(x, np.ndarray):
        if not x.flags["C_CONTIGUOUS"]:
            raise ValueError("buffers must be contiguous")
        return x.ctypes.data
    raise TypeError(f"unsupported buffer type {type(x)}")


def _stream(stream) -> Optional[int]:
    if stream is not None:
        return int(stream)
    try:
        import torch
        if torch.cuda.is_available() and torch.cuda.is_initialized():
            return torch.cuda.current_stream().cuda_stream
    except Exception:  # pragma: no cover
        pass
    return None


def make_config(model_cfg, max_batch: int, max_seq: int, page_size: int = 64, max_pending: int = 256,
                router_mode: int = NV_ROUTER_NORMAL) -> Config:
    """nv_config from any object with the model fields (n_layers, d_model,
    n_heads, head_dim, d_ff, vocab, exit_layers, dtype, rms_eps, rope_theta)."""
    c = Config()
    c.n_layers = model_cfg.n_layers
    c.d_model = model_cfg.d_model
    c.n_heads = model_cfg.n_heads
    c.head_dim = model_cfg.head_dim
    c.d_ff = model_cfg.d_ff
    c.vocab = model_cfg.vocab
    c.n_exits = len(model_cfg.exit_layers)
    for i, l in enumerate(model_cfg.exit_layers):
        c.exit_layers[i] = int(l)
    c.dtype = int(model_cfg.dtype)
    c.rms_eps = float(getattr(model_cfg, "rms_eps", 1e-5))
    c.rope_theta = float(getattr(model_cfg, "rope_theta", 10000.0))
    c.max_batch = max_batch
    c.max_seq = max_seq
    c.page_size = page_size
    c.max_pending = max_pending
    c.router_mode = router_mode
    c.router_hidden = int(getattr(model_cfg, "router_hidden", 0))
    c.adapter_hidden = int(getattr(model_cfg, "adapter_hidden", 0))
    return c


class Model:
    """nv_create / nv_destroy, nv_score_mixture.

    ``weights``: {"tok_emb", "layers": [{attn_norm, wq, wk, wv, wo, mlp_norm,
    wg, wu, wd}], "exits": [{norm, head, router_w?, router_b?}]} with tensors
    as numpy arrays or torch tensors holding the config dtype's bits (bf16 may
    be given as uint16 bit patterns).
    """

    def __init__(self, model_cfg, weights: dict, max_batch: int, max_seq: int, page_size: int = 64,
                 max_pending: int = 256, router_mode: int = NV_ROUTER_NORMAL):
        self.cfg = make_config(model_cfg, max_batch, max_seq, page_size, max_pending, router_mode)
        self.model_cfg = model_cfg
        keep = []

        def p(a):
            if not hasattr(a, "data_ptr"):
                a = np.ascontiguousarray(a)
            keep.append(a)
            return _ptr(a)

        n_layers, n_exits = self.cfg.n_layers, self.cfg.n_exits
        lw = (LayerWeights * n_layers)()
        for i, L in enumerate(weights["layers"]):
            for f in ("attn_norm", "wq", "wk", "wv", "wo", "mlp_norm", "wg", "wu", "wd"):
                setattr(lw[i], f, p(L[f]))
        ew = (ExitWeights * n_exits)()
        for k, E in enumerate(weights["exits"]):
            ew[k].norm = p(E["norm"])
            ew[k].head = p(E["head"]) if "head" in E else None
            ew[k].router_w = p(E["router_w"]) if "router_w" in E else None
            ew[k].router_b = float(E.get("router_b", 0.0))
            for f in ("router_w1", "router_b1", "router_w2", "adapter_w1", "adapter_w2"):
                if f in E:
                    setattr(ew[k], f, p(E[f]))
        w = Weights(p(weights["tok_emb"]), lw, ew)
        h = ctypes.c_void_p()
        _check(lib().nv_create(ctypes.byref(self.cfg), ctypes.byref(w), ctypes.byref(h)))
        self.handle = h
        del keep

    def score_mixture(self, tokens, logp_out, mean_nll_out=None, stream=None):
        """tokens [B, S] int32 -> logp_out [B, S-1] float32, mean_nll_out [1]."""
        B, S = tokens.shape
        _check(lib().nv_score_mixture(self.handle, _ptr(tokens), B, S, _ptr(logp_out), _ptr(mean_nll_out),
                                      _stream(stream)))

    def score_mixture_ex(self, tokens, logp_out, mean_nll_out=None, depth_out=None, mean_depth_out=None,
                         stream=None):
        """score_mixture plus the expected normalised layer depth of every
        position (depth_out [B, S-1]) and its mean (mean_depth_out [1])."""
        B, S = tokens.shape
        _check(lib().nv_score_mixture_ex(self.handle, _ptr(tokens), B, S, _ptr(logp_out), _ptr(mean_nll_out),
                                         _ptr(depth_out), _ptr(mean_depth_out), _stream(stream)))

    def score_mixture_profiled(self, tokens, logp_out, mean_nll_out=None, stats=None, stream=None):
        """score_mixture with per-kernel CUDA-event timing (KernelStat array)."""
        if stats is None:
            stats = (KernelStat * len(KERNEL_KINDS))()
        B, S = tokens.shape
        _check(lib().nv_score_mixture_profiled(self.handle, _ptr(tokens), B, S, _ptr(logp_out), _ptr(mean_nll_out),
                                               ctypes.cast(stats, ctypes.c_void_p), _stream(stream)))
        return stats

    def close(self):
        if getattr(self, "handle", None):
            lib().nv_destroy(self.handle)
            self.handle = None

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass


class State:
    """nv_state_create and the decode-state calls."""

    def __init__(self, model: Model, batch: int):
        self.model = model
        self.B = batch
        h = ctypes.c_void_p()
        _check(lib().nv_state_create(model.handle, batch, ctypes.byref(h)))
        self.handle = h

    def prefill(self, tokens, lens: Sequence[int], stream=None):
        lens = np.ascontiguousarray(np.asarray(lens, dtype=np.int32))
        _check(lib().nv_prefill(self.handle, _ptr(tokens), _ptr(lens), _stream(stream)))

    def rewind(self, stream=None):
        _check(lib().nv_rewind(self.handle, _stream(stream)))

    def decode_step(self, seed: int, tokens_out, exits_out, logp_out=None, stream=None):
        _check(lib().nv_decode_step(self.handle, ctypes.c_uint64(seed), _ptr(tokens_out), _ptr(exits_out),
                                    _ptr(logp_out), _stream(stream)))

    def decode_step_profiled(self, seed: int, tokens_out, exits_out, stats=None, stream=None):
        """One decode step with per-kernel CUDA-event timing; accumulates into
        and returns `stats` (a KernelStat array indexed like KERNEL_KINDS)."""
        if stats is None:
            stats = (KernelStat * len(KERNEL_KINDS))()
        _check(lib().nv_decode_step_profiled(self.handle, ctypes.c_uint64(seed), _ptr(tokens_out), _ptr(exits_out),
                                             ctypes.cast(stats, ctypes.c_void_p), _stream(stream)))
        return stats

    def flush(self, stream=None):
        _check(lib().nv_flush_deferred(self.handle, _stream(stream)))

    def read_kv(self, b: int, layer: int, max_len: int):
        """(K, V, len): numpy arrays [len, H, hd] of the config dtype's bits."""
        c = self.model.cfg
        dt = np.uint16 if c.dtype == NV_BF16 else np.float32
        K = np.zeros((max_len, c.n_heads, c.head_dim), dtype=dt)
        V = np.zeros_like(K)
        n = ctypes.c_int()
        _check(lib().nv_read_kv(self.handle, b, layer, _ptr(K), _ptr(V), ctypes.byref(n), _stream(None)))
        return K[: n.value], V[: n.value], n.value

    def router_probs(self) -> np.ndarray:
        """[n_exits - 1, B] float32: the w_k each sequence's token was compared
        against at junction k in the last decode step (NaN where the token
        stopped earlier)."""
        c = self.model.cfg
        out = np.zeros((c.n_exits - 1, self.B), dtype=np.float32)
        if out.size:
            _check(lib().nv_read_router_probs(self.handle, _ptr(out), _stream(None)))
        return out

    def counters(self) -> np.ndarray:
        out = np.zeros(NV_CTR_COUNT, dtype=np.int64)
        _check(lib().nv_read_counters(self.handle, _ptr(out), NV_CTR_COUNT))
        return out

    def reset_counters(self):
        _check(lib().nv_reset_counters(self.handle))

    def sync_status(self):
        _check(lib().nv_sync_status(self.handle))

    def close(self):
        if getattr(self, "handle", None):
            lib().nv_state_destroy(self.handle)
            self.handle = None

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass


def philox4x32_10(seed: int, counters: np.ndarray) -> np.ndarray:
    """Device Philox4x32-10 on host counters [n, 4] uint32 (test hook)."""
    ctr = np.ascontiguousarray(counters, dtype=np.uint32).reshape(-1, 4)
    out = np.zeros_like(ctr)
    _check(lib().nv_philox4x32_10(ctypes.c_uint64(seed), _ptr(ctr), ctr.shape[0], _ptr(out), None))
    return out


def selftest_bounded_wait(limit_us: int) -> bool:
    """Run the bounded-wait self-test (a wait that nothing completes, given
    up after limit_us); True when the wait gave up as it should."""
    out = np.zeros(1, np.int32)
    _check(lib().nv_selftest_bounded_wait(int(limit_us), _ptr(out), None))
    return bool(out[0])


def philox4x32_10_noalloc(seed: int, counters: np.ndarray) -> np.ndarray:
    """nv_philox4x32_10 without any device allocation (staging through the
    library's fixed array; at most NV_PHILOX_NOALLOC_MAX counters)."""
    ctr = np.ascontiguousarray(counters, dtype=np.uint32).reshape(-1, 4)
    out = np.zeros_like(ctr)
    _check(lib().nv_philox4x32_10_noalloc(ctypes.c_uint64(seed), _ptr(ctr), ctr.shape[0], _ptr(out), None))
    return out
