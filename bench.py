#!/usr/bin/env python
"""Decode throughput of the N-vium 1.5B 4-exit model on B200.

One bench step = one generation pass of the whole hot path on one batch:
rewind to the post-prefill state, `decode_steps` decode steps for every
sequence (mixture-of-exits routing, exact sampling, deferred upper layers
batched with later tokens), and the final flush of the deferred rows.
`value` = decoded tokens / time with inputs resident in HBM; `e2e` = the same
pass through the C ABI from pinned host memory (prompt upload and prefill
inside, sampled tokens and exits copied back to the host every step).

  python bench.py [--workload X64|X1|S|T] [--steps K] [--warmup W] [--gpus N]
  python bench.py --impl reference ...     # the CPU oracle on the same config

Multi-GPU (torchrun): every rank decodes its own batch of independent
sequences (weak scaling, no data-path collective); time = max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "decode tokens/s, 1.5B 4-exit model, B=1/B=64 on 1 B200; % of HBM roofline"
SCORE_METRIC = "mixture scoring tokens/s, 1.5B 4-exit model, 16 x 2048; GEMMs as % of bf16 tensor peak"
FALLBACK_HBM_GBS = 6650.0
PHILOX_SEED = 1234


# ---------------------------------------------------------------------------
# ranks
# ---------------------------------------------------------------------------
def rank_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def dist_init(backend: str):
    import torch.distributed as dist
    rank, world, _ = rank_env()
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return rank, world


def barrier():
    import torch.distributed as dist
    if dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not dist.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seeds(rank: int):
    """Inputs of rank r: prompt ids seed, prompt length seed, Philox seed."""
    return 1 + 1000 * rank, 2 + 1000 * rank, PHILOX_SEED + 7919 * rank


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
REASON_FIELDS = ["clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
                 "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]


class ClockSampler:
    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ",".join(["clocks.sm", "clocks.max.sm", "power.draw"] + REASON_FIELDS)
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(5)
            except Exception:
                self.proc.kill()
            self.out.close()

    def summary(self):
        if not self.proc or not self.path:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[0]))
                smax.append(float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [x for x in sm if x > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# roofline inputs
# ---------------------------------------------------------------------------
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


KERNEL_SOURCES = {
    "gemm": "exact_early_exit_b200/csrc/gemm_tc.cu",
    "attention": "exact_early_exit_b200/csrc/attn_mma.cu",
    "head": "exact_early_exit_b200/csrc/kernels.cu",
    "epilogue": "exact_early_exit_b200/csrc/kernels.cu",
    "plan_norm": "exact_early_exit_b200/csrc/kernels.cu",
}


def source_hash(kind: str) -> str:
    p = os.path.join(ROOT, KERNEL_SOURCES.get(kind, "exact_early_exit_b200/csrc/kernels.cu"))
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]


def ncu_traffic(kind: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary of this kernel on this
    workload, if it was taken from the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", f"{kind}_{workload}.md")
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    h = re.search(r"source_sha256_16:\s*([0-9a-f]+)", txt)
    t = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    if not h or not t or h.group(1) != source_hash(kind):
        return None
    return float(t.group(1))


def workload_for(args):
    """The named workload, or a shortened copy for profiling runs."""
    import dataclasses
    wl = W.WORKLOADS[args.workload]
    if args.layers:
        L = args.layers
        ne = wl.model.n_exits
        exits = tuple(max(1, round(L * (k + 1) / ne)) for k in range(ne))
        model = dataclasses.replace(wl.model, name=f"{wl.model.name}-{L}layers", n_layers=L, exit_layers=exits)
        wl = dataclasses.replace(wl, model=model, name=f"{wl.name}-{L}layers")
    if args.decode_steps:
        wl = dataclasses.replace(wl, steps=args.decode_steps, name=f"{wl.name}-{args.decode_steps}steps")
    return wl


# ---------------------------------------------------------------------------
# the CUDA arm
# ---------------------------------------------------------------------------
def measure_decode(args, wl, n_steps, n_warmup, dev, rank, world, weights=None, want_cpu=False):
    """Decode passes of workload `wl` (the bench step: rewind + decode_steps
    decode steps + flush), e2e through the C ABI from host buffers, the same
    kernels forced to full depth, and the per-kernel profiled pass; returns
    the measurement dict (the JSON line's keys)."""
    import torch

    import exact_early_exit_b200 as nv

    cfg = wl.model
    pseed, lseed, xseed = rank_seeds(rank)
    lens = W.make_prompt_lengths(wl, seed=lseed)
    prompts = W.make_prompts(wl, seed=pseed, lengths=lens)
    B, steps = wl.batch, wl.steps
    if weights is None:
        weights = W.make_weights(cfg, seed=0)
    max_seq = int(lens.max()) + steps + 64
    model = nv.Model(cfg, weights, max_batch=B, max_seq=max_seq, max_pending=256)
    st = nv.State(model, B)
    tok_host = torch.from_numpy(np.concatenate(prompts).astype(np.int32)).pin_memory()
    stream = torch.cuda.current_stream(dev)
    st.prefill(tok_host, lens)

    tok_d = torch.zeros(B, dtype=torch.int32, device=dev)
    ex_d = torch.zeros(B, dtype=torch.int32, device=dev)

    def gen_pass(seed):
        st.rewind()
        for s in range(steps):
            st.decode_step(seed + s, tok_d, ex_d)
        st.flush()

    for i in range(n_warmup):
        gen_pass(xseed + 100000 * (i + 1))
    torch.cuda.synchronize()
    st.sync_status()
    st.reset_counters()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(n_steps):
            gen_pass(xseed)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms_total = e0.elapsed_time(e1)
    st.sync_status()
    ctr = st.counters()
    ms_max = max_over_ranks(ms_total, dev)
    ms_per_step = ms_max / n_steps
    tokens_per_step = B * steps
    value = tokens_per_step * world * n_steps / (ms_max / 1e3)
    launches = int(ctr[nv.CTR["launches"]])

    # algorithmic bytes of one pass (weights per layer run, K/V attended and
    # written, exit heads), from the device counters of the timed passes
    pass_bytes = float(ctr[nv.CTR["weight_bytes"]] + ctr[nv.CTR["kv_read_bytes"]] +
                       ctr[nv.CTR["kv_write_bytes"]] + ctr[nv.CTR["head_bytes"]]) / n_steps
    exits = ctr[nv.CTR["exit0"]:nv.CTR["exit0"] + cfg.n_exits].astype(float)
    exit_mass = (exits / max(exits.sum(), 1)).round(4).tolist()

    # e2e through the C ABI from pinned host memory
    tok_h = torch.zeros(B, dtype=torch.int32).pin_memory()
    ex_h = torch.zeros(B, dtype=torch.int32).pin_memory()
    torch.cuda.synchronize()
    barrier()
    e2 = torch.cuda.Event(enable_timing=True)
    e3 = torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for i in range(n_steps):
        st.prefill(tok_host, lens)
        for s in range(steps):
            st.decode_step(xseed + s, tok_h, ex_h)
        st.flush()
    e3.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e2.elapsed_time(e3), dev)
    e2e_value = tokens_per_step * world * n_steps / (e2e_ms / 1e3)

    # prefill and the final flush on their own (decode tokens/s excludes the
    # prefill; the flush is owed work and sits inside every timed pass)
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    ea.record(stream)
    st.prefill(tok_host, lens)
    eb.record(stream)
    torch.cuda.synchronize()
    prefill_ms = ea.elapsed_time(eb)
    for s in range(steps):
        st.decode_step(xseed + s, tok_d, ex_d)
    ea.record(stream)
    st.flush()
    eb.record(stream)
    torch.cuda.synchronize()
    flush_ms = ea.elapsed_time(eb)

    # the same kernels forced to full depth (every token leaves at the last
    # exit): the dense-decode comparison of the same workload
    fmodel = nv.Model(cfg, weights, max_batch=B, max_seq=max_seq, max_pending=256,
                      router_mode=nv.NV_ROUTER_FORCE_LAST)
    fst = nv.State(fmodel, B)
    fst.prefill(tok_host, lens)

    def full_pass(seed):
        fst.rewind()
        for s in range(steps):
            fst.decode_step(seed + s, tok_d, ex_d)
        fst.flush()

    for i in range(n_warmup):
        full_pass(xseed + 100000 * (i + 1))
    torch.cuda.synchronize()
    barrier()
    ea.record(stream)
    for i in range(n_steps):
        full_pass(xseed)
    eb.record(stream)
    torch.cuda.synchronize()
    barrier()
    full_ms = max_over_ranks(ea.elapsed_time(eb), dev) / n_steps
    fst.sync_status()
    fst.close()
    fmodel.close()
    full_value = tokens_per_step * world / (full_ms / 1e3)

    # per-kernel times: one profiled pass (each launch bracketed by events)
    stats = (nv.KernelStat * len(nv.KERNEL_KINDS))()
    st.rewind()
    for s in range(steps):
        st.decode_step_profiled(xseed + s, tok_d, ex_d, stats)
    kern = {k: dict(ms=stats[i].ms, launches=int(stats[i].launches), bytes=int(stats[i].bytes),
                    flops=int(stats[i].flops)) for i, k in enumerate(nv.KERNEL_KINDS)}
    total_k_ms = sum(v["ms"] for v in kern.values())
    dom = max(kern, key=lambda k: kern[k]["ms"])
    dk = kern[dom]
    per_launch_ms = dk["ms"] / max(dk["launches"], 1)
    per_launch_bytes = dk["bytes"] / max(dk["launches"], 1)
    achieved = per_launch_bytes / (per_launch_ms / 1e3) / 1e9
    peak, peak_src = measured_peaks()
    traffic = ncu_traffic(dom, wl.name)
    roofline = {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": traffic,
                "bytes_per_launch": round(per_launch_bytes), "ms_per_launch": round(per_launch_ms, 5),
                "peak_source": f"{peak_src} copy bandwidth",
                "kernel_share": {k: round(v["ms"] / total_k_ms, 4) for k, v in kern.items()},
                "step_algorithmic_GBps": round(pass_bytes / (ms_per_step / 1e3) / 1e9, 1),
                "step_frac": round(pass_bytes / (ms_per_step / 1e3) / 1e9 / peak, 4)}

    out = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": n_steps,
           "warmup": n_warmup, "ms_per_step": round(ms_per_step, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if cfg.dtype == W.BF16 else "f32",
           "data": "synthetic",
           "config": {"workload": wl.name, "global_batch": B * world,
                      "prompt_len": (f"U[{wl.prompt_len_lo},{wl.prompt_len}]" if wl.prompt_len_lo != wl.prompt_len
                                     else wl.prompt_len),
                      "decode_steps": steps, "parallelism": f"dp{world}" if world > 1 else "single",
                      "step": "rewind + decode_steps decode steps + flush of deferred rows",
                      "l2": "inputs larger than L2 (weights and KV streamed each step)"},
           "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s",
                   "h2d_bytes_per_step": int(tok_host.numel() * 4),
                   "d2h_bytes_per_step": int(steps * B * 8)},
           "gpu_launches": launches,
           "roofline": roofline,
           "realised_exit_mass": exit_mass,
           "full_depth": {"value": round(full_value, 1), "unit": "tokens/s", "ms_per_step": round(full_ms, 3),
                          "speedup": round(value / full_value, 3),
                          "what": "same workload and kernels, router forced to the last exit"},
           "prefill_ms": round(prefill_ms, 3),
           "flush_ms": round(flush_ms, 3)}
    if want_cpu:
        out["cpu_baseline"] = cpu_baseline(wl, lens=lens, prompts=prompts, xseed=xseed)
    out["clocks"] = clk.summary()
    st.close()
    model.close()
    return out


SUB_KEYS = ("value", "unit", "steps", "warmup", "ms_per_step", "config", "e2e", "gpu_launches", "roofline",
            "realised_exit_mass", "full_depth", "prefill_ms", "flush_ms", "mean_nll", "mean_expected_depth",
            "clocks")


def sub_line(d: dict, metric: str) -> dict:
    """A second workload's measurement nested inside the headline line."""
    out = {"metric": metric}
    out.update({k: d[k] for k in SUB_KEYS if k in d})
    return out


def run_ours(args):
    """The decode workload's JSON line; with the default workload (B=64) on
    one GPU it also carries the B=1 decode (`b1`) and the 16 x 2048 scoring
    (`scoring`) measurements, each with its own roofline and e2e."""
    import torch

    rank, world = dist_init("nccl")
    _, _, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = workload_for(args)
    weights = W.make_weights(wl.model, seed=0)
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    out = measure_decode(args, wl, args.steps, args.warmup, dev, rank, world, weights=weights, want_cpu=want_cpu)
    if args.workload == "X64" and not args.layers and not args.decode_steps and not args.headline_only:
        # the other two configurations of the metric, with fewer timed passes
        sub_steps = max(3, min(args.steps, 5))
        b1 = measure_decode(args, W.WORKLOADS["X1"], sub_steps, 3, dev, rank, world, weights=weights)
        out["b1"] = sub_line(b1, METRIC)
        del weights
        sc = measure_scoring(W.WORKLOADS["XS"], sub_steps, 3, dev, rank, world)
        out["scoring"] = sub_line(sc, SCORE_METRIC)
    if rank == 0:
        print(json.dumps(out))
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


def measured_tensor_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["bf16_tflops_sustained"]), "measured sustained"
    except Exception:
        return 1400.0, "fallback sustained"


def measure_scoring(wl, n_steps, n_warmup, dev, rank, world):
    """Mixture scoring of 16 x 2048 tokens (log pi_mix at every position and
    the mean NLL): one nv_score_mixture call per step; returns the
    measurement dict."""
    import torch

    import exact_early_exit_b200 as nv

    cfg = wl.model
    pseed, _, _ = rank_seeds(rank)
    toks = np.stack(W.make_prompts(wl, seed=pseed)).astype(np.int32)
    B, S = toks.shape
    weights = W.make_weights(cfg, seed=0)
    model = nv.Model(cfg, weights, max_batch=1, max_seq=S)
    del weights
    tok_d = torch.from_numpy(toks).to(dev)
    logp_d = torch.zeros((B, S - 1), dtype=torch.float32, device=dev)
    nll_d = torch.zeros(1, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(n_warmup):
        model.score_mixture(tok_d, logp_d, nll_d)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(n_steps):
            model.score_mixture(tok_d, logp_d, nll_d)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms = max_over_ranks(e0.elapsed_time(e1), dev) / n_steps
    tokens = B * (S - 1)
    value = tokens * world / (ms / 1e3)
    # e2e: host tokens in, host log-probs out
    tok_h = torch.from_numpy(toks).pin_memory()
    logp_h = torch.zeros((B, S - 1), dtype=torch.float32).pin_memory()
    nll_h = torch.zeros(1, dtype=torch.float32).pin_memory()
    torch.cuda.synchronize()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for _ in range(n_steps):
        model.score_mixture(tok_h, logp_h, nll_h)
    e3.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e2.elapsed_time(e3), dev) / n_steps
    # the compute-penalty forward on the same batch (untimed): mean expected
    # normalised layer depth
    depth_d = torch.zeros_like(logp_d)
    mdepth_d = torch.zeros(1, dtype=torch.float32, device=dev)
    model.score_mixture_ex(tok_d, logp_d, nll_d, depth_d, mdepth_d)
    torch.cuda.synchronize()
    mean_depth = float(mdepth_d.item())
    stats = model.score_mixture_profiled(tok_d, logp_d, nll_d)
    kern = {k: dict(ms=stats[i].ms, launches=int(stats[i].launches), kernels=int(stats[i].kernels),
                    flops=int(stats[i].flops))
            for i, k in enumerate(nv.KERNEL_KINDS)}
    total_k = sum(v["ms"] for v in kern.values())
    gemm_ms = kern["gemm"]["ms"] + kern["head"]["ms"]
    gemm_flops = kern["gemm"]["flops"] + kern["head"]["flops"]
    achieved = gemm_flops / (gemm_ms / 1e3) / 1e12
    peak, src = measured_tensor_peak()
    out = {"metric": SCORE_METRIC,
           "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": n_steps,
           "warmup": n_warmup, "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
           "config": {"workload": wl.name, "global_batch": B * world, "seq_len": S,
                      "parallelism": f"dp{world}" if world > 1 else "single",
                      "l2": "inputs larger than L2 (weights and activations streamed each step)"},
           "e2e": {"value": round(tokens * world / (e2e_ms / 1e3), 1), "unit": "tokens/s",
                   "h2d_bytes_per_step": int(toks.nbytes), "d2h_bytes_per_step": int(B * (S - 1) * 4 + 4)},
           "gpu_launches": sum(v["kernels"] for v in kern.values()) * n_steps,
           "roofline": {"bound": "tensor", "kernel": "gemm (layers + exit heads)", "achieved": round(achieved, 1),
                        "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                        "traffic": ncu_traffic("gemm", wl.name),
                        "peak_source": src, "kernel_share": {k: round(v["ms"] / total_k, 4) for k, v in kern.items()},
                        "gemm_tflop_per_step": round(gemm_flops / 1e12, 2)},
           "mean_nll": float(nll_d.item()),
           "mean_expected_depth": round(mean_depth, 5)}
    out["clocks"] = clk.summary()
    model.close()
    return out


def run_scoring(args):
    import torch

    rank, world = dist_init("nccl")
    _, _, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    out = measure_scoring(workload_for(args), args.steps, args.warmup, dev, rank, world)
    if rank == 0:
        print(json.dumps(out))
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# the CPU oracle: baseline sample and the reference arm
# ---------------------------------------------------------------------------
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_setup(wl, lens, prompts, max_new=64):
    """The oracle decoder on one sequence of the workload: the batch's
    shortest prompt (all of it), prefilled at full depth (untimed)."""
    from oracle import nvium_oracle as O
    weights = W.make_weights(wl.model, seed=0)
    om = O.OracleModel(wl.model, weights)
    b = int(np.argmin(lens))
    dec = O.OracleDecoder(om, [prompts[b]], max_new)
    dec.ids = [b]
    return dec, b


def cpu_baseline(wl, lens, prompts, xseed, n_steps=16):
    """The oracle on a bounded sample of the workload: one of its sequences
    (the shortest prompt, prefilled in full, untimed), the first `n_steps`
    decode steps of that sequence timed with the workload's Philox seeds;
    tokens/s of that sample (the oracle's per-token rate, extrapolated to the
    workload)."""
    dec, b = oracle_setup(wl, lens, prompts)
    t0 = time.perf_counter()
    for s in range(n_steps):
        dec.step(xseed + s)
    dt = time.perf_counter() - t0
    out = {"value": round(n_steps / dt, 4), "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
           "sample": f"sequence {b} of the workload ({len(prompts[b])}-token prompt prefilled untimed), its first "
                     f"{n_steps} decode steps timed (1 token each), float64 numpy; tokens/s extrapolated per token"}
    # the same sample on one host thread (the oracle's matrix products are the
    # only multi-threaded part)
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            t0 = time.perf_counter()
            dec.step(xseed + n_steps)
            out["value_1_thread"] = round(1.0 / (time.perf_counter() - t0), 4)
    except ImportError:
        pass
    return out


def run_reference_scoring(args, wl, world):
    """The oracle's mixture scoring on a bounded sample of the scoring
    workload: one sequence's first 65 tokens (64 scored positions) per step."""
    from oracle import nvium_oracle as O
    pseed, _, _ = rank_seeds(0)
    toks = np.stack(W.make_prompts(wl, seed=pseed)).astype(np.int32)[:1, :65]
    om = O.OracleModel(wl.model, W.make_weights(wl.model, seed=0))
    for _ in range(args.warmup):
        O.score_mixture(om, toks[:, :9])
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.score_mixture(om, toks)
    dt = time.perf_counter() - t0
    value = args.steps * (toks.shape[1] - 1) / dt
    sample = "sequence 0, first 65 tokens (64 scored positions) per step, float64 numpy oracle"
    out = {"metric": SCORE_METRIC, "impl": "reference", "value": round(value, 4), "unit": "tokens/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(dt / args.steps * 1e3, 1), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": wl.name, "global_batch": wl.batch, "seq_len": wl.prompt_len},
           "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out))


def run_reference(args):
    rank, world, _ = rank_env()
    if rank != 0:
        return
    wl = W.WORKLOADS[args.workload]
    if args.workload == "XS":
        run_reference_scoring(args, wl, world)
        return
    pseed, lseed, xseed = rank_seeds(0)
    lens = W.make_prompt_lengths(wl, seed=lseed)
    prompts = W.make_prompts(wl, seed=pseed, lengths=lens)
    dec, b = oracle_setup(wl, lens, prompts, max_new=args.warmup + args.steps + 1)
    # warm-up steps are the sequence's first decode steps; the timed steps follow them
    for i in range(args.warmup):
        dec.step(xseed + i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        dec.step(xseed + args.warmup + i)
    dt = time.perf_counter() - t0
    value = args.steps / dt
    cores = blas_threads()
    sample = (f"sequence {b} of the workload ({len(prompts[b])}-token prompt prefilled untimed); each step = 1 "
              f"decode step of that sequence (1 token), float64 numpy oracle; tokens/s extrapolated per token")
    out = {"metric": METRIC, "impl": "reference", "value": round(value, 4), "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 1),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "f64", "data": "synthetic",
           "config": {"workload": wl.name, "global_batch": wl.batch,
                      "decode_steps": wl.steps},
           "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out))


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["X64", "X1", "XS", "S", "T"], default="X64")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", action="store_true",
                    help="default workload: skip the nested B=1 and scoring measurements")
    ap.add_argument("--layers", type=int, default=0,
                    help="profiling only: the workload's model with this many layers (exits spread evenly)")
    ap.add_argument("--decode-steps", type=int, default=0, help="profiling only: decode steps per pass")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "XS":
        run_scoring(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
