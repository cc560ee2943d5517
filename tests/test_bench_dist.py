"""Host logic of the multi-GPU benchmark on CPU: two gloo ranks.  Every rank
decodes its own independent batch (weak scaling, no data-path collective);
the reported time is the maximum over ranks."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    r, w = bench.dist_init("gloo")
    assert (r, w) == (rank, world)
    bench.barrier()
    m = bench.max_over_ranks(10.0 + 5 * rank)
    seeds = bench.rank_seeds(rank)
    wl = W.WORKLOADS["X64"]
    lens = W.make_prompt_lengths(wl, seed=seeds[1])
    out[rank] = (m, seeds, int(lens.sum()))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_distinct_inputs():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 15.0
    assert out[0][1] != out[1][1]
    assert out[0][2] != out[1][2]


def test_single_rank_needs_no_process_group():
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert bench.rank_env() == (0, 1, 0)
    assert bench.max_over_ranks(3.5) == 3.5


def test_bench_rejects_short_warmup():
    import pytest
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "1"])


def _reference_line(workload):
    import contextlib
    import io
    import json
    import bench
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.main(["--impl", "reference", "--workload", workload, "--steps", "1", "--warmup", "3"])
    lines = [l for l in buf.getvalue().splitlines() if l.startswith("{")]
    assert len(lines) == 1
    return json.loads(lines[0])


@pytest.mark.parametrize("workload,metric", [("T", "METRIC"), ("XS", "SCORE_METRIC")])
def test_reference_arm_prints_the_contract_line(workload, metric):
    """The reference arm (the oracle on the host cores) prints one JSON line
    with the base contract's keys, its cpu_baseline and an e2e of zero bytes."""
    d = _reference_line(workload)
    assert d["impl"] == "reference" and d["metric"] == getattr(bench, metric)
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    for k in ("n_gpus", "steps", "warmup", "ms_per_step", "scaling", "vs_baseline", "dtype", "data", "config"):
        assert k in d
    # the config names the workload, without model keys
    assert d["config"]["workload"] and "model" not in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_cpu_baseline_reports_all_threads_and_one_thread():
    """The CPU baseline times the oracle on a bounded sample with the host's
    BLAS threads and again on one thread."""
    wl = W.WORKLOADS["T"]
    lens = W.make_prompt_lengths(wl)
    prompts = W.make_prompts(wl, lengths=lens)
    cb = bench.cpu_baseline(wl, lens=lens, prompts=prompts, xseed=7, n_steps=2)
    assert cb["kind"] == "oracle" and cb["unit"] == "tokens/s" and cb["cores"] >= 1
    assert cb["value"] > 0 and cb["value_1_thread"] > 0 and "sample" in cb
    # the sample is a whole prompt of the workload, not a truncated one
    assert f"({len(prompts[int(np.argmin(lens))])}-token prompt" in cb["sample"]


def test_sub_line_keeps_only_measurement_keys():
    d = {"metric": "m", "value": 1.0, "unit": "tokens/s", "n_gpus": 1, "roofline": {"frac": 0.5},
         "e2e": {"value": 0.5}, "config": {"workload": "w"}, "vs_baseline": None}
    sub = bench.sub_line(d, "other")
    assert sub["metric"] == "other" and sub["value"] == 1.0 and sub["roofline"] == {"frac": 0.5}
    assert "n_gpus" not in sub and "vs_baseline" not in sub
