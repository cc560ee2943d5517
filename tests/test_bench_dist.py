"""Host logic of the multi-GPU benchmark on CPU: two gloo ranks.  Every rank
decodes its own independent batch (weak scaling, no data-path collective);
the reported time is the maximum over ranks."""
import os
import socket

import numpy as np
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
