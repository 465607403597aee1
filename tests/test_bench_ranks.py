"""The multi-rank host logic of bench.py on CPU: two gloo ranks (one process
per GPU on a real run) agree on the slowest rank's time, the whole-job
throughput counts both ranks' work, and the config describes the replicas.
No GPU and no collective on the data path are involved."""
import os

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.rank_barrier(world)
        mine = 10.0 + 5.0 * rank                     # per-rank duration of the timed region (ms)
        t = bench.rank_max(mine, world)
        value = bench.whole_job_tflops(2.0e12, 4, world, t)
        cfg = bench.workload_config(4096, 3072, 12288, world)
        out[rank] = (t, value, cfg["global_batch_tokens"], cfg["parallelism"])
        bench.rank_barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_max_and_count_all_work():
    world, port = 2, 29517
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1]
    t, value, tokens, par = res[0]
    assert t == 15.0                                  # the slower rank's time
    assert value == pytest.approx(2 * 2.0e12 * 4 / 15e-3 / 1e12)
    assert tokens == 2 * 4096 and par == "replicas x2"


def test_single_rank_needs_no_process_group():
    assert bench.rank_max(3.0, 1) == 3.0
    bench.rank_barrier(1)
    assert bench.whole_job_tflops(1e12, 1, 1, 1.0) == pytest.approx(1000.0)
