"""Multi-rank host logic on CPU (gloo, world size 2): the path shards by
sequence with no data-path collective; ranks only agree on timing.

Each rank draws its own batch (bench.rank_seed), runs the oracle on it (CPU
stand-in for its GPU), and the job's time is the max over ranks
(bench.max_over_ranks) -- the same helpers bench.py uses under NCCL."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    import oracle as orc
    import workloads as W
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = W.GQAConfig("shard", B=2, H_q=4, H_kv=2, d=16, seq_lens=[70, 130],
                          dtype=torch.float32, seed=11)
        x = W.make_gqa_inputs(cfg, seed=bench.rank_seed(cfg.seed, rank))
        out = orc.decode_gqa(x.q, x.k_cache, x.v_cache, x.seq_lens, x.block_table,
                             x.scale)
        fake_ms = 10.0 + 5.0 * rank            # per-rank device time stand-in
        ms_max = bench.max_over_ranks(fake_ms, world)
        value = bench.whole_job_tokens_per_s(world, cfg.B, 4, ms_max)
        q.put((rank, float(out.sum()), float(x.q.sum()), ms_max, value))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_rank_weak_scaling_shards_and_timing():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    # ranks drew different batches (own sequences) ...
    assert res[0][2] != res[1][2]
    # ... and agree on the job time = the slowest rank
    assert res[0][3] == res[1][3] == 15.0
    # whole-job throughput counts every rank's sequences over that time
    assert res[0][4] == pytest.approx(2 * 2 * 4 / 0.015)


def test_single_rank_helpers_without_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.rank_seed(100, 0) != bench.rank_seed(100, 1)
    assert bench.whole_job_tokens_per_s(1, 16, 50, 5.0) == pytest.approx(16 * 50 / 0.005)
