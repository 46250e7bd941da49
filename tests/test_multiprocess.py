"""The N > 1 host path of bench.py on CPU: two gloo ranks take the same
collective steps (barrier, max over ranks) and the whole-job rate uses the
slowest rank's time; replicas draw their own seeded inputs."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench
from token_level_top_hs2_b200 import inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    w, r, local = bench.dist_setup(world, backend="gloo")
    assert (w, r, local) == (world, rank, rank)
    bench.barrier(w)
    # per-rank timings differ; every rank sees the element-wise maximum
    mine = [1.0 + rank, 5.0 - rank, 2.5]
    got = bench.max_over_ranks(mine, w)
    out[rank] = got
    bench.barrier(w)
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_timings():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    want = [2.0, 5.0, 2.5]
    assert out[0] == want and out[1] == want


def test_whole_job_rate_uses_slowest_rank():
    # 2 ranks x 131072 tokens, slowest rank 0.125 s
    assert bench.whole_job_rate(2, 131072, 0.125) == pytest.approx(2 * 131072 / 0.125)
    assert bench.whole_job_rate(1, 10, 2.0) == 5.0


def test_replicas_draw_distinct_inputs():
    a = inputs.make_prefill(1, 64, 4, 64, 8, 8, seed=inputs.seed_for(2, 0))
    b = inputs.make_prefill(1, 64, 4, 64, 8, 8, seed=inputs.seed_for(2, 1))
    assert not torch.equal(a.q, b.q)
    assert inputs.seed_for(2, 1) - inputs.seed_for(2, 0) == 1000
