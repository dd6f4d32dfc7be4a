"""Multi-rank host logic on CPU (gloo, world size 2).

With more than one GPU the benchmark runs independent replicas: every rank
solves its own problem, no collective touches the data path, and the only
cross-rank steps are a barrier and a max-reduction of the per-rank device
times.  These tests run that logic as two gloo processes on the CPU:
  * max_over_ranks gives every rank the slowest rank's time;
  * replica_throughput counts all ranks' work against that time;
  * the per-rank problems are independent: each rank's result equals what the
    same rank computes alone (checked with the CPU oracle on small shards).
"""
import os
import socket

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


def _rank_main(rank, world, port, outdir):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        import oracle
        import workloads as WL
        # per-rank "device times": the slowest rank decides
        mine = [10.0 + 5.0 * rank, 1.0 + rank]
        got = bench.max_over_ranks(mine, "cpu")
        # each rank solves its own shard (seed = rank): no data exchange
        case = WL.make_wqmm_case(x1_shape=(4, 128), n=64, act="bf16", wdt="i4", mode="group", group_size=64,
                                 seed=100 + rank)
        ye, _ = oracle.wqmm(case)
        np.save(os.path.join(outdir, f"rank{rank}.npy"), ye)
        with open(os.path.join(outdir, f"rank{rank}.txt"), "w") as f:
            f.write(" ".join(str(v) for v in got))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_rank_run(tmp_path_factory):
    outdir = str(tmp_path_factory.mktemp("ranks"))
    import oracle
    oracle.build()  # build before spawning so the ranks only load it
    mp.spawn(_rank_main, args=(2, _free_port(), outdir), nprocs=2, join=True)
    return outdir


def test_every_rank_sees_the_slowest_time(two_rank_run):
    for r in range(2):
        vals = [float(v) for v in open(os.path.join(two_rank_run, f"rank{r}.txt")).read().split()]
        assert vals == [15.0, 2.0]


def test_replica_shards_are_independent(two_rank_run):
    import oracle
    import workloads as WL
    for r in range(2):
        case = WL.make_wqmm_case(x1_shape=(4, 128), n=64, act="bf16", wdt="i4", mode="group", group_size=64,
                                 seed=100 + r)
        alone, _ = oracle.wqmm(case)
        assert np.array_equal(np.load(os.path.join(two_rank_run, f"rank{r}.npy")), alone)


def test_replica_throughput_counts_all_ranks_against_the_slowest():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    flops = 2.0 * 4096 ** 3
    one = bench.replica_throughput(flops, 1, 10, 2.0)
    two = bench.replica_throughput(flops, 2, 10, 2.0)
    assert two == pytest.approx(2 * one)
    assert one == pytest.approx(flops * 10 / 2e-3 / 1e12)
    # a single process (no process group) is the identity
    assert bench.max_over_ranks([3.0, 4.0], "cpu") == [3.0, 4.0]
