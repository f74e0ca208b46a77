"""Multi-GPU path of the benchmark on CPU: two `gloo` ranks as B-sharded replicas.

Each rank verifies its own batch (distinct seeds, so distinct sequences), no collective
touches the data path, and the whole-job throughput is all ranks' blocks over the slowest
rank's time."""

import os
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    from lossless_draft_verification_speculative_b200 import workloads as wl
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank's batch: the first sequence of its own logits
        w = wl.Workload("r", B=2, K=1, V=16, dtype="f32", kind="iid", params={"sd": 2.0})
        P, _ = wl.logits(w, [0], seed=bench.rank_seed(rank))
        ms_local = 10.0 + 5.0 * rank            # rank 1 is the slow one
        value, ms_max = bench.aggregate(ms_local, blocks_per_rank=300, world=world, dist=dist)
        out[rank] = (float(P.sum()), value, ms_max)
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_take_max_time_and_distinct_batches():
    port = 29500 + os.getpid() % 1000
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    (s0, v0, t0), (s1, v1, t1) = res[0], res[1]
    assert s0 != s1                                   # different sequences on each rank
    assert t0 == t1 == pytest.approx(15.0)            # both see the max over ranks
    assert v0 == v1 == pytest.approx(2 * 300 / 0.015)  # all ranks' blocks / slowest time
