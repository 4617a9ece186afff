"""Host logic of the multi-GPU benchmark path, on CPU with two gloo ranks.

Each rank processes its own batch (seed + rank), times it, and the job time
is the maximum over ranks; no collective touches the data path.
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


def _worker(rank, world, port, out):
    import sys

    sys.path.insert(0, ROOT)
    import bench
    from synthetic import get_workload

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        w = get_workload("tiny")
        d = bench.rank_inputs(w, rank)
        # a per-rank "elapsed time": the job time is the slowest rank's
        job = bench.max_over_ranks(10.0 + 5.0 * rank)
        # every rank sees the same job time; each rank's batch is its own
        digest = torch.tensor([float(d["logits"].astype(np.float64).sum())], dtype=torch.float64)
        gathered = [torch.zeros_like(digest) for _ in range(world)]
        dist.all_gather(gathered, digest)
        out[rank] = (job, [float(g.item()) for g in gathered])
    finally:
        dist.destroy_process_group()


def test_two_ranks_share_the_max_time_and_own_batches():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    digests = res[0][1]
    assert digests == res[1][1]
    assert digests[0] != digests[1]  # independent batches per rank


def test_single_process_max_is_identity():
    import sys

    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.25) == 3.25


def test_rank_inputs_are_deterministic():
    import sys

    sys.path.insert(0, ROOT)
    import bench
    from synthetic import get_workload

    w = get_workload("tiny")
    a, b = bench.rank_inputs(w, 1), bench.rank_inputs(w, 1)
    assert all(np.array_equal(a[k], b[k]) for k in a)
    c = bench.rank_inputs(w, 0)
    assert not np.array_equal(a["hidden"], c["hidden"])
