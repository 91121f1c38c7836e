"""Host-side logic of the multi-GPU bench path on CPU: two gloo ranks agree
on the max-over-ranks time, draw independent batches, and only rank 0 runs
the reference arm (the data path itself has no collective)."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import bench
    from gist_token_chunk_b200.inputs import WORKLOADS, make_inputs

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # the slowest rank's time wins
        t = bench.max_over_ranks(10.0 + rank, dist, "cpu")
        # each rank decodes its own, different batch
        w = WORKLOADS["tiny_fp32"]
        x = make_inputs(w, seed=bench.rank_seed(1003, 0, rank), device="cpu")
        q = [torch.zeros_like(x["q"]) for _ in range(world)]
        dist.all_gather(q, x["q"])
        distinct = not torch.equal(q[0], q[1])

        # reference arm: ranks > 0 exit at once without work
        class A:
            config, seed, warmup, steps, gpus = "tiny_fp32", 1003, 3, 2, world

        ref_rc = bench.run_reference(A) if rank > 0 else 0
        out[rank] = (t, distinct, ref_rc, bench.rank_seed(1003, 0, rank))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()  # no fork of a process with OpenMP threads
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    assert out[0][0] == out[1][0] == 11.0
    assert out[0][1] and out[1][1]
    assert out[1][2] == 0
    assert out[0][3] != out[1][3]
