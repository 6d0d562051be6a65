"""The N > 1 path of bench.py on the CPU: two gloo ranks.

The layer has no cross-GPU exchange, so N GPUs run N independent replicas; the
only collectives are a barrier and a max-reduction of the per-rank timings
(the job's time is the slowest rank's).  These tests run that plumbing with
world size 2 on the host; METIS_DIST_BACKEND=gloo keeps them on the gloo
backend and host tensors even where a GPU is present.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "METIS_DIST_BACKEND": "gloo"})
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    r, w, local = bench.dist_init()
    try:
        assert dist.get_backend() == "gloo"
        bench.barrier(w)
        # rank 1 is the slow one: the job time is its time
        t = bench.reduce_max(1.5 if r == 1 else 1.0, w)
        out[r] = (r, w, local, t)
        bench.barrier(w)
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_to_the_slowest():
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    for r, (rank, world, local, t) in res.items():
        assert (rank, world, local) == (r, 2, r)
        assert t == pytest.approx(1.5)


def _ref_worker(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "METIS_DIST_BACKEND": "gloo"})
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    r, w, _ = bench.dist_init()
    try:
        if r != 0:
            # the reference arm: ranks other than 0 return without work
            class A:
                steps, warmup, gpus = 1, 0, w
            bench.run_reference(A, r, w)
            out[r] = "returned"
        else:
            out[r] = "skipped"
        bench.barrier(w)
    finally:
        dist.destroy_process_group()


def test_reference_arm_runs_on_rank_zero_only():
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_ref_worker, args=(2, port, out), nprocs=2, join=True)
        assert dict(out) == {0: "skipped", 1: "returned"}
