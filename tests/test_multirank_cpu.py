"""The N > 1 host path of bench.py with two gloo ranks on the CPU.

Each rank quantizes its own batch of tokens (weak scaling: same shapes,
different seeds) and the job's number is the bytes summed over ranks divided
by the slowest rank's time.  Nothing here touches a GPU.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    r, w, local = bench.dist_env()
    assert (r, w, local) == (rank, world, rank)
    bench.dist_init(w, "gloo")
    ws = bench.step_workloads(r)
    bench.barrier(w)
    elapsed = 10.0 + rank            # pretend rank 1 is slower
    slowest = bench.max_over_ranks(elapsed, w)
    total = bench.sum_over_ranks(bench.step_bytes(ws), w)
    out[rank] = (slowest, total, [(x.M, x.d, x.seed) for x in ws])
    dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    sys.path.insert(0, ROOT)
    import bench
    (s0, t0, w0), (s1, t1, w1) = out[0], out[1]
    assert s0 == s1 == 11.0                       # max over ranks
    assert t0 == t1 == 2 * bench.step_bytes(bench.step_workloads(0))
    assert [m for m, _, _ in w0] == [m for m, _, _ in w1]          # same shapes
    assert [d for _, d, _ in w0] == [d for _, d, _ in w1]
    assert all(a[2] != b[2] for a, b in zip(w0, w1))              # own tokens per rank


def test_rank_plan_and_bytes():
    sys.path.insert(0, ROOT)
    import bench
    ws = bench.step_workloads(0)
    assert [(w.M, w.d) for w in ws] == [(4608, 3072), (4608, 12288)]
    assert bench.algorithmic_bytes(4608, 12288) == 4608 * 12288 * 2.53125 + 384 * 60
    # the ring of input/output sets exceeds four times L2
    l2 = 126 * 2 ** 20
    for w in ws:
        assert bench.ring_depth(w, l2) * w.M * w.d * 2.53125 >= 4 * l2
