"""The multi-process (weak scaling) logic of bench.py on CPU: two gloo ranks.

Each rank runs an independent problem of the same shape (its own seed), no
collective touches the data, and the job time is the maximum over ranks.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import gdr_workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench.rank_workload(W.WORKLOADS["kda_tiny_fp32"], rank)
        x = W.generate(w)
        # a rank-dependent "measured" time: the job time must be the slowest rank's
        t_ms = 10.0 + 5.0 * rank
        t_max = bench.reduce_max(t_ms, world, torch.device("cpu"))
        out[rank] = (w.seed, float(x["q"].double().sum()), t_max,
                     bench.job_throughput(w.B * w.T, world, t_max, steps=4))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, start_method="spawn")
    (s0, q0, m0, v0), (s1, q1, m1, v1) = out[0], out[1]
    assert s0 != s1 and q0 != q1              # independent problems per rank
    assert m0 == m1 == 15.0                   # max over ranks, seen by every rank
    w = W.WORKLOADS["kda_tiny_fp32"]
    assert v0 == v1 == pytest.approx(w.B * w.T * world / (15.0 / 4 / 1e3))


def test_single_rank_needs_no_process_group():
    assert bench.reduce_max(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.job_throughput(100, 1, 2.0, steps=2) == pytest.approx(100 / 1e-3)
