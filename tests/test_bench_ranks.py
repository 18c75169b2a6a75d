"""Multi-rank host logic of bench.py on the CPU: two gloo ranks agree on the
MAX of their step times, and the whole-job value counts every rank's replica.
(No GPU: the ranks exchange only host tensors.)"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [0.25, 0.75][rank]
        t_max = bench.max_over_ranks(local, dist, "cpu")
        out[rank] = t_max
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_step_time():
    world = 2
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_rank, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0] == out[1] == 0.75


def test_single_process_is_identity_and_value_counts_replicas():
    assert bench.max_over_ranks(0.5) == 0.5
    # two replicas of a 152,043,520-byte step, 100 steps in 0.01 s of max time
    v = bench.whole_job_value(2, 152043520, 100, 0.01)
    assert v == pytest.approx(2 * 152043520 * 100 / 0.01 / 1e9)
