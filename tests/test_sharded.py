"""Row-sharded GEMV over a process group, on CPU with gloo ranks.

Each rank holds a run of whole 32-row groups of the packed matrix; its local
y (here from the oracle, the CPU stand-in for the CUDA GEMV) and one
all-gather give every rank the whole y, which must equal the unsharded
oracle product exactly.  Covers equal and unequal shares, B = 1 and B > 1,
and a rank with no rows.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from bit_gemv_sherry_b200 import sharded  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_group_ranges_cover_all_rows_once():
    for N in (1, 31, 32, 33, 512, 2048, 3000):
        for W in (1, 2, 3, 4, 8):
            rows = [sharded.row_range(N, r, W) for r in range(W)]
            assert rows[0][0] == 0 and rows[-1][1] == N
            for (a0, a1), (b0, b1) in zip(rows, rows[1:]):
                assert a1 == b0 and a0 <= a1
            for r in range(W):
                g0, g1 = sharded.group_range(N, r, W)
                assert rows[r][0] == min(N, 32 * g0)
                assert rows[r][1] - rows[r][0] <= sharded.max_share_rows(N, W)
    # the LLaMA-3.2-1B shapes split evenly over 2, 4 and 8 ranks
    for N in (512, 2048, 8192):
        for W in (2, 4, 8):
            assert {b - a for a, b in (sharded.row_range(N, r, W) for r in range(W))} == {N // W}
    with pytest.raises(ValueError):
        sharded.group_range(64, 2, 2)


def _oracle_local_gemv(K):
    import oracle

    def run(codes, scales, x, y):
        c = codes.numpy().view(np.uint32)
        out = torch.from_numpy(oracle.gemv(c, scales.numpy(), x.numpy(), K).astype(np.float32))
        if y is None:
            return out
        y.copy_(out)
        return y
    return run


def _rank(rank, world, port, cases, out):
    import oracle
    import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = []
        for N, K, B in cases:
            codes, scales = oracle.pack(synth.latent_weights(N, K, seed=N + K))
            x = synth.int8_uniform((B, K), seed=B + 3)
            ref = oracle.gemv(codes, scales, x, K).astype(np.float32)
            tc = torch.from_numpy(codes.view(np.int32))
            ts = torch.from_numpy(scales)
            c_r, s_r, (n0, n1) = sharded.shard(tc, ts, rank, world)
            g = sharded.ShardedGemv(c_r, s_r, N, K, B, local_gemv=_oracle_local_gemv(K))
            y = g(torch.from_numpy(x))
            res.append(bool(np.array_equal(y.numpy(), ref)) and tuple(y.shape) == (B, N))
        out[rank] = res
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,cases", [
    (2, [(256, 1024, 1), (96, 512, 3), (33, 384, 2)]),   # equal; unequal (3 groups); tail group
    (3, [(64, 256, 1), (100, 640, 1)]),                  # a rank with no rows; unequal at B = 1
])
def test_sharded_gemv_gathers_the_unsharded_product(world, cases):
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_rank, args=(world, port, cases, out), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        assert out[r] == [True] * len(cases), (r, out[r])
