"""Row-sharded GEMV on the device through NCCL (needs a B200).

Only one GPU is available to a test run, so the process group has one rank:
the shard is the whole matrix and the all-gather is NCCL's one-rank copy.
This checks the device path of ShardedGemv (the library's GEMV into the
gather buffer, NCCL's all_gather_into_tensor, the re-assembly) against the
oracle; the multi-rank split and gather logic is tested on CPU with gloo.
"""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
import synth
from bit_gemv_sherry_b200 import sharded
from tests.gpu_helpers import assert_y_matches, dev, dev_codes

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def nccl_group():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("N,K,B", [(2048, 2048, 1), (512, 2048, 2), (100, 1024, 3)])
def test_one_rank_sharded_gemv_equals_oracle(nccl_group, N, K, B):
    codes, scales = oracle.pack(synth.latent_weights(N, K, seed=N + 7))
    x = synth.int8_uniform((B, K), seed=B + 11)
    c_r, s_r, (n0, n1) = sharded.shard(dev_codes(codes), dev(scales), 0, 1)
    assert (n0, n1) == (0, N)
    g = sharded.ShardedGemv(c_r, s_r, N, K, B)
    y = g(dev(x))
    torch.cuda.synchronize()
    assert tuple(y.shape) == (B, N)
    assert_y_matches(y.cpu().numpy(), oracle.gemv(codes, scales, x, K))
