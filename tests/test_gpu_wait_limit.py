"""The GEMM's bounded barrier waits run out on purpose (needs a B200).

With a limit of a few dozen SM cycles, the epilogue's wait for the first
accumulator cannot complete (the decoders have not even loaded their codes),
so the kernel records SHERRY_ERR_TIMEOUT, lets the copies and MMAs it issued
finish, releases its tensor memory and returns.  The host reads the status
with sherry_device_error(); the context stays usable, which a normal GEMM
right after shows bit-exact against the oracle.  No fault and no hang: every
wait in the kernel is bounded and the drains keep their long limit.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from bit_gemv_sherry_b200 import sherry as S
from tests.gpu_helpers import assert_y_matches, dev, dev_codes

pytestmark = pytest.mark.gpu

TIMEOUT = 6  # SHERRY_ERR_TIMEOUT


@pytest.fixture(autouse=True)
def _restore_limit():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert S.device_error() == 0
    yield
    S.set_wait_limit(0)


@pytest.mark.parametrize("M,N,K", [(256, 256, 256), (300, 384, 1024)])
def test_short_wait_limit_times_out_then_a_normal_gemm_is_exact(M, N, K):
    codes, scales = oracle.pack(synth.latent_weights(N, K, seed=21))
    x = synth.int8_clipped_normal((M, K), seed=22)
    tc, ts, tx = dev_codes(codes), dev(scales), dev(x)

    S.set_wait_limit(64)
    S.gemm(tc, ts, tx)                       # gives up: its output is undefined
    assert S.device_error() == TIMEOUT       # synchronises, reads and clears
    assert S.device_error() == 0             # cleared

    S.set_wait_limit(0)                      # default limit again
    y = S.gemm(tc, ts, tx)
    assert_y_matches(y.cpu().numpy(), oracle.gemm(codes, scales, x, K))
    acc = S.gemm_acc(tc, tx, N)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), oracle.gemm_acc(codes, x, N, K))
    assert S.device_error() == 0


def test_timeouts_back_to_back_leave_the_context_usable():
    N, K, M = 256, 512, 512
    codes, scales = oracle.pack(synth.latent_weights(N, K, seed=23))
    x = synth.int8_clipped_normal((M, K), seed=24)
    tc, ts, tx = dev_codes(codes), dev(scales), dev(x)
    S.set_wait_limit(32)
    for _ in range(3):
        S.gemm(tc, ts, tx)
    assert S.device_error() == TIMEOUT
    S.set_wait_limit(0)
    y = S.gemm(tc, ts, tx)
    assert_y_matches(y.cpu().numpy(), oracle.gemm(codes, scales, x, K))
    assert S.device_error() == 0
