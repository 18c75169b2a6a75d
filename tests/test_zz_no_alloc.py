"""sherry_gemv_static (the GEMV whose scratch is a fixed device array inside the
library) against sherry_gemv with a caller workspace, through the C ABI.

Collected last on purpose: it must pass in a fresh process and after every
other test, i.e. whatever the static array holds from earlier calls.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from bit_gemv_sherry_b200 import sherry as S

pytestmark = pytest.mark.gpu


def _layer(N, K, seed):
    w = torch.from_numpy(synth.latent_weights(N, K, seed=seed)).cuda()
    codes, scales = S.pack(w)
    return codes, scales


def _x(B, K, seed):
    return torch.from_numpy(synth.int8_uniform((B, K), seed=seed)).cuda()


# (2048, 16384, 4): rows longer than 8192 are split into K-parts, so the static
# array also holds the int32 partial sums and the per-unit counters, which each
# call must find cleared by the call before it.
@pytest.mark.parametrize("N,K,B", [(2048, 8192, 1), (1000, 2048, 5), (4096, 4096, 16),
                                   (33, 384, 3), (2048, 16384, 4), (70, 17408, 1),
                                   # the largest K: 16 K-parts, 2 MiB of activations
                                   (40, 131072, 16)])
def test_static_matches_workspace_gemv_two_calls_in_a_row(N, K, B):
    codes, scales = _layer(N, K, seed=900 + N % 97)
    x1, x2 = _x(B, K, seed=901), _x(B, K, seed=902)
    y1 = torch.full((B, N), float("nan"), device="cuda")
    y2 = torch.full((B, N), float("nan"), device="cuda")
    L = S.lib()
    stream = torch.cuda.current_stream().cuda_stream
    for x, y in ((x1, y1), (x2, y2)):   # back to back on one stream, no host sync between
        st = L.sherry_gemv_static(codes.data_ptr(), scales.data_ptr(), x.data_ptr(),
                                  y.data_ptr(), N, K, B, ctypes.c_void_p(stream))
        assert st == 0, S.lib().sherry_last_error()
    r1 = S.gemv(codes, scales, x1)
    r2 = S.gemv(codes, scales, x2)
    torch.cuda.synchronize()
    assert torch.equal(y1, r1)
    assert torch.equal(y2, r2)
    assert not torch.equal(y1, y2)
    assert S.device_error() == 0


def test_static_binding_and_repeat_after_other_shapes():
    codes, scales = _layer(512, 2048, seed=911)
    x = _x(2, 2048, seed=912)
    ref = S.gemv(codes, scales, x)
    for _ in range(2):
        y = S.gemv_static(codes, scales, x)
        torch.cuda.synchronize()
        assert torch.equal(y, ref)


def test_static_rejects_sizes_beyond_the_scratch():
    N, K, B = 100000, 131072, 16  # K-part sums of rows split past K = 8192
    assert S.gemv_workspace_bytes(N, K, B) > S.STATIC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x100000)
    L = S.lib()
    assert L.sherry_gemv_static(fake, fake, fake, fake, N, K, B, None) == 7
    msg = L.sherry_last_error().decode()
    assert "sherry_gemv_static" in msg and str(S.STATIC_SCRATCH_BYTES) in msg
    assert np.int64(S.gemv_workspace_bytes(4096, 8192, 16)) <= S.STATIC_SCRATCH_BYTES
