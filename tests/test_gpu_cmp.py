"""The comparison formats on the GPU against the oracle (needs a B200).

The pages set Sherry's 1.25 bits per weight against a 2-bit aligned packing
and a packing of three weights in five bits (arXiv 2601.07892, abstract;
Figure 2 caption).  The library holds the same ternary matrix in those
formats (a transcode of Sherry codes) and runs the same decode GEMV on them.
Bars: transcoded words bit-exact against the oracle's encoder of the oracle's
unpacked matrix; int32 accumulators bit-exact against the oracle's GEMV in
that format; y equal to the fp32 rounding of s * acc (the same acc as
Sherry's, since the matrix is the same).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from bit_gemv_sherry_b200 import sherry as S
from tests.gpu_helpers import assert_y_matches, dev, dev_codes, host_codes

pytestmark = pytest.mark.gpu
FMTS = [(S.CMP_I2, oracle.FMT_I2), (S.CMP_T3, oracle.FMT_T3)]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    S.lib()
    yield
    assert S.device_error() == 0


@pytest.mark.parametrize("fmt,ofmt", FMTS, ids=["i2", "t3"])
@pytest.mark.parametrize("N,K", [(1, 128), (33, 384), (70, 1152), (64, 2048), (40, 8192)])
def test_transcode_matches_oracle_encoder(fmt, ofmt, N, K):
    codes, _ = oracle.pack(synth.latent_weights(N, K, seed=N + 3 * K))
    got = host_codes(S.cmp_transcode(fmt, dev_codes(codes), N))
    want = oracle.cmp_encode(ofmt, oracle.unpack(codes, N, K))
    assert got.shape == want.shape
    assert np.array_equal(got, want)


@pytest.mark.parametrize("fmt,ofmt", FMTS, ids=["i2", "t3"])
@pytest.mark.parametrize("N,K,B", [(256, 1024, 1), (33, 2048, 2), (300, 512, 1), (96, 8192, 2),
                                   (2048, 2048, 1)])
def test_cmp_gemv_acc_matches_oracle(fmt, ofmt, N, K, B):
    codes, _ = oracle.pack(synth.latent_weights(N, K, seed=N + K))
    x = synth.int8_uniform((B, K), seed=B + 10)
    wt = oracle.unpack(codes, N, K)
    c = oracle.cmp_encode(ofmt, wt)
    acc = S.cmp_gemv_acc(fmt, dev_codes(c), dev(x), N, K).cpu().numpy().astype(np.int64)
    want = oracle.cmp_gemv_acc(ofmt, c, x, N, K)
    assert np.array_equal(acc, want)
    # the same ternary matrix: the same products as Sherry's oracle
    assert np.array_equal(want, oracle.gemv_acc(codes, x, N, K))


@pytest.mark.parametrize("fmt", [S.CMP_I2, S.CMP_T3], ids=["i2", "t3"])
def test_cmp_grouped_llama_1b_layer_as_benched(fmt):
    """One 1B layer (q, k, v, o, gate, up, down), B = 1, codes transcoded on the
    GPU from GPU-packed codes; every output compared."""
    items, refs = [], []
    xs = {k: synth.int8_uniform((1, k), seed=1 if k == 2048 else 2) for k in (2048, 8192)}
    dxs = {k: dev(v) for k, v in xs.items()}
    for pi, (name, n, k) in enumerate(synth.LLAMA_1B_LAYERS):
        w = torch.from_numpy(synth.latent_weights(n, k, seed=synth.layer_seed(0, pi))).cuda()
        codes, scales = S.pack(w)
        del w
        cc = S.cmp_transcode(fmt, codes, n)
        y = torch.full((1, n), float("nan"), device="cuda")
        items.append((cc, scales, dxs[k], y, k))
        refs.append((host_codes(codes), scales.cpu().numpy(), k))
    S.GroupedCmpGemv(fmt, items, B=1)()
    torch.cuda.synchronize()
    for (_, _, _, y, _), (c, s, k) in zip(items, refs):
        assert_y_matches(y.cpu().numpy(), oracle.gemv(c, s, xs[k], k))


def test_cmp_argument_checks():
    L = S.lib()
    fake = torch.zeros(64, dtype=torch.int32, device="cuda")
    x = torch.zeros((3, 512), dtype=torch.int8, device="cuda")
    acc = torch.zeros((3, 32), dtype=torch.int32, device="cuda")
    ws = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    # B > 2, unknown format, I2 with K not a multiple of 512
    assert L.sherry_cmp_gemv_acc(1, fake.data_ptr(), x.data_ptr(), acc.data_ptr(), 32, 512, 3,
                                 ws.data_ptr(), ws.numel(), st) == 4
    assert L.sherry_cmp_gemv_acc(9, fake.data_ptr(), x.data_ptr(), acc.data_ptr(), 32, 512, 1,
                                 ws.data_ptr(), ws.numel(), st) == 4
    assert L.sherry_cmp_gemv_acc(1, fake.data_ptr(), x.data_ptr(), acc.data_ptr(), 32, 384, 1,
                                 ws.data_ptr(), ws.numel(), st) == 2
    assert L.sherry_cmp_packed_bytes(2, 32, 2048) == 32 * 22 * 5 * 4
