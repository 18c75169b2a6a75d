"""GPU parity of the activation front-end (bf16 -> per-token int8) and of the
GEMV on bf16 activations, through the C ABI, against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from bit_gemv_sherry_b200 import sherry as S
from tests.gpu_helpers import dev, dev_codes

pytestmark = pytest.mark.gpu


def bf16_rows(B, K, seed):
    """Seeded bf16 bit patterns: normal rows of very different magnitudes, an
    all-zero row, and a row of hand values with exact rounding ties."""
    rng = np.random.default_rng(seed)
    mags = np.array([1.0, 1e-3, 37.0, 2e4, 0.25, 3.0], np.float32)
    x = rng.standard_normal((B, K)).astype(np.float32) * mags[np.arange(B) % len(mags)][:, None]
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    if B >= 2:
        bits[1] = 0
    if B >= 3 and K >= 8:
        bits[2, :8] = oracle.bf16_bits([127.0, 1.0, -0.5, 0.25, -127.0, 63.5, 0.0, 126.5])
        bits[2, 8:] = 0
    return bits


def to_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.parametrize("B,K", [(1, 128), (3, 2048), (16, 1024), (5, 8), (2, 8192)])
def test_quantize_act_matches_oracle(B, K):
    bits = bf16_rows(B, K, seed=30 + B)
    q_ref, s_ref = oracle.quantize_act(bits)
    q, s = S.quantize_act(to_bf16(bits))
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy(), s_ref)


@pytest.mark.parametrize("N,K,B", [(256, 1024, 1), (100, 3072, 2), (70, 2048, 5), (37, 640, 3),
                                   (48, 8192, 16), (31, 8192, 1)])
def test_gemv_bf16_matches_oracle(N, K, B):
    codes, scales = oracle.pack(synth.latent_weights(N, K, seed=40 + N))
    bits = bf16_rows(B, K, seed=50 + B)
    q_ref, s_ref = oracle.quantize_act(bits)
    acc = oracle.gemv_acc(codes, q_ref, N, K)
    # one fp32 rounding for s_w * s_b, one for the product with the exact acc
    expect = (scales[None, :] * s_ref[:, None]).astype(np.float32) * acc.astype(np.float32)
    y = S.gemv_bf16(dev_codes(codes), dev(scales), to_bf16(bits)).cpu().numpy()
    assert np.array_equal(y, expect.astype(np.float32))
    ref = oracle.gemv_act(codes, scales, q_ref, s_ref, K)
    rel = np.abs(y.astype(np.float64) - ref) / np.maximum(np.abs(ref), 1e-300)
    rel[(ref == 0) & (y == 0)] = 0.0
    assert rel.max() <= 1e-6


def test_gemv_bf16_grouped_equals_single_calls():
    dev_ = torch.device("cuda")
    items, singles = [], []
    for i, (name, n, k) in enumerate(synth.LLAMA_1B_LAYERS):
        w = torch.from_numpy(synth.latent_weights(n, k, seed=60 + i)).to(dev_)
        c, s = S.pack(w)
        x = to_bf16(bf16_rows(1, k, seed=70 + i))
        y = torch.empty((1, n), dtype=torch.float32, device=dev_)
        items.append((c, s, x, y))
        singles.append(S.gemv_bf16(c, s, x))
    S.gemv_bf16_grouped(items, 1)
    torch.cuda.synchronize()
    for (_, _, _, y), ref in zip(items, singles):
        assert torch.equal(y, ref)
    assert S.device_error() == 0


@pytest.mark.parametrize("B", [1, 2])
def test_gemv_bf16_small_calls_quantize_in_the_gemv(B):
    """Small bf16 calls (B <= 2) skip the re-order launch: each warp takes the
    token's absmax and quantizes its chunks itself.  One activation buffer read
    as two row lengths (a 2048-value prefix of an 8192-value token) in one
    grouped call must give two different scales; y is the oracle's bit for bit."""
    cuda = torch.device("cuda")
    bits = bf16_rows(B, 8192, seed=170 + B)
    xfull = to_bf16(bits)
    cases = [(64, 8192, xfull, bits)]
    if B == 1:
        cases.append((96, 2048, xfull[:, :2048], bits[:, :2048]))
    items, refs = [], []
    for i, (n, k, xt, xb) in enumerate(cases):
        codes, scales = oracle.pack(synth.latent_weights(n, k, seed=180 + i))
        q_ref, s_ref = oracle.quantize_act(np.ascontiguousarray(xb))
        acc = oracle.gemv_acc(codes, q_ref, n, k)
        refs.append((scales[None, :] * s_ref[:, None]).astype(np.float32) * acc.astype(np.float32))
        y = torch.empty((B, n), dtype=torch.float32, device=cuda)
        items.append((dev_codes(codes), dev(scales), xt, y))
        assert np.array_equal(S.gemv_bf16(items[-1][0], items[-1][1], xt).cpu().numpy(), refs[-1])
    S.gemv_bf16_grouped(items, B)
    torch.cuda.synchronize()
    for (_, _, _, y), ref in zip(items, refs):
        assert np.array_equal(y.cpu().numpy(), ref)
    assert S.device_error() == 0


@pytest.mark.parametrize("B", [1, 2])
def test_gemv_bf16_large_group_through_the_reorder_launch(B):
    """A bf16 call too large for the in-kernel quantization (3 layers of the 1B
    stack, 21 GEMVs, 11,136 chunks) quantizes in the re-order launch and the dot
    kernel reads the scales from the workspace; every output of every GEMV
    against the oracle, bit for bit."""
    cuda = torch.device("cuda")
    rng = np.random.default_rng(190 + B)
    xb = {k: bf16_rows(B, k, seed=200 + k + B) for k in (2048, 8192)}
    xt = {k: to_bf16(v) for k, v in xb.items()}
    q_s = {k: oracle.quantize_act(v) for k, v in xb.items()}
    items, host = [], []
    for _, _, n, k, _ in synth.decode_stack(3):
        codes = rng.integers(0, 2 ** 32, size=((n + 31) // 32, k // 128, 5, 32),
                             dtype=np.uint64).astype(np.uint32)
        scales = (rng.random(n) * 0.05 + 1e-3).astype(np.float32)
        y = torch.empty((B, n), dtype=torch.float32, device=cuda)
        items.append((dev_codes(codes), dev(scales), xt[k], y))
        host.append((codes, scales, k))
    S.gemv_bf16_grouped(items, B)
    torch.cuda.synchronize()
    for (codes, scales, k), it in zip(host, items):
        q_ref, s_ref = q_s[k]
        acc = oracle.gemv_acc(codes, q_ref, scales.shape[0], k)
        ref = (scales[None, :] * s_ref[:, None]).astype(np.float32) * acc.astype(np.float32)
        assert np.array_equal(it[3].cpu().numpy(), ref)
    assert S.device_error() == 0


def test_gemv_bf16_grouped_shared_activations():
    """bf16 GEMVs sharing one activation tensor, in a call that takes the
    re-order launch (a split-K row rules out the in-kernel quantization): the
    GEMVs after the first read its quantized copy and its token scales; y is
    the oracle's bit for bit for every GEMV."""
    cuda = torch.device("cuda")
    B = 2
    bits_a, bits_b = bf16_rows(B, 2048, seed=990), bf16_rows(B, 10752, seed=991)
    xa, xb = to_bf16(bits_a), to_bf16(bits_b)
    spec = [(96, 2048, xa, bits_a), (64, 10752, xb, bits_b), (200, 2048, xa, bits_a),
            (33, 10752, xb, bits_b), (7, 2048, xa, bits_a)]
    items, refs = [], []
    for i, (n, k, xt, bits) in enumerate(spec):
        codes, scales = oracle.pack(synth.latent_weights(n, k, seed=1000 + i))
        q_ref, s_ref = oracle.quantize_act(bits)
        acc = oracle.gemv_acc(codes, q_ref, n, k)
        refs.append((scales[None, :] * s_ref[:, None]).astype(np.float32) * acc.astype(np.float32))
        items.append((dev_codes(codes), dev(scales), xt,
                      torch.full((B, n), float("nan"), dtype=torch.float32, device=cuda)))
    S.gemv_bf16_grouped(items, B)
    torch.cuda.synchronize()
    for (_, _, _, y), ref in zip(items, refs):
        assert np.array_equal(y.cpu().numpy(), ref)
    assert S.device_error() == 0
