"""CUDA path vs the CPU oracle on the same seeded inputs (needs a B200).

Bars: packed codes and integer accumulators bit-exact; scales within 1 ulp
(double sums in a different order; the count of non-identical rows is
checked too); fp32 outputs equal to the fp32 rounding of the exact
s * acc, hence within 1e-6 relative.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from bit_gemv_sherry_b200 import sherry as S
from tests.gpu_helpers import assert_y_matches, dev, dev_codes, host_codes
from tests.helpers import load_tiles, ulp_diff_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    S.lib()
    yield
    assert S.device_error() == 0


# ----------------------------------------------------------------------------- pack
@pytest.mark.parametrize("N,K", [(256, 1024), (1, 128), (7, 384), (33, 640), (5, 1152),
                                 (300, 2048), (9, 8192),
                                 # rows shared by 2 and 4 warps, each ending on a short batch
                                 (7, 25600), (5, 38400), (3, 67200)])
def test_pack_matches_oracle(N, K):
    w = synth.latent_weights(N, K, seed=0)
    codes_ref, scales_ref = oracle.pack(w)
    codes, scales = S.pack(dev(w))
    torch.cuda.synchronize()
    assert np.array_equal(host_codes(codes), codes_ref)
    d = ulp_diff_f32(scales.cpu().numpy(), scales_ref)
    assert d.max() <= 1
    assert (d > 0).sum() <= max(1, N // 1000)


def test_pack_golden_tiles(golden_dir):
    tiles = load_tiles(golden_dir)
    w = np.stack([t["latent"] for t in tiles])
    codes_ref, scales_ref = oracle.pack(w)
    codes, scales = S.pack(dev(w))
    assert np.array_equal(host_codes(codes), codes_ref)
    assert np.array_equal(scales.cpu().numpy(), scales_ref)
    for n, t in enumerate(tiles):
        assert [int(host_codes(codes)[0, 0, p, n]) for p in range(5)] == t["words"]


@pytest.mark.parametrize("layer", range(7))
def test_pack_full_size_1b_layers(layer):
    name, N, K = synth.LLAMA_1B_LAYERS[layer]
    w = synth.latent_weights(N, K, seed=synth.layer_seed(0, layer))
    codes_ref, scales_ref = oracle.pack(w)
    codes, scales = S.pack(dev(w))
    assert np.array_equal(host_codes(codes), codes_ref), name
    d = ulp_diff_f32(scales.cpu().numpy(), scales_ref)
    assert d.max() <= 1 and (d > 0).sum() <= max(1, N // 1000), name


def test_pack_grouped_matches_single_calls_and_oracle():
    # one launch over matrices of mixed shapes (ragged rows, K from 128 to 8192),
    # bit for bit the codes and scales of one sherry_pack call per matrix
    shapes = [(33, 640), (1, 128), (256, 1024), (7, 8192), (300, 2048), (64, 384), (5, 1152)]
    ws = [synth.latent_weights(N, K, seed=30 + i) for i, (N, K) in enumerate(shapes)]
    outs = S.pack_grouped([dev(w) for w in ws])
    torch.cuda.synchronize()
    for (N, K), w, (codes, scales) in zip(shapes, ws, outs):
        c1, s1 = S.pack(dev(w))
        assert np.array_equal(host_codes(codes), host_codes(c1)), (N, K)
        assert np.array_equal(scales.cpu().numpy(), s1.cpu().numpy()), (N, K)
        codes_ref, scales_ref = oracle.pack(w)
        assert np.array_equal(host_codes(codes), codes_ref), (N, K)
        assert ulp_diff_f32(scales.cpu().numpy(), scales_ref).max() <= 1, (N, K)


# ----------------------------------------------------------------------------- gemv
GEMV_CASES = [(256, 1024, 1), (1, 128, 1), (17, 384, 3), (33, 640, 5), (40, 1152, 8),
              (19, 256, 9), (64, 512, 16), (2048, 2048, 1), (512, 2048, 4), (100, 3072, 2),
              (31, 8192, 1), (48, 8192, 16), (50, 1536, 2), (23, 512, 1), (70, 2560, 9),
              (129, 4096, 8), (37, 8192, 2), (130, 2048, 3),
              # B = 5 ... 7 and 13 on the MMA kernel (activation groups of 8, padded rows)
              (96, 1024, 5), (200, 512, 6), (45, 2048, 7), (33, 1536, 13),
              # rows split into K-parts (K > 8192), short last parts included:
              # 21 chunks = 11 + 10, 34 = 12 + 12 + 10, 40 = 3 x 14 - 2, 128 = 8 x 16
              (70, 10752, 1), (33, 17408, 2), (40, 20480, 9), (20, 65536, 1), (65, 17408, 16)]


@pytest.mark.parametrize("N,K,B", GEMV_CASES)
def test_gemv_matches_oracle(N, K, B):
    w = synth.latent_weights(N, K, seed=0)
    codes, scales = oracle.pack(w)
    x = synth.int8_uniform((B, K), seed=1)
    tc, ts, tx = dev_codes(codes), dev(scales), dev(x)
    acc = S.gemv_acc(tc, tx, N)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), oracle.gemv_acc(codes, x, N, K))
    y = S.gemv(tc, ts, tx)
    assert_y_matches(y.cpu().numpy(), oracle.gemv(codes, scales, x, K))


@pytest.mark.parametrize("N,K,B", [(37, 640, 1), (16, 1152, 7), (70, 384, 12),
                                   # the MMA kernel's accumulator form, each activation group size
                                   (100, 512, 3), (64, 2048, 5), (33, 1024, 12), (40, 10752, 16)])
def test_gemv_random_words_full_int8_range(N, K, B):
    # every 32-bit pattern is a valid code; activations cover [-128, 127]
    rng = np.random.default_rng(N + K + B)
    codes = rng.integers(0, 2 ** 32, size=((N + 31) // 32, K // 128, 5, 32),
                         dtype=np.uint64).astype(np.uint32)
    x = rng.integers(-128, 128, size=(B, K)).astype(np.int8)
    acc = S.gemv_acc(dev_codes(codes), dev(x), N)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), oracle.gemv_acc(codes, x, N, K))


def test_gemv_unaligned_codes_take_the_register_path():
    # codes only 4-byte aligned: the cp.async path needs 16; results must not change
    N, K, B = 40, 2048, 3
    codes, scales = oracle.pack(synth.latent_weights(N, K, seed=8))
    x = synth.int8_uniform((B, K), seed=9)
    flat = torch.zeros(codes.size + 1, dtype=torch.int32, device="cuda")
    flat[1:].copy_(dev_codes(codes).view(-1))
    shifted = flat[1:].view(codes.shape)
    assert shifted.data_ptr() % 16 == 4
    acc = S.gemv_acc(shifted, dev(x), N)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), oracle.gemv_acc(codes, x, N, K))


def test_gemv_extreme_and_zero_activations():
    N, K = 64, 2048
    codes, scales = oracle.pack(synth.latent_weights(N, K, seed=3))
    x = np.stack([np.full(K, -128, np.int8), np.full(K, 127, np.int8), np.zeros(K, np.int8)])
    y = S.gemv(dev_codes(codes), dev(scales), dev(x)).cpu().numpy()
    assert_y_matches(y, oracle.gemv(codes, scales, x, K))
    assert np.all(y[2] == 0)


@pytest.mark.parametrize("B", [1, 4, 16])
def test_gemv_full_size_3b_layers(B):
    """All seven LLaMA-3.2-3B-shaped projections at B = 1, 4, 16: every output
    of every projection against the oracle, one call each and the seven as one
    grouped call."""
    x = {k: synth.int8_uniform((B, k), seed={1: 1, 4: 2, 16: 3}[B]) for k in (3072, 8192)}
    items, refs = [], []
    for li, (name, N, K) in enumerate(synth.LLAMA_3B_LAYERS):
        codes, scales = oracle.pack(synth.latent_weights(N, K, seed=synth.layer_seed(0, li)))
        ref = oracle.gemv(codes, scales, x[K], K)
        tc, ts = dev_codes(codes), dev(scales)
        assert_y_matches(S.gemv(tc, ts, dev(x[K])).cpu().numpy(), ref)
        items.append((tc, ts, dev(x[K]), torch.empty((B, N), dtype=torch.float32, device="cuda")))
        refs.append(ref)
    S.gemv_grouped(items, B=B)
    for (_, _, _, y), ref in zip(items, refs):
        assert_y_matches(y.cpu().numpy(), ref)


def test_gemv_grouped_1b_stack_layer():
    items, refs = [], []
    for li, (name, N, K) in enumerate(synth.LLAMA_1B_LAYERS):
        codes, scales = oracle.pack(synth.latent_weights(N, K, seed=synth.layer_seed(0, li)))
        x = synth.int8_uniform((1, K), seed=100 + li)
        y = torch.empty((1, N), dtype=torch.float32, device="cuda")
        items.append((dev_codes(codes), dev(scales), dev(x), y))
        refs.append(oracle.gemv(codes, scales, x, K))
    S.gemv_grouped(items, B=1)
    for (_, _, _, y), ref in zip(items, refs):
        assert_y_matches(y.cpu().numpy(), ref)


GROUPED_PIPELINED = [(33, 1536), (96, 8192), (1, 512), (70, 2560), (200, 2048), (45, 3584),
                     (64, 5120), (7, 1024), (130, 4096), (31, 2560), (40, 10752), (9, 17408)] * 3
# one K with T mod 4 != 0 sends the whole group to the register kernel
GROUPED_REGISTER = [(33, 640), (96, 8192), (1, 128), (70, 2560), (200, 2048), (45, 3584),
                    (64, 5120), (7, 384), (130, 4096), (31, 1152), (40, 10752), (9, 17408)] * 3


@pytest.mark.parametrize("B", [1, 2, 5])
@pytest.mark.parametrize("shapes", [GROUPED_PIPELINED, GROUPED_REGISTER], ids=["pipelined", "register"])
def test_gemv_grouped_cut_items(B, shapes):
    # many small GEMVs of mixed K (short last K-parts included) in one launch,
    # through prepare + run (the re-order launch): warp ranges cut items at many
    # places, inside and across GEMVs (dot kernel at B <= 2, MMA kernel at B = 5)
    items, refs = [], []
    for li, (N, K) in enumerate(shapes):
        codes, scales = oracle.pack(synth.latent_weights(N, K, seed=200 + li))
        x = synth.int8_uniform((B, K), seed=300 + li)
        y = torch.zeros((B, N), dtype=torch.float32, device="cuda")
        items.append((dev_codes(codes), dev(scales), dev(x), y))
        refs.append(oracle.gemv(codes, scales, x, K))
    g = S.GroupedGemv(items, B=B)
    g.prepare()
    for _ in range(2):
        for it in items:
            it[3].zero_()
        g.run()
        for (_, _, _, y), ref in zip(items, refs):
            assert_y_matches(y.cpu().numpy(), ref)


@pytest.mark.parametrize("B", [1, 2])
def test_gemv_grouped_two_unit_items_with_odd_units(B):
    """A call large enough for items of two 32-row units (more than 64 chunks
    of 32 rows x 512 weights per SM), whose GEMVs have an odd number of units
    and ragged rows, so the last item of a GEMV holds one unit; items are cut
    between warps at many places.  Every output against the oracle, through the
    in-kernel re-order (one grouped call) and the re-order launch (prepare + run)."""
    shapes = [(4000, 8192), (1000, 8192), (33, 8192), (4064, 4096), (1, 8192), (2100, 8192),
              (4000, 8192), (999, 2048)] * 2
    items, refs = [], []
    for li, (N, K) in enumerate(shapes):
        codes, scales = oracle.pack(synth.latent_weights(N, K, seed=500 + li))
        x = synth.int8_uniform((B, K), seed=600 + li)
        items.append((dev_codes(codes), dev(scales), dev(x),
                      torch.zeros((B, N), dtype=torch.float32, device="cuda")))
        refs.append(oracle.gemv(codes, scales, x, K))
    chunks = sum((N + 31) // 32 * (K // 512) for N, K in shapes)
    assert chunks > 64 * torch.cuda.get_device_properties(0).multi_processor_count
    g = S.GroupedGemv(items, B=B)
    for run in (g, lambda: (g.prepare(), g.run())):
        for it in items:
            it[3].fill_(float("nan"))
        run()
        torch.cuda.synchronize()
        for (_, _, _, y), ref in zip(items, refs):
            assert_y_matches(y.cpu().numpy(), ref)


def test_gemv_full_size_decode_stack_as_benched():
    """The benchmark's launch: the 16-layer 1B stack, 112 GEMVs at B = 1, one
    re-order launch and one GEMV launch (one grouped call, and prepare + run),
    on random code words (every word pattern is a valid code) and random
    scales; every output of every GEMV against the oracle, bit for bit."""
    rng = np.random.default_rng(2024)
    xs = {2048: synth.int8_uniform((1, 2048), seed=1), 8192: synth.int8_uniform((1, 8192), seed=2)}
    xd = {k: dev(v) for k, v in xs.items()}
    items, host = [], []
    for _, _, N, K, _ in synth.decode_stack(16):
        codes = rng.integers(0, 2 ** 32, size=((N + 31) // 32, K // 128, 5, 32),
                             dtype=np.uint64).astype(np.uint32)
        scales = (rng.random(N) * 0.05 + 1e-3).astype(np.float32)
        y = torch.empty((1, N), dtype=torch.float32, device="cuda")
        items.append((dev_codes(codes), dev(scales), xd[K], y))
        host.append((codes, scales, K))
    g = S.GroupedGemv(items, B=1)
    refs = [oracle.gemv(codes, scales, xs[K], K) for codes, scales, K in host]
    for run in (g, lambda: (g.prepare(), g.run())):
        for it in items:
            it[3].fill_(float("nan"))
        run()
        torch.cuda.synchronize()
        for ref, it in zip(refs, items):
            assert_y_matches(it[3].cpu().numpy(), ref)
    assert S.device_error() == 0


def test_gemv_on_gpu_packed_codes():
    # end to end on the device: pack on the GPU, then GEMV
    N, K = 2048, 2048
    w = synth.latent_weights(N, K, seed=0)
    codes, scales = S.pack(dev(w))
    x = synth.int8_uniform((1, K), seed=1)
    y = S.gemv(codes, scales, dev(x)).cpu().numpy()
    c_ref, s_ref = oracle.pack(w)
    acc_ref = oracle.gemv_acc(c_ref, x, N, K)
    y_ref = scales.cpu().numpy().astype(np.float64)[None, :] * acc_ref
    assert_y_matches(y, y_ref)


# ----------------------------------------------------------------------------- gemm
GEMM_CASES = [(1, 128, 128), (100, 200, 384), (256, 128, 128), (300, 256, 640),
              (513, 129, 1152), (64, 1000, 256), (1024, 384, 2048)]


@pytest.mark.parametrize("M,N,K", GEMM_CASES)
def test_gemm_matches_oracle(M, N, K):
    codes, scales = oracle.pack(synth.latent_weights(N, K, seed=0))
    x = synth.int8_clipped_normal((M, K), seed=1)
    tc, ts, tx = dev_codes(codes), dev(scales), dev(x)
    acc = S.gemm_acc(tc, tx, N)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), oracle.gemm_acc(codes, x, N, K))
    y = S.gemm(tc, ts, tx)
    assert_y_matches(y.cpu().numpy(), oracle.gemm(codes, scales, x, K))


def test_gemm_random_words_full_int8_range():
    rng = np.random.default_rng(11)
    M, N, K = 200, 160, 768
    codes = rng.integers(0, 2 ** 32, size=((N + 31) // 32, K // 128, 5, 32),
                         dtype=np.uint64).astype(np.uint32)
    x = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
    acc = S.gemm_acc(dev_codes(codes), dev(x), N)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), oracle.gemm_acc(codes, x, N, K))


@pytest.mark.parametrize("case", synth.PREFILL_GEMMS, ids=lambda c: c[0])
def test_gemm_full_size_prefill(case):
    _, M, N, K = case
    codes, scales = oracle.pack(synth.latent_weights(N, K, seed=0))
    x = synth.int8_clipped_normal((M, K), seed=1)
    y = S.gemm(dev_codes(codes), dev(scales), dev(x)).cpu().numpy()
    # every output: the oracle takes a few seconds on all host cores per shape
    assert_y_matches(y, oracle.gemm(codes, scales, x, K))


@pytest.mark.parametrize("N,K,B", [(256, 1024, 1), (96, 2048, 2), (320, 4096, 3)])
def test_pack_then_gemv_back_to_back_on_one_stream(N, K, B):
    """The GEMV right after the kernel that wrote its codes, with no host
    synchronisation: small calls (the first two shapes) skip the re-order
    launch, so the pack kernel is the GEMV launch's direct predecessor and the
    GEMV must read the codes only after its grid-dependency wait."""
    w1, w2 = synth.latent_weights(N, K, seed=41), synth.latent_weights(N, K, seed=42)
    x = synth.int8_uniform((B, K), seed=43)
    c1, _ = oracle.pack(w1)
    c2, _ = oracle.pack(w2)
    tw1, tw2, tx = dev(w1), dev(w2), dev(x)
    codes = torch.zeros(S.codes_shape(N, K), dtype=torch.int32, device="cuda")
    sc1 = torch.zeros(N, dtype=torch.float32, device="cuda")
    sc2 = torch.zeros_like(sc1)
    ws = S.workspace(S.gemv_workspace_bytes(N, K, B), torch.device("cuda"))
    y1 = torch.empty((B, N), dtype=torch.float32, device="cuda")
    y2 = torch.empty_like(y1)
    torch.cuda.synchronize()
    for tw, sc, y in ((tw1, sc1, y1), (tw2, sc2, y2)):   # the second pack overwrites the codes
        S.pack(tw, codes, sc)
        S.gemv(codes, sc, tx, y, ws)
    torch.cuda.synchronize()
    for c, sc, y in ((c1, sc1, y1), (c2, sc2, y2)):
        # y against the oracle's dot products with the scales the GPU wrote, so
        # that only the codes each GEMV read decide the comparison
        assert_y_matches(y.cpu().numpy(), oracle.gemv(c, sc.cpu().numpy(), x, K))


def test_gemm_m1_equals_gemv():
    N, K = 384, 1024
    codes, scales = oracle.pack(synth.latent_weights(N, K, seed=5))
    x = synth.int8_uniform((1, K), seed=6)
    tc, ts, tx = dev_codes(codes), dev(scales), dev(x)
    assert torch.equal(S.gemm(tc, ts, tx), S.gemv(tc, ts, tx))


def test_gemv_prepare_then_run_equals_grouped():
    items, refs = [], []
    for li, (N, K) in enumerate([(64, 2048), (48, 8192), (100, 384)]):
        codes, scales = oracle.pack(synth.latent_weights(N, K, seed=40 + li))
        x = synth.int8_uniform((3, K), seed=50 + li)
        y = torch.zeros((3, N), dtype=torch.float32, device="cuda")
        items.append((dev_codes(codes), dev(scales), dev(x), y))
        refs.append(oracle.gemv(codes, scales, x, K))
    g = S.GroupedGemv(items, B=3)
    g.prepare()
    g.run()
    for (_, _, _, y), ref in zip(items, refs):
        assert_y_matches(y.cpu().numpy(), ref)
    for it in items:
        it[3].zero_()
    g()
    for (_, _, _, y), ref in zip(items, refs):
        assert_y_matches(y.cpu().numpy(), ref)


def test_gemv_run_repeats_after_one_prepare():
    # K-parts meet in the workspace; every run must leave it ready for the next
    items, refs = [], []
    for li, (N, K) in enumerate([(96, 8192), (70, 3072), (33, 2048), (48, 12288), (40, 17408)]):
        codes, scales = oracle.pack(synth.latent_weights(N, K, seed=60 + li))
        x = synth.int8_uniform((2, K), seed=70 + li)
        y = torch.zeros((2, N), dtype=torch.float32, device="cuda")
        items.append((dev_codes(codes), dev(scales), dev(x), y))
        refs.append(oracle.gemv(codes, scales, x, K))
    g = S.GroupedGemv(items, B=2)
    g.prepare()
    for _ in range(3):
        for it in items:
            it[3].zero_()
        g.run()
        for (_, _, _, y), ref in zip(items, refs):
            assert_y_matches(y.cpu().numpy(), ref)


@pytest.mark.parametrize("B", [1, 2])
def test_gemv_in_kernel_reorder_equals_reorder_launch(B):
    """Small int8 calls re-order x inside the dot kernel (no re-order launch);
    the split prepare/run calls and an x that is only 4-byte aligned take the
    re-order launch.  All three give the oracle's y bit for bit."""
    for li, (N, K) in enumerate([(2048, 2048), (512, 2048), (33, 8192), (100, 1024), (1, 512)]):
        codes, scales = oracle.pack(synth.latent_weights(N, K, seed=80 + li))
        x = synth.int8_uniform((B, K), seed=90 + li)
        ref = oracle.gemv(codes, scales, x, K)
        tc, ts = dev_codes(codes), dev(scales)
        tx = dev(x)
        assert_y_matches(S.gemv(tc, ts, tx).cpu().numpy(), ref)            # in-kernel re-order
        y = torch.zeros((B, N), dtype=torch.float32, device="cuda")
        g = S.GroupedGemv([(tc, ts, tx, y)], B=B)
        g.prepare()
        g.run()                                                             # re-order launch
        assert_y_matches(y.cpu().numpy(), ref)
        buf = torch.zeros(B * K + 4, dtype=torch.int8, device="cuda")
        xo = buf[4:].view(B, K)                                             # 4-byte aligned only
        xo.copy_(tx)
        assert_y_matches(S.gemv(tc, ts, xo).cpu().numpy(), ref)


@pytest.mark.parametrize("B", [3, 16])
def test_gemv_grouped_shared_activations(B):
    """GEMVs of one grouped call that share an activation tensor (q, k, v and
    gate, up of a layer do) re-use one re-ordered copy of it; the same pointer
    with another K (a prefix view) is a different activation and is prepared on
    its own.  Shares in mixed order, one split-K row among them (whose partial
    sums are still cleared), every output against the oracle; then the same
    items through prepare + run, which prepares every GEMV's own copy."""
    cuda = torch.device("cuda")
    xa = synth.int8_uniform((B, 3072), seed=901)
    xb = synth.int8_uniform((B, 10752), seed=902)
    xa_d, xb_d = dev(xa), dev(xb)
    xa_pre = xa_d[:, :1024]                       # same pointer as xa_d, K = 1024 (strided rows)
    xa_pre_c = xa_pre.contiguous()
    spec = [(96, 3072, xa_d, xa), (64, 10752, xb_d, xb), (33, 3072, xa_d, xa),
            (70, 1024, xa_pre_c, np.ascontiguousarray(xa[:, :1024])), (128, 3072, xa_d, xa),
            (40, 10752, xb_d, xb)]
    items, refs = [], []
    for i, (n, k, xt, xh) in enumerate(spec):
        codes, scales = oracle.pack(synth.latent_weights(n, k, seed=910 + i))
        items.append((dev_codes(codes), dev(scales), xt,
                      torch.full((B, n), float("nan"), dtype=torch.float32, device=cuda)))
        refs.append(oracle.gemv(codes, scales, xh, k))
    S.gemv_grouped(items, B=B)
    torch.cuda.synchronize()
    for (_, _, _, y), ref in zip(items, refs):
        assert_y_matches(y.cpu().numpy(), ref)
    g = S.GroupedGemv(items, B=B)
    for _ in range(2):
        for it in items:
            it[3].fill_(float("nan"))
        g.prepare()
        g.run()
        torch.cuda.synchronize()
        for (_, _, _, y), ref in zip(items, refs):
            assert_y_matches(y.cpu().numpy(), ref)
    assert S.device_error() == 0


# ----------------------------------------------------------------------------- limits
def _one_sign_rows(N, K, seed):
    """Latent rows whose kept weights all share a sign in rows 0 (+) and 1 (-):
    against an all -128 activation row such a row's accumulator is
    -/+ 128 * 3K/4, the largest magnitude the format allows (12,582,912 at
    K = 131072, below 2^24, so s * acc is still one fp32 rounding)."""
    w = synth.latent_weights(N, K, seed=seed)
    w[0] = np.abs(w[0]) + 1e-3
    w[1] = -np.abs(w[1]) - 1e-3
    return w


def _extreme_x(B, K, seed):
    x = synth.int8_uniform((B, K), seed=seed)
    x[0] = -128
    if B > 1:
        x[1] = 127
    return x


@pytest.mark.parametrize("B", [1, 2, 5, 16])
def test_gemv_largest_k_and_accumulator(B):
    """K = SHERRY_MAX_K (131072: 1,024 tiles, 16 K-parts of 8,192) with a
    ragged last row group, on each kernel: the dot kernel (B <= 2) and the MMA
    kernel with both activation group sizes and both batch-group counts."""
    N, K = 40, 131072
    codes, scales = oracle.pack(_one_sign_rows(N, K, seed=120))
    x = _extreme_x(B, K, seed=121)
    tc, ts, tx = dev_codes(codes), dev(scales), dev(x)
    acc_ref = oracle.gemv_acc(codes, x, N, K)
    assert acc_ref[0, 0] == -128 * 3 * K // 4 and acc_ref[0, 1] == 128 * 3 * K // 4
    acc = S.gemv_acc(tc, tx, N)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), acc_ref)
    assert_y_matches(S.gemv(tc, ts, tx).cpu().numpy(), oracle.gemv(codes, scales, x, K))


def test_gemm_largest_k_and_accumulator():
    """The GEMM at K = 131072 (1,024 stages through the 4-stage ring of one
    CTA) with a token tail and a ragged weight tile, every output."""
    M, N, K = 130, 40, 131072
    codes, scales = oracle.pack(_one_sign_rows(N, K, seed=122))
    x = _extreme_x(M, K, seed=123)
    tc, ts, tx = dev_codes(codes), dev(scales), dev(x)
    acc_ref = oracle.gemm_acc(codes, x, N, K)
    assert acc_ref[0, 0] == -128 * 3 * K // 4
    assert np.array_equal(S.gemm_acc(tc, tx, N).cpu().numpy().astype(np.int64), acc_ref)
    assert_y_matches(S.gemm(tc, ts, tx).cpu().numpy(), oracle.gemm(codes, scales, x, K))


@pytest.mark.parametrize("N", [1, 33])
def test_pack_largest_k(N):
    """Rows of 131072 weights: several warps per row, their double partial
    sums of |w| combined into one scale."""
    K = 131072
    w = synth.latent_weights(N, K, seed=124)
    codes_ref, scales_ref = oracle.pack(w)
    codes, scales = S.pack(dev(w))
    torch.cuda.synchronize()
    assert np.array_equal(host_codes(codes), codes_ref)
    assert ulp_diff_f32(scales.cpu().numpy(), scales_ref).max() <= 1
