"""Pins of the CPU oracle against what the pages and the mathematics fix.

The pages (arXiv 2601.07892, abstract and Figure 2 caption) fix: ternary
weights, exactly one zero per block of four (3:4), four weights in five bits
(1.25 bits/weight), against 2-bit and 1.67-bit (3 weights in 5 bits) packing.
They print no worked example, so the expected values here are hand-derived
from the written layout (tests/golden), closed forms, invariants, and brute
force against numpy's dense int64 matmul on matrices built with a known
prune.  None of these recompute the oracle's own code path.
"""
import os

import numpy as np
import pytest

import oracle
import synth
from tests.helpers import (VALID_BLOCKS, load_tiles, random_ternary, ternary_latents,
                           ulp_diff_f32)


def test_code_space_is_exactly_32_blocks():
    # 4 zero positions x 2^3 sign patterns = 32 = 2^5 (four weights in five bits).
    assert len(VALID_BLOCKS) == 32 == 2 ** 5
    seen = set()
    for c in range(32):
        w = tuple(int(v) for v in oracle.code_weights(c))
        assert w.count(0) == 1 and all(v in (-1, 1) for v in w if v != 0)
        seen.add(w)
        p = w.index(0)
        neg = [1 if v < 0 else 0 for i, v in enumerate(w) if i != p]
        assert oracle.block_code(p, neg) == c
    assert seen == set(VALID_BLOCKS)


@pytest.mark.parametrize("code,expected", [
    (0, (0, 1, 1, 1)), (1, (1, 0, 1, 1)), (2, (1, 1, 0, 1)), (3, (1, 1, 1, 0)),
    (7, (-1, 1, 1, 0)), (30, (-1, -1, 0, -1)), (17, (1, 0, 1, -1)), (12, (0, -1, -1, 1)),
])
def test_code_examples(code, expected):
    # c = p | s0<<2 | s1<<3 | s2<<4, signs of the kept weights in ascending position.
    assert tuple(int(v) for v in oracle.code_weights(code)) == expected


def test_prune_cases(golden_dir):
    with open(os.path.join(golden_dir, "prune_cases.txt")) as f:
        lines = [ln for ln in f if ln.strip() and not ln.startswith("#")]
    assert len(lines) >= 10
    for ln in lines:
        lhs, rhs = ln.split("|")
        w = np.array([float(v) for v in lhs.split()], np.float32)
        exp = [int(v) for v in rhs.split()]
        p, neg = oracle.prune_block(w)
        assert [p] + neg == exp, ln


def test_golden_tiles(golden_dir):
    for t in load_tiles(golden_dir):
        codes, scales = oracle.pack(t["latent"].reshape(1, 128))
        assert codes.shape == (1, 1, 5, 32)
        got = [int(codes[0, 0, p, 0]) for p in range(5)]
        assert got == t["words"], (t["name"], [hex(v) for v in got])
        assert not codes[0, 0, :, 1:].any()          # padding rows 1..31 are zero
        assert scales[0] == t["scale"], (t["name"], scales[0], t["scale"])
        assert np.array_equal(oracle.unpack(codes, 1, 128)[0], t["dense"]), t["name"]


def test_golden_words_unpack_without_pack(golden_dir):
    # Unpack and dot straight from the hand-derived words (no pack involved).
    for t in load_tiles(golden_dir):
        codes = np.zeros((1, 1, 5, 32), np.uint32)
        codes[0, 0, :, 0] = t["words"]
        assert np.array_equal(oracle.unpack(codes, 1, 128)[0], t["dense"]), t["name"]
        x = synth.int8_uniform((3, 128), seed=11)
        acc = oracle.gemv_acc(codes, x, 1, 128)
        assert np.array_equal(acc[:, 0], x.astype(np.int64) @ t["dense"].astype(np.int64))


def test_blocked_layout_across_rows_and_tiles(golden_dir):
    tiles = {t["name"][0]: t for t in load_tiles(golden_dir)}
    # row 0 = [A | B], row 1 = [C | E], row 2 = [G | F]
    rows = [("A", "B"), ("C", "E"), ("G", "F")]
    lat = np.stack([np.concatenate([tiles[a]["latent"], tiles[b]["latent"]]) for a, b in rows])
    codes, scales = oracle.pack(lat)
    assert codes.shape == (1, 2, 5, 32)
    flat = codes.reshape(-1)
    # word (plane p, row n, tile t) sits at ((n // 32) * T + t) * 160 + 32 p + n % 32;
    # hand-computed positions (T = 2):
    assert flat[1 * 160 + 2 * 32 + 0] == tiles["B"]["words"][2]    # row 0, tile 1, S0 of B
    assert flat[0 * 160 + 3 * 32 + 2] == tiles["G"]["words"][3]    # row 2, tile 0, S1 of G
    assert flat[0 * 160 + 0 * 32 + 1] == tiles["C"]["words"][0]    # row 1, tile 0, Z0 of C
    assert flat[1 * 160 + 1 * 32 + 1] == tiles["E"]["words"][1]    # row 1, tile 1, Z1 of E
    assert flat[1 * 160 + 4 * 32 + 2] == tiles["F"]["words"][4]    # row 2, tile 1, S2 of F
    for n, pair in enumerate(rows):
        for t, name in enumerate(pair):
            for p in range(5):
                assert codes[0, t, p, n] == tiles[name]["words"][p]
    assert not codes[0, :, :, 3:].any()                            # padding rows
    # second group: row 35 of a 40-row matrix sits in group 1 at position 3
    lat2 = np.zeros((40, 256), np.float32)
    lat2[35] = np.concatenate([tiles["D"]["latent"], tiles["C"]["latent"]])
    c2, _ = oracle.pack(lat2)
    f2 = c2.reshape(-1)
    assert c2.shape == (2, 2, 5, 32)
    assert f2[(1 * 2 + 0) * 160 + 1 * 32 + 3] == tiles["D"]["words"][1]   # Z1 of D
    assert f2[(1 * 2 + 1) * 160 + 2 * 32 + 3] == tiles["C"]["words"][2]   # S0 of C
    # mean over 192 kept weights: [A|B] = (96*1 + 96*2)/192 = 1.5
    assert scales[0] == np.float32(1.5)
    assert scales[1] == np.float32((96 * 2 + 96 * 3) / 192)
    assert scales[2] == np.float32((64 + 56) / 192)


def test_all_32_codes_in_one_tile():
    rng = np.random.default_rng(5)
    T = np.array(VALID_BLOCKS, np.int8).reshape(1, 128)   # block j = pattern j
    lat = ternary_latents(T, rng)
    codes, _ = oracle.pack(lat)
    assert np.array_equal(oracle.unpack(codes, 1, 128), T)


def test_random_words_decode_to_valid_blocks():
    # Every 5-bit pattern is a valid block: any words unpack to exactly one zero per block.
    rng = np.random.default_rng(7)
    codes = rng.integers(0, 2 ** 32, size=(1, 3, 5, 32), dtype=np.uint64).astype(np.uint32)
    wt = oracle.unpack(codes, 7, 384).reshape(7, 96, 4)
    assert np.all((wt == 0).sum(axis=2) == 1)
    assert np.all(np.isin(wt, (-1, 0, 1)))


def test_pack_unpack_roundtrip_and_scale():
    rng = np.random.default_rng(3)
    for N, K in [(1, 128), (9, 384), (4, 1024)]:
        T = random_ternary(N, K, rng)
        lat = ternary_latents(T, rng)
        codes, scales = oracle.pack(lat)
        assert np.array_equal(oracle.unpack(codes, N, K), T)
        kept_mean = np.where(T != 0, np.abs(lat.astype(np.float64)), 0).sum(1) / (0.75 * K)
        assert np.all(ulp_diff_f32(scales, kept_mean.astype(np.float32)) <= 1)


def test_constant_magnitude_rows_have_exact_scale():
    rng = np.random.default_rng(9)
    for a in (0.02, 1.0 / 3.0, 7.5e-3, 1e-20):
        a32 = np.float32(a)
        lat = (rng.choice([-1, 1], size=(3, 512)) * a32).astype(np.float32)
        _, s = oracle.pack(lat)
        assert np.all(s == a32)


def test_zero_rows_and_zero_activations():
    lat = np.zeros((2, 256), np.float32)
    codes, s = oracle.pack(lat)
    assert np.all(s == 0.0)
    x = synth.int8_uniform((2, 256), seed=4)
    assert np.all(oracle.gemv(codes, s, x, 256) == 0.0)
    lat = synth.latent_weights(5, 256, seed=2)
    codes, s = oracle.pack(lat)
    assert np.all(oracle.gemv(codes, s, np.zeros((1, 256), np.int8), 256) == 0.0)


def test_all_ones_activation_gives_sum_of_signs():
    N, K = 33, 640
    lat = synth.latent_weights(N, K, seed=0)
    codes, _ = oracle.pack(lat)
    acc = oracle.gemv_acc(codes, np.ones((1, K), np.int8), N, K)[0]
    neg = np.array([sum(bin(int(w)).count("1") for w in codes[n // 32, :, 2:, n % 32].reshape(-1))
                    for n in range(N)])
    assert np.array_equal(acc, 3 * K // 4 - 2 * neg)


@pytest.mark.parametrize("N", [1, 3, 17])
@pytest.mark.parametrize("K", [128, 256, 640])
@pytest.mark.parametrize("B", [1, 2, 5])
def test_bruteforce_dense_matmul(N, K, B):
    rng = np.random.default_rng(N * 1000 + K + B)
    T = random_ternary(N, K, rng)
    lat = ternary_latents(T, rng)
    codes, scales = oracle.pack(lat)
    x = rng.integers(-128, 128, size=(B, K)).astype(np.int8)
    ref = x.astype(np.int64) @ T.astype(np.int64).T
    assert np.array_equal(oracle.gemv_acc(codes, x, N, K), ref)
    assert np.array_equal(oracle.gemm_acc(codes, x, N, K), ref)
    y = oracle.gemv(codes, scales, x, K)
    assert np.array_equal(y, scales.astype(np.float64)[None, :] * ref)
    assert np.array_equal(oracle.gemm(codes, scales, x, K), y)


def test_extreme_activations_bound():
    # |acc| <= (3K/4) * 128: all kept weights aligned with x = -128 / +127.
    K = 1024
    T = np.tile(np.array([1, 1, 1, 0], np.int8), (2, K // 4))
    T[1] *= -1
    lat = ternary_latents(T, np.random.default_rng(0))
    codes, _ = oracle.pack(lat)
    x = np.full((2, K), -128, np.int8)
    x[1] = 127
    acc = oracle.gemv_acc(codes, x, 2, K)
    assert acc[0, 0] == -128 * 3 * K // 4 and acc[0, 1] == 128 * 3 * K // 4
    assert acc[1, 0] == 127 * 3 * K // 4 and acc[1, 1] == -127 * 3 * K // 4


def test_size_closed_forms():
    for N, K in [(32, 128), (256, 1024), (2048, 8192), (8192, 2048)]:
        nbytes = oracle.packed_bytes(N, K)
        assert nbytes * 32 == N * K * 5          # 5 bits per 4 weights
        assert 8 * nbytes / (N * K) == 1.25      # 1.25 bits per weight (scales excluded)
    assert oracle.packed_bytes(1, 128) == 32 * 20    # one 32-row group of one tile
    assert oracle.packed_bytes(33, 256) == 64 * 2 * 20
    assert 1 - 1.25 / (5 / 3) == pytest.approx(0.25, abs=1e-15)   # vs 3-in-5-bit packing
    assert 1 - 1.25 / 2 == 0.375                                  # vs 2-bit packing
    assert oracle.packed_bytes(4, 100) == -1


def test_bad_shapes_rejected():
    with pytest.raises(Exception):
        oracle.pack(np.zeros((2, 100), np.float32))


# ---------------------------------------------------------------------------
# Activation front-end (int8 activations of the W1.25A8 setting; the rule is
# the reading stated in the oracle: per-token absmax, s = amax / 127,
# q = clamp(rint(x * (127 / amax)), -127, 127) in fp32, ties to even).
# Expected values below are derived by hand.
# ---------------------------------------------------------------------------
def test_quantize_act_hand_cases():
    # amax = 127: s = 1 and 127 / amax = 1, so q = rint(x) with ties to even
    q, s = oracle.quantize_act(oracle.bf16_bits([127.0, 1.0, -0.5, 0.25, -127.0, 63.5, 0.0, 126.5]))
    assert s.tolist() == [1.0]
    assert q.tolist() == [[127, 1, 0, 0, -127, 64, 0, 126]]
    # amax = 2: 127 / 2 = 63.5 exactly; 1.0 -> 63.5 -> 64 (even), 0.5 -> 31.75 -> 32,
    # 2^-6 -> 0.9921875 -> 1; s = fl32(2 / 127)
    q, s = oracle.quantize_act(oracle.bf16_bits([2.0, 1.0, -1.0, 0.5, 0.015625, -2.0, 0.0, -0.75]))
    assert s[0] == np.float32(2.0) / np.float32(127.0)
    assert q.tolist() == [[127, 64, -64, 32, 1, -127, 0, -48]]   # -0.75 * 63.5 = -47.625 -> -48
    # an all-zero row
    q, s = oracle.quantize_act(np.zeros((1, 16), np.uint16))
    assert s.tolist() == [0.0] and not q.any()


def test_quantize_act_bounds_on_random_rows():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((6, 384)).astype(np.float32) * np.array([1, 1e-3, 10, 1e4, 0.5, 3],
                                                                    np.float32)[:, None]
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)          # truncate to bf16
    xb = (bits.astype(np.uint32) << 16).view(np.float32)
    q, s = oracle.quantize_act(bits)
    amax = np.abs(xb).max(axis=1)
    assert np.array_equal(s, (amax / np.float32(127.0)).astype(np.float32))
    assert np.abs(q.astype(np.int32)).max() <= 127
    for b in range(6):
        k = np.argmax(np.abs(xb[b]))
        assert abs(int(q[b, k])) == 127 and np.sign(q[b, k]) == np.sign(xb[b, k])
        # dequantisation error: at most half a step (plus fp32 rounding of x * inv)
        err = np.abs(q[b].astype(np.float64) * float(s[b]) - xb[b].astype(np.float64))
        assert err.max() <= 0.5 * float(s[b]) * (1 + 1e-5)


def test_gemv_act_equals_scaled_bruteforce():
    N, K, B = 21, 384, 3
    codes, scales = oracle.pack(synth.latent_weights(N, K, seed=8))
    wt = oracle.unpack(codes, N, K).astype(np.int64)
    rng = np.random.default_rng(9)
    x = rng.standard_normal((B, K)).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    q, sx = oracle.quantize_act(bits)
    acc = q.astype(np.int64) @ wt.T
    ref = scales.astype(np.float64)[None, :] * sx.astype(np.float64)[:, None] * acc
    assert np.array_equal(oracle.gemv_act(codes, scales, q, sx, K), ref)


# ---------------------------------------------------------------------------
# Front-end on fp32 activations (re-quantization of a GEMV's y for the next
# layer): the per-token rule above, read from fp32 values.  Expected values
# are derived by hand.
# ---------------------------------------------------------------------------
def test_quantize_f32_hand_cases():
    # amax = 1: 127 / 1 = 127 and s = fl32(1 / 127).  -0.5 -> -63.5 -> -64
    # (ties to even); 0.25 -> 31.75 -> 32; fl32(0.3) * 127 = 38.100002 -> 38;
    # 0.99999994 (the float below 1) -> 126.99999 -> 127.  0.7441181 is read
    # as fp32: 0.7441181 * 127 = 94.503 -> 95, where a bf16 copy of it
    # (0.7421875, rounded or truncated) would give 94.26 -> 94.
    x = np.array([[1.0, 0.99999994, -0.5, 0.25, 0.0, -1.0, 0.3, 0.7441181]], np.float32)
    q, s = oracle.quantize_f32(x)
    assert s[0] == np.float32(1.0) / np.float32(127.0)
    assert q.tolist() == [[127, 127, -64, 32, 0, -127, 38, 95]]
    # amax = 254 (second row): 127 / 254 = 0.5 exactly; 3.0 -> 1.5 -> 2,
    # 5.0 -> 2.5 -> 2, -7.0 -> -3.5 -> -4; s = 2
    q, s = oracle.quantize_f32(np.array([[3.0, 5.0, -7.0, 254.0], [0.0, 0.0, 0.0, 0.0]], np.float32))
    assert s.tolist() == [2.0, 0.0]
    assert q.tolist() == [[2, 2, -4, 127], [0, 0, 0, 0]]


def test_quantize_f32_bounds_on_random_rows():
    rng = np.random.default_rng(15)
    x = rng.standard_normal((6, 384)).astype(np.float32) * np.array([1, 1e-3, 10, 1e4, 0.5, 3],
                                                                    np.float32)[:, None]
    q, s = oracle.quantize_f32(x)
    amax = np.abs(x).max(axis=1)
    assert np.array_equal(s, (amax / np.float32(127.0)).astype(np.float32))
    assert np.abs(q.astype(np.int32)).max() <= 127
    for b in range(6):
        k = np.argmax(np.abs(x[b]))
        assert abs(int(q[b, k])) == 127 and np.sign(q[b, k]) == np.sign(x[b, k])
        err = np.abs(q[b].astype(np.float64) * float(s[b]) - x[b].astype(np.float64))
        assert err.max() <= 0.5 * float(s[b]) * (1 + 1e-5)


# ---------------------------------------------------------------------------
# SwiGLU h = silu(g) * u, silu(g) = g / (1 + e^-g): closed forms of the
# logistic function and the known minimum of silu.
# ---------------------------------------------------------------------------
def test_swiglu_closed_forms():
    # silu(0) = 0; e^-ln3 = 1/3, so silu(ln 3) = (3/4) ln 3 (to fp32 rounding of
    # ln 3, whose effect on the logistic factor is below 2e-8)
    ln3 = np.float32(np.log(3.0))
    g = np.array([0.0, ln3, ln3, -ln3, 40.0, -40.0, 2.0], np.float32)
    u = np.array([5.0, 1.0, -2.0, 1.0, -3.0, 1.0, 0.0], np.float32)
    h = oracle.swiglu(g, u).astype(np.float64)
    assert h[0] == 0.0 and h[6] == 0.0
    assert abs(h[1] - 0.75 * float(ln3)) <= 2e-7 * abs(h[1])
    assert abs(h[2] + 1.5 * float(ln3)) <= 2e-7 * abs(h[2])
    # silu(-g) = -g * e^-g / (1 + e^-g): at -ln 3 the factor is 1/4
    assert abs(h[3] + 0.25 * float(ln3)) <= 2e-7 * abs(h[3])
    # far tails: silu(40) = 40 to fp32; silu(-40) = -40 e^-40 / (1 + e^-40)
    assert h[4] == -120.0
    assert abs(h[5] + 40.0 * np.exp(-40.0)) <= 1e-6 * 40.0 * np.exp(-40.0)
    # odd part: silu(g) - silu(-g) = g, since the logistic function satisfies
    # sigma(g) + sigma(-g) = 1
    rng = np.random.default_rng(21)
    gr = (rng.standard_normal(4096) * 4).astype(np.float32)
    one = np.ones_like(gr)
    d = oracle.swiglu(gr, one).astype(np.float64) - oracle.swiglu(-gr, one).astype(np.float64)
    assert np.all(np.abs(d - gr.astype(np.float64)) <= 2.4e-7 * np.maximum(np.abs(gr), 1.0))


def test_swiglu_minimum_is_lambert_w():
    # d/dg [g sigma(g)] = 0  <=>  e^g (g + 1) = -1  <=>  g* = -1 - W(1/e), and
    # there silu(g*) = g* + 1 = -W(1/e)  (W: Lambert's W, principal branch)
    from scipy.special import lambertw
    w = float(lambertw(np.exp(-1.0)).real)
    gs = np.float32(-1.0 - w)
    g = np.array([gs, gs - np.float32(0.05), gs + np.float32(0.05)], np.float32)
    h = oracle.swiglu(g, np.ones(3, np.float32)).astype(np.float64)
    assert abs(h[0] + w) <= 1e-6
    assert h[1] > h[0] and h[2] > h[0]
