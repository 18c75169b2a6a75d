"""Pins of the oracle's comparison formats (no GPU).

The pages set Sherry's 1.25 bits per weight against a 2-bit aligned ternary
packing and a 1.67-bit packing of three weights in five bits ("Sherry:
Hardware-Efficient 1.25-Bit Ternary Quantization via Fine-grained
Sparsification", arXiv 2601.07892, abstract; Figure 2 caption).  The oracle's
encoders for both are pinned here by hand-derived words, the closed-form
sizes, exhaustive code tables, round trips, and the fact that all three
formats hold the same ternary matrix, so the dot products agree with Sherry's
oracle and with a dense brute force.  Planted mistakes in a copy of the oracle
source must each fail one of these pins.
"""
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle
import oracle.oracle as oracle_mod
import synth

I2, T3 = oracle.FMT_I2, oracle.FMT_T3
SRC = os.path.join(os.path.dirname(oracle_mod.__file__), "sherry_oracle.c")


def test_sizes_closed_forms():
    # 2 bits per weight: 32 rows x 1024 weights -> 8192 bytes
    assert oracle.cmp_packed_bytes(I2, 32, 1024) == 32 * 1024 * 2 // 8 == 8192
    # three weights in five bits: 1920 = 10 x 192 weights per row, no padding
    assert oracle.cmp_tiles(T3, 1920) == 20
    assert oracle.cmp_packed_bytes(T3, 32, 1920) == 32 * 1920 * 5 // 3 // 8 == 12800
    # rows padded to whole 32-row groups, as for Sherry
    assert oracle.cmp_packed_bytes(I2, 33, 128) == 64 * 128 * 2 // 8
    # T3 pads a row to an even number of 96-weight tiles: K = 2048 -> 22 tiles
    assert oracle.cmp_tiles(T3, 2048) == 22 and oracle.cmp_tiles(T3, 8192) == 86
    # 1024 weights: 10.67 tiles of 96, i.e. 5.33 pairs -> 6 pairs = 12 tiles (1152 weights)
    assert oracle.cmp_tiles(T3, 1024) == 12
    # Sherry against the two: 37.5 % and 25 % fewer bits at these sizes
    sherry = oracle.packed_bytes(32, 1920 * 2)   # K a multiple of 128 and of 192: 3840
    assert oracle.cmp_packed_bytes(I2, 32, 3840) * 5 == sherry * 8
    assert oracle.cmp_packed_bytes(T3, 32, 3840) * 3 == sherry * 4
    assert oracle.cmp_tiles(I2, 100) == 0 and oracle.cmp_packed_bytes(7, 32, 128) == -1


def test_i2_hand_word():
    # word 0 of a tile holds weights 0..15; nibble n = weight n (low two bits)
    # and weight n + 8 (high two bits); codes 0 -> 0, 1 -> +1, 3 -> -1.
    row = np.zeros((1, 128), np.int8)
    row[0, [0, 4, 15]] = 1
    row[0, [1, 8]] = -1
    c = oracle.cmp_encode(I2, row)
    # w0 = +1 -> 0x1; w1 = -1 -> 0x3 << 4; w4 = +1 -> 1 << 16; w8 = -1 -> 0x3 << 2;
    # w15 = +1 -> 1 << (4 * 7 + 2)
    assert c[0, 0, 0, 0] == 0x4001003D
    assert not c[0, 0, 1:, 0].any() and not c[0, 0, :, 1:].any()
    # a weight in word 5 (k = 80 + 9): nibble 1, high half
    row2 = np.zeros((1, 128), np.int8)
    row2[0, 89] = -1
    c2 = oracle.cmp_encode(I2, row2)
    assert c2[0, 0, 5, 0] == 0x3 << 6


def test_t3_code_table_is_exhaustive():
    seen = set()
    for a in (-1, 0, 1):
        for b in (-1, 0, 1):
            for c in (-1, 0, 1):
                code = oracle.t3_code([a, b, c])
                assert 0 <= code <= 26
                seen.add(code)
                assert list(oracle.t3_weights(code)) == [a, b, c]
    assert seen == set(range(27))                     # 27 of the 32 five-bit states
    # hand values: all -1 -> 0, all 0 -> 13, all +1 -> 26, (-1, 0, 1) -> 0 + 3 + 18
    assert oracle.t3_code([-1, -1, -1]) == 0 and oracle.t3_code([0, 0, 0]) == 13
    assert oracle.t3_code([1, 1, 1]) == 26 and oracle.t3_code([-1, 0, 1]) == 21
    assert oracle.t3_code([1, 0, -1]) == 5
    for bad in range(27, 32):
        assert list(oracle.t3_weights(bad)) == [0, 0, 0]


def test_t3_hand_tiles_with_straddling_fields():
    K = 384                                           # 4 tiles of 96 weights
    row = -np.ones((1, K), np.int8)                   # every triple (-1,-1,-1): code 0
    row[0, 0:3] = 1                                   # tile 0, triple 0: code 26
    row[0, 18:21] = [-1, 0, 1]                        # tile 0, triple 6: code 21, bits 30..34
    row[0, 96 + 93:96 + 96] = 0                       # tile 1, triple 31: code 13, bits 155..159
    c = oracle.cmp_encode(T3, row)
    assert c.shape == (1, 4, 5, 32)
    # tile 0: word 0 = 26 | (21 & 3) << 30; word 1 = 21 >> 2
    assert list(c[0, 0, :, 0]) == [0x4000001A, 0x5, 0, 0, 0]
    # tile 1: word 4 bits 27..31 = 13
    assert list(c[0, 1, :, 0]) == [0, 0, 0, 0, 0x68000000]
    assert not c[0, 2:, :, 0].any()
    assert np.array_equal(oracle.cmp_unpack(T3, c, 1, K), row)


def test_t3_pads_rows_with_zero_weights():
    K = 128                                           # 2 tiles = 192 weights, 64 of padding
    row = -np.ones((1, K), np.int8)
    c = oracle.cmp_encode(T3, row)
    assert c.shape == (1, 2, 5, 32)
    # tile 1, triple 10 = (w126, w127, pad) = (-1, -1, 0): code 9 at bits 50..54 (word 1)
    assert (c[0, 1, 1, 0] >> 18) & 31 == 9
    # tile 1, triple 31 is all padding: code 13 at bits 155..159
    assert c[0, 1, 4, 0] >> 27 == 13
    # tile 1, triple 0 (w96..w98 = -1): code 0
    assert c[0, 1, 0, 0] & 31 == 0


@pytest.mark.parametrize("fmt", [I2, T3])
@pytest.mark.parametrize("N,K", [(1, 128), (33, 384), (70, 1152), (5, 2048)])
def test_roundtrip_random_ternary(fmt, N, K):
    rng = np.random.default_rng(N * 7 + K + fmt)
    wt = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    c = oracle.cmp_encode(fmt, wt)
    assert c.nbytes == oracle.cmp_packed_bytes(fmt, N, K)
    assert np.array_equal(oracle.cmp_unpack(fmt, c, N, K), wt)
    # padding rows of the last group hold zero words in both formats
    if N % 32:
        assert not c[-1, :, :, N % 32:].any()


@pytest.mark.parametrize("N,K,B", [(40, 1024, 1), (33, 2048, 3), (64, 384, 2)])
def test_same_ternary_matrix_same_dot_products_in_all_formats(N, K, B):
    codes, _ = oracle.pack(synth.latent_weights(N, K, seed=N + K))
    wt = oracle.unpack(codes, N, K)
    x = synth.int8_uniform((B, K), seed=B)
    ref = wt.astype(np.int64) @ x.astype(np.int64).T          # brute force [N, B]
    assert np.array_equal(oracle.gemv_acc(codes, x, N, K), ref.T)
    for fmt in (I2, T3):
        c = oracle.cmp_encode(fmt, wt)
        assert np.array_equal(oracle.cmp_gemv_acc(fmt, c, x, N, K), ref.T), fmt


def test_all_ones_activation_gives_row_sums():
    rng = np.random.default_rng(5)
    N, K = 37, 768
    wt = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    x = np.ones((1, K), np.int8)
    for fmt in (I2, T3):
        acc = oracle.cmp_gemv_acc(fmt, oracle.cmp_encode(fmt, wt), x, N, K)
        assert np.array_equal(acc[0], wt.astype(np.int64).sum(axis=1))


# ----------------------------------------------------------------------------- mutants
MUTANTS = {
    "i2_halves_swapped": ("w[q] |= c << (4 * (m % 8) + 2 * (m / 8));",
                          "w[q] |= c << (4 * (m / 2) + 2 * (m % 2));"),
    "i2_sign_code_2": ("static uint32_t orc_i2_code(int8_t w) { return w == 0 ? 0u : (w > 0 ? 1u : 3u); }",
                       "static uint32_t orc_i2_code(int8_t w) { return w == 0 ? 0u : (w > 0 ? 1u : 2u); }"),
    "i2_decode_ignores_sign": ("return (c & 1u) ? ((c & 2u) ? -1 : 1) : 0;",
                               "return (c & 1u) ? 1 : 0;"),
    "t3_digits_reversed": ("return (w[0] + 1) + 3 * (w[1] + 1) + 9 * (w[2] + 1);",
                           "return (w[2] + 1) + 3 * (w[1] + 1) + 9 * (w[0] + 1);"),
    "t3_fields_of_six_bits": ("const int bit = 5 * j + b;\n                        w[bit / 32]",
                              "const int bit = 5 * j + b + j / 6;\n                        w[bit / 32]"),
    "t3_odd_tile_count": ("if (fmt == ORC_FMT_T3) return 2 * ((K + 191) / 192);",
                          "if (fmt == ORC_FMT_T3) return (K + 95) / 96;"),
    "cmp_dot_drops_last_term": ("for (int64_t k = 0; k < K; k++) a += (int64_t)row[k] * (int64_t)x[b * K + k];",
                                "for (int64_t k = 1; k < K; k++) a += (int64_t)row[k] * (int64_t)x[b * K + k];"),
    "cmp_rows_of_16": ("return ((n / ORC_GROUP) * T + t) * (tw * ORC_GROUP) + q * ORC_GROUP + n % ORC_GROUP;",
                       "return ((n / 16) * T + t) * (tw * 16) + q * 16 + n % 16;"),
}


def _pins_pass():
    checks = [
        test_sizes_closed_forms,
        test_i2_hand_word,
        test_t3_code_table_is_exhaustive,
        test_t3_hand_tiles_with_straddling_fields,
        test_t3_pads_rows_with_zero_weights,
        lambda: test_same_ternary_matrix_same_dot_products_in_all_formats(33, 2048, 3),
        test_all_ones_activation_gives_row_sums,
    ]
    for c in checks:
        try:
            c()
        except AssertionError:
            return False
    return True


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_cmp_mutant_is_caught(name):
    old, new = MUTANTS[name]
    with open(SRC) as f:
        src = f.read()
    assert src.count(old) == 1, "mutation anchor not found: " + name
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "m.c")
        so = os.path.join(d, "libm_%s.so" % name)
        with open(c, "w") as f:
            f.write(src.replace(old, new))
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", so, c])
        try:
            oracle_mod.use_library(so)
            assert not _pins_pass(), "pins did not catch mutant " + name
        finally:
            oracle_mod.use_library(None)


def test_committed_oracle_passes_cmp_pins():
    assert _pins_pass()
