"""ctypes binding of the C oracle (test infrastructure only).

Argument marshalling only: every computation happens in ``sherry_oracle.c``.
"""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sherry_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_sherry.so")
_lib = None


def build(force=False):
    """Compile the oracle with gcc (plain C, OpenMP over output rows)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _load(path=None):
    global _lib
    if _lib is not None and path is None:
        return _lib
    lib = ctypes.CDLL(path or build())
    i64, p = ctypes.c_int64, ctypes.c_void_p
    lib.oracle_packed_bytes.argtypes = [i64, i64]
    lib.oracle_packed_bytes.restype = i64
    lib.oracle_prune_block.argtypes = [p, p, p]
    lib.oracle_prune_block.restype = None
    lib.oracle_block_code.argtypes = [ctypes.c_int32, p]
    lib.oracle_block_code.restype = ctypes.c_int32
    lib.oracle_code_weights.argtypes = [ctypes.c_int32, p]
    lib.oracle_code_weights.restype = None
    lib.oracle_pack.argtypes = [p, i64, i64, p, p]
    lib.oracle_unpack.argtypes = [p, i64, i64, p]
    lib.oracle_gemv_acc.argtypes = [p, p, i64, i64, i64, p]
    lib.oracle_gemv.argtypes = [p, p, p, i64, i64, i64, p]
    lib.oracle_gemm_acc.argtypes = [p, p, i64, i64, i64, p]
    lib.oracle_gemm.argtypes = [p, p, p, i64, i64, i64, p]
    lib.oracle_quantize_act.argtypes = [p, i64, i64, p, p]
    lib.oracle_gemv_act.argtypes = [p, p, p, p, i64, i64, i64, p]
    lib.oracle_quantize_f32.argtypes = [p, i64, i64, p, p]
    lib.oracle_swiglu.argtypes = [p, p, i64, p]
    i32 = ctypes.c_int32
    lib.oracle_cmp_tiles.argtypes = [i32, i64]
    lib.oracle_cmp_tiles.restype = i64
    lib.oracle_cmp_packed_bytes.argtypes = [i32, i64, i64]
    lib.oracle_cmp_packed_bytes.restype = i64
    lib.oracle_t3_code.argtypes = [p]
    lib.oracle_t3_code.restype = i32
    lib.oracle_t3_weights.argtypes = [i32, p]
    lib.oracle_t3_weights.restype = None
    lib.oracle_cmp_encode.argtypes = [i32, p, i64, i64, p]
    lib.oracle_cmp_unpack.argtypes = [i32, p, i64, i64, p]
    lib.oracle_cmp_gemv_acc.argtypes = [i32, p, p, i64, i64, i64, p]
    for f in ("oracle_pack", "oracle_unpack", "oracle_gemv_acc", "oracle_gemv",
              "oracle_gemm_acc", "oracle_gemm", "oracle_quantize_act", "oracle_gemv_act",
              "oracle_quantize_f32", "oracle_swiglu", "oracle_cmp_encode", "oracle_cmp_unpack",
              "oracle_cmp_gemv_acc"):
        getattr(lib, f).restype = ctypes.c_int
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
    lib.oracle_set_num_threads.restype = None
    _lib = lib
    return lib


def use_library(path):
    """Point the binding at another build of the oracle source (mutation tests);
    `use_library(None)` returns to the committed source."""
    global _lib
    _lib = None
    if path is not None:
        _load(path)


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data)


def _check(rc, name):
    if rc != 0:
        raise ValueError("%s failed with status %d" % (name, rc))


def num_threads():
    return _load().oracle_num_threads()


def set_num_threads(n):
    _load().oracle_set_num_threads(int(n))


def packed_bytes(N, K):
    return int(_load().oracle_packed_bytes(N, K))


def prune_block(w4):
    w = np.ascontiguousarray(w4, dtype=np.float32)
    assert w.shape == (4,)
    p = np.zeros(1, np.int32)
    neg = np.zeros(3, np.int32)
    _load().oracle_prune_block(_ptr(w), _ptr(p), _ptr(neg))
    return int(p[0]), [int(v) for v in neg]


def block_code(zero_pos, neg):
    n = np.ascontiguousarray(neg, dtype=np.int32)
    return int(_load().oracle_block_code(int(zero_pos), _ptr(n)))


def code_weights(code):
    w = np.zeros(4, np.int8)
    _load().oracle_code_weights(int(code), _ptr(w))
    return w


GROUP = 32  # rows per group of the layout


def pack(w):
    """w: float32 [N, K] -> (codes uint32 [ceil(N/32), K/128, 5, 32], scales float32 [N]).

    codes[g, t, p, r] is word p (Z0, Z1, S0, S1, S2) of tile t of row 32 g + r;
    rows past N are padding (zeros)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    codes = np.zeros(((N + GROUP - 1) // GROUP, max(K // 128, 1), 5, GROUP), np.uint32)
    scales = np.zeros(N, np.float32)
    _check(_load().oracle_pack(_ptr(w), N, K, _ptr(codes), _ptr(scales)), "oracle_pack")
    return codes, scales


def unpack(codes, N, K):
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    wt = np.zeros((N, K), np.int8)
    _check(_load().oracle_unpack(_ptr(codes), N, K, _ptr(wt)), "oracle_unpack")
    return wt


def _x2(x, K):
    x = np.ascontiguousarray(x, dtype=np.int8)
    if x.ndim == 1:
        x = x.reshape(1, -1)
    assert x.shape[1] == K
    return x


def gemv_acc(codes, x, N, K):
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    x = _x2(x, K)
    acc = np.zeros((x.shape[0], N), np.int64)
    _check(_load().oracle_gemv_acc(_ptr(codes), _ptr(x), N, K, x.shape[0], _ptr(acc)),
           "oracle_gemv_acc")
    return acc


def gemv(codes, scales, x, K):
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    N = scales.shape[0]
    x = _x2(x, K)
    y = np.zeros((x.shape[0], N), np.float64)
    _check(_load().oracle_gemv(_ptr(codes), _ptr(scales), _ptr(x), N, K, x.shape[0], _ptr(y)),
           "oracle_gemv")
    return y


def gemm_acc(codes, x, N, K):
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    x = _x2(x, K)
    acc = np.zeros((x.shape[0], N), np.int64)
    _check(_load().oracle_gemm_acc(_ptr(codes), _ptr(x), x.shape[0], N, K, _ptr(acc)),
           "oracle_gemm_acc")
    return acc


def gemm(codes, scales, x, K):
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    N = scales.shape[0]
    x = _x2(x, K)
    y = np.zeros((x.shape[0], N), np.float64)
    _check(_load().oracle_gemm(_ptr(codes), _ptr(scales), _ptr(x), x.shape[0], N, K, _ptr(y)),
           "oracle_gemm")
    return y


def quantize_act(x_bf16):
    """Per-token absmax int8 quantization of bf16 activations (uint16 bit
    patterns, [B][K]) -> (q int8 [B][K], s float32 [B])."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    if x.ndim == 1:
        x = x.reshape(1, -1)
    B, K = x.shape
    q = np.zeros((B, K), np.int8)
    s = np.zeros(B, np.float32)
    _check(_load().oracle_quantize_act(_ptr(x), B, K, _ptr(q), _ptr(s)), "oracle_quantize_act")
    return q, s


def quantize_f32(x):
    """Per-token absmax int8 quantization of fp32 activations [B][K] -> (q int8
    [B][K], s float32 [B]); the rule of quantize_act, read from fp32 values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if x.ndim == 1:
        x = x.reshape(1, -1)
    B, K = x.shape
    q = np.zeros((B, K), np.int8)
    s = np.zeros(B, np.float32)
    _check(_load().oracle_quantize_f32(_ptr(x), B, K, _ptr(q), _ptr(s)), "oracle_quantize_f32")
    return q, s


def swiglu(g, u):
    """h = silu(g) * u elementwise (fp32 in, double evaluation, fp32 out)."""
    g = np.ascontiguousarray(g, dtype=np.float32)
    u = np.ascontiguousarray(u, dtype=np.float32)
    if g.shape != u.shape:
        raise ValueError("g and u differ in shape")
    h = np.zeros(g.shape, np.float32)
    _check(_load().oracle_swiglu(_ptr(g), _ptr(u), g.size, _ptr(h)), "oracle_swiglu")
    return h


def gemv_act(codes, scales, q, sx, K):
    """y[b][n] = scales[n] * sx[b] * (W . q^T)[b][n] in double."""
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    N = scales.shape[0]
    q = _x2(q, K)
    y = np.zeros((q.shape[0], N), np.float64)
    _check(_load().oracle_gemv_act(_ptr(codes), _ptr(scales), _ptr(q), _ptr(sx), N, K,
                                   q.shape[0], _ptr(y)), "oracle_gemv_act")
    return y


def bf16_bits(values):
    """bf16 bit patterns of float values that bf16 represents exactly (test data)."""
    v = np.ascontiguousarray(values, dtype=np.float32)
    u = v.view(np.uint32)
    if np.any(u & 0xFFFF):
        raise ValueError("value not representable in bf16")
    return (u >> 16).astype(np.uint16)


# ----------------------------------------------------------------------------- comparison formats
FMT_I2 = 1  # 2 bits per weight, aligned
FMT_T3 = 2  # three weights in five bits (base 3)
_TILE_WORDS = {FMT_I2: 8, FMT_T3: 5}


def cmp_tiles(fmt, K):
    return int(_load().oracle_cmp_tiles(fmt, K))


def cmp_packed_bytes(fmt, N, K):
    return int(_load().oracle_cmp_packed_bytes(fmt, N, K))


def t3_code(tri):
    t = np.ascontiguousarray(tri, dtype=np.int8)
    assert t.shape == (3,)
    return int(_load().oracle_t3_code(_ptr(t)))


def t3_weights(code):
    w = np.zeros(3, np.int8)
    _load().oracle_t3_weights(int(code), _ptr(w))
    return w


def cmp_encode(fmt, wt):
    """Ternary int8 [N, K] -> codes uint32 [ceil(N/32), tiles, words, 32] of format fmt."""
    wt = np.ascontiguousarray(wt, dtype=np.int8)
    N, K = wt.shape
    T = cmp_tiles(fmt, K)
    if T == 0:
        raise ValueError("bad format or K")
    codes = np.zeros(((N + GROUP - 1) // GROUP, T, _TILE_WORDS[fmt], GROUP), np.uint32)
    _check(_load().oracle_cmp_encode(fmt, _ptr(wt), N, K, _ptr(codes)), "oracle_cmp_encode")
    return codes


def cmp_unpack(fmt, codes, N, K):
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    wt = np.zeros((N, K), np.int8)
    _check(_load().oracle_cmp_unpack(fmt, _ptr(codes), N, K, _ptr(wt)), "oracle_cmp_unpack")
    return wt


def cmp_gemv_acc(fmt, codes, x, N, K):
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    x = _x2(x, K)
    acc = np.zeros((x.shape[0], N), np.int64)
    _check(_load().oracle_cmp_gemv_acc(fmt, _ptr(codes), _ptr(x), N, K, x.shape[0], _ptr(acc)),
           "oracle_cmp_gemv_acc")
    return acc
