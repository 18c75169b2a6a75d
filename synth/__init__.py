"""Seeded synthetic inputs for the Sherry path (no method arithmetic here).

The generator is written in C (``synth.c``) and compiled with gcc on first
use; the definitions of the draws are given there.  Both the CPU oracle tests
and the GPU tests and benchmark take their inputs from this module, so both
sides always read the same host bytes.
"""
import ctypes
import os
import subprocess

import numpy as np

from .workloads import (  # noqa: F401
    LLAMA_1B_LAYERS, LLAMA_3B_LAYERS, PREFILL_GEMMS, decode_stack, layer_seed,
)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(force=False):
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", tmp, _SRC,
                               "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u64, i64, p = ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p
        lib.synth_u64.argtypes = [u64, u64]
        lib.synth_u64.restype = u64
        lib.synth_normal_f32.argtypes = [u64, u64, i64, ctypes.c_double, p]
        lib.synth_normal_f32.restype = None
        lib.synth_int8_uniform.argtypes = [u64, u64, i64, p]
        lib.synth_int8_uniform.restype = None
        lib.synth_int8_clipped_normal.argtypes = [u64, u64, i64, p]
        lib.synth_int8_clipped_normal.restype = None
        _lib = lib
    return _lib


def u64(seed, ctr):
    return int(_load().synth_u64(seed, ctr))


def latent_weights(N, K, seed=0, sigma=0.02, out=None):
    """fp32 latent weights [N, K], element (n, k) is normal draw n*K + k of `seed`."""
    if out is None:
        out = np.empty((N, K), np.float32)
    assert out.dtype == np.float32 and out.flags.c_contiguous and out.size == N * K
    _load().synth_normal_f32(seed, 0, N * K, sigma, ctypes.c_void_p(out.ctypes.data))
    return out


def int8_uniform(shape, seed=1, out=None):
    """int8 activations uniform on [-127, 127]."""
    if out is None:
        out = np.empty(shape, np.int8)
    _load().synth_int8_uniform(seed, 0, out.size, ctypes.c_void_p(out.ctypes.data))
    return out


def int8_clipped_normal(shape, seed=1, out=None):
    """int8 activations round(127 * clip(z/3, -1, 1)), z ~ N(0, 1)."""
    if out is None:
        out = np.empty(shape, np.int8)
    _load().synth_int8_clipped_normal(seed, 0, out.size, ctypes.c_void_p(out.ctypes.data))
    return out
