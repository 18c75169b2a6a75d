"""Per-device set-up in a second CUDA context (needs a B200).

The library sets the GEMV and GEMM kernels' shared-memory attributes once per
device and keeps them with the context they were set in.  A child process
drives the library through the driver API: the device's primary context, then
a context of its own (created with cuCtxCreate, current on the thread), then
the primary context again.  In each, a GEMV (dot kernel), an MMA GEMV and a
GEMM run on buffers of that context and must give the oracle's results.  Had
the set-up been kept per device only, the launches in the new context would
fail with a launch error (the attribute is missing there), not fault.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import ctypes
import numpy as np
import oracle, synth
from bit_gemv_sherry_b200 import sherry as S

cu = ctypes.CDLL("libcuda.so.1")
u64, vp, c_int, c_uint, sz = ctypes.c_uint64, ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t
sig = {
    "cuInit": [c_uint],
    "cuDeviceGet": [ctypes.POINTER(c_int), c_int],
    "cuDevicePrimaryCtxRetain": [ctypes.POINTER(vp), c_int],
    "cuDevicePrimaryCtxRelease_v2": [c_int],
    "cuCtxCreate_v2": [ctypes.POINTER(vp), c_uint, c_int],
    "cuCtxDestroy_v2": [vp],
    "cuCtxSetCurrent": [vp],
    "cuCtxSynchronize": [],
    "cuMemAlloc_v2": [ctypes.POINTER(u64), sz],
    "cuMemFree_v2": [u64],
    "cuMemcpyHtoD_v2": [u64, vp, sz],
    "cuMemcpyDtoH_v2": [vp, u64, sz],
}
for name, args in sig.items():
    getattr(cu, name).argtypes = args
    getattr(cu, name).restype = c_int


def ck(r, what):
    if r != 0:
        raise RuntimeError("%s: CUresult %d" % (what, r))


L = S.lib()


def to_dev(a, bufs):
    a = np.ascontiguousarray(a)
    d = u64(0)
    ck(cu.cuMemAlloc_v2(ctypes.byref(d), max(a.nbytes, 16)), "cuMemAlloc")
    bufs.append(d.value)
    ck(cu.cuMemcpyHtoD_v2(d.value, a.ctypes.data, a.nbytes), "cuMemcpyHtoD")
    return d.value


def from_dev(d, shape, dtype):
    out = np.empty(shape, dtype)
    ck(cu.cuMemcpyDtoH_v2(out.ctypes.data, d, out.nbytes), "cuMemcpyDtoH")
    return out


def run_case(tag):
    bufs = []
    N, K = 512, 2048
    codes, scales = oracle.pack(synth.latent_weights(N, K, seed=301))
    dc, ds = to_dev(codes, bufs), to_dev(scales, bufs)
    for B in (1, 4):   # the dot kernel, the MMA kernel
        x = synth.int8_uniform((B, K), seed=302 + B)
        dx = to_dev(x, bufs)
        dy = to_dev(np.full((B, N), np.nan, np.float32), bufs)
        wsb = S.gemv_workspace_bytes(N, K, B)
        dws = to_dev(np.zeros(max(wsb, 16), np.uint8), bufs)
        st = L.sherry_gemv(vp(dc), vp(ds), vp(dx), vp(dy), N, K, B, vp(dws), wsb, None)
        assert st == 0, (tag, "gemv", B, st, L.sherry_last_error())
        ck(cu.cuCtxSynchronize(), "sync")
        y = from_dev(dy, (B, N), np.float32)
        assert np.array_equal(y, oracle.gemv(codes, scales, x, K).astype(np.float32)), (tag, B)
    M = 300
    x = synth.int8_clipped_normal((M, K), seed=305)
    dx = to_dev(x, bufs)
    dy = to_dev(np.full((M, N), np.nan, np.float32), bufs)
    st = L.sherry_gemm(vp(dc), vp(ds), vp(dx), vp(dy), M, N, K, None)
    assert st == 0, (tag, "gemm", st, L.sherry_last_error())
    ck(cu.cuCtxSynchronize(), "sync")
    y = from_dev(dy, (M, N), np.float32)
    assert np.array_equal(y, oracle.gemm(codes, scales, x, K).astype(np.float32)), tag
    for d in bufs:
        ck(cu.cuMemFree_v2(d), "cuMemFree")


ck(cu.cuInit(0), "cuInit")
dev = c_int(0)
ck(cu.cuDeviceGet(ctypes.byref(dev), 0), "cuDeviceGet")
prim, own = vp(), vp()
ck(cu.cuDevicePrimaryCtxRetain(ctypes.byref(prim), dev), "cuDevicePrimaryCtxRetain")
ck(cu.cuCtxSetCurrent(prim), "cuCtxSetCurrent")
run_case("primary")
ck(cu.cuCtxCreate_v2(ctypes.byref(own), 0, dev), "cuCtxCreate")   # current from here on
run_case("own context")
ck(cu.cuCtxSetCurrent(prim), "cuCtxSetCurrent")
run_case("primary again")
assert L.sherry_device_error() == 0
ck(cu.cuCtxDestroy_v2(own), "cuCtxDestroy")
ck(cu.cuCtxSetCurrent(prim), "cuCtxSetCurrent")
ck(cu.cuDevicePrimaryCtxRelease_v2(dev), "cuDevicePrimaryCtxRelease")
print("contexts ok")
'''


def test_setup_is_made_again_in_another_context():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and "contexts ok" in r.stdout, r.stdout + r.stderr
