"""Python binding of libsherry.so (argument marshalling only).

Every step of the path runs in the library's CUDA kernels; this module only
checks tensor properties, passes raw device pointers and the current CUDA
stream, and turns status codes into exceptions.  PyTorch provides device
memory and streams.  There is no CPU fallback: if the library cannot be
loaded, importing the functions raises.
"""
import ctypes
import os

import torch

from . import build as _build

_lib = None

STATUS = {
    0: "SHERRY_OK", 1: "SHERRY_ERR_NULL", 2: "SHERRY_ERR_SHAPE", 3: "SHERRY_ERR_ALIGN",
    4: "SHERRY_ERR_UNSUPPORTED", 5: "SHERRY_ERR_CUDA", 6: "SHERRY_ERR_TIMEOUT",
    7: "SHERRY_ERR_WORKSPACE",
}
TILE_K = 128
MAX_GEMV_BATCH = 16
MAX_GROUP = 128


class SherryError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        msg = "%s: %s (%s)" % (where, STATUS.get(status, status),
                               lib().sherry_status_string(status).decode())
        if status == 5:
            msg += ": " + lib().sherry_last_error().decode()
        super().__init__(msg)


class PackDesc(ctypes.Structure):
    _fields_ = [("w", ctypes.c_void_p), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("N", ctypes.c_int64), ("K", ctypes.c_int64)]


class GemvDesc(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("x", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64)]


class F32Desc(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("x", ctypes.c_void_p),
                ("u", ctypes.c_void_p), ("y", ctypes.c_void_p), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64)]


def library_path():
    return _build.LIB


def lib():
    """Load libsherry.so (built in-tree).  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.LIB
    if not os.path.exists(path):
        raise RuntimeError("libsherry.so not built: run `python -m bit_gemv_sherry_b200.build` "
                           "(expected at %s)" % path)
    L = ctypes.CDLL(path)
    p, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    sig = {
        "sherry_packed_bytes": ([i64, i64], sz),
        "sherry_pack": ([p, i64, i64, p, p, p], i32),
        "sherry_pack_grouped": ([p, i32, p], i32),
        "sherry_gemv_workspace_bytes": ([i64, i64, i32], sz),
        "sherry_gemv": ([p, p, p, p, i64, i64, i32, p, sz, p], i32),
        "sherry_gemv_acc": ([p, p, p, i64, i64, i32, p, sz, p], i32),
        "sherry_gemv_static": ([p, p, p, p, i64, i64, i32, p], i32),
        "sherry_quantize_act": ([p, i64, i64, p, p, p], i32),
        "sherry_gemv_bf16_workspace_bytes": ([i64, i64, i32], sz),
        "sherry_gemv_bf16": ([p, p, p, p, i64, i64, i32, p, sz, p], i32),
        "sherry_gemv_bf16_grouped": ([p, i32, i32, p, sz, p], i32),
        "sherry_quantize_f32": ([p, i64, i64, p, p, p], i32),
        "sherry_quantize_swiglu": ([p, p, i64, i64, p, p, p], i32),
        "sherry_gemv_f32_workspace_bytes": ([i64, i64, i32], sz),
        "sherry_gemv_f32": ([p, p, p, p, i64, i64, i32, p, sz, p], i32),
        "sherry_gemv_swiglu": ([p, p, p, p, p, i64, i64, i32, p, sz, p], i32),
        "sherry_gemv_f32_grouped": ([p, i32, i32, p, sz, p], i32),
        "sherry_gemv_grouped": ([p, i32, i32, p, sz, p], i32),
        "sherry_gemv_prepare": ([p, i32, i32, p, sz, p], i32),
        "sherry_gemv_run": ([p, i32, i32, p, sz, p], i32),
        "sherry_gemm": ([p, p, p, p, i64, i64, i64, p], i32),
        "sherry_gemm_acc": ([p, p, p, i64, i64, i64, p], i32),
        "sherry_cmp_packed_bytes": ([i32, i64, i64], sz),
        "sherry_cmp_workspace_bytes": ([i32, i64, i64, i32], sz),
        "sherry_cmp_transcode": ([i32, p, i64, i64, p, p], i32),
        "sherry_cmp_gemv_grouped": ([i32, p, i32, i32, p, sz, p], i32),
        "sherry_cmp_gemv_acc": ([i32, p, p, p, i64, i64, i32, p, sz, p], i32),
        "sherry_probe_mma_i8": ([i32, p, p], i32),
        "sherry_device_error": ([], i32),
        "sherry_set_wait_limit": ([i64], i32),
        "sherry_status_string": ([i32], ctypes.c_char_p),
        "sherry_last_error": ([], ctypes.c_char_p),
        "sherry_version": ([], i32),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


def _check(status, where):
    if status != 0:
        raise SherryError(status, where)


# The raw handle of a device's current stream.  torch's private accessor skips
# building a Stream object (about 2 us per call on the host); the public one is
# the fallback.
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream_handle(device):
    if _raw_stream is not None:
        idx = device.index if device.index is not None else torch.cuda.current_device()
        return _raw_stream(idx)
    return torch.cuda.current_stream(device).cuda_stream


def _stream(t):
    return ctypes.c_void_p(_stream_handle(t.device))


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _need(t, dtype, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


_workspaces = {}


def workspace(nbytes, device):
    """A cached device scratch buffer of at least `nbytes` for (device, current stream)."""
    device = torch.device(device)
    key = (device.index, _stream_handle(device))
    buf = _workspaces.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 1 << 16), dtype=torch.uint8, device=device)
        _workspaces[key] = buf
    return buf


def packed_bytes(N, K):
    return int(lib().sherry_packed_bytes(N, K))


def gemv_workspace_bytes(N, K, B):
    return int(lib().sherry_gemv_workspace_bytes(N, K, B))


GROUP = 32  # rows per group of the code layout


def codes_shape(N, K):
    """Shape of the int32 tensor holding the codes of an N x K matrix."""
    return ((N + GROUP - 1) // GROUP, K // TILE_K, 5, GROUP)


def pack(w, codes=None, scales=None):
    """w: float32 [N, K] CUDA -> (codes int32 [ceil(N/32), K/128, 5, 32] holding the
    uint32 words, scales float32 [N])."""
    _need(w, torch.float32, "w")
    N, K = w.shape
    if codes is None:
        codes = torch.empty(codes_shape(N, max(K, TILE_K)), dtype=torch.int32, device=w.device)
    if scales is None:
        scales = torch.empty(N, dtype=torch.float32, device=w.device)
    _check(lib().sherry_pack(_ptr(w), N, K, _ptr(codes), _ptr(scales), _stream(w)), "sherry_pack")
    return codes, scales


class GroupedPack:
    """Pre-marshalled grouped pack (sherry_pack_grouped): items are
    (w float32 [N, K], codes, scales) with codes/scales shaped as pack() makes them."""

    def __init__(self, items):
        n = len(items)
        self.descs = (PackDesc * n)()
        for i, (w, codes, scales) in enumerate(items):
            _need(w, torch.float32, "w")
            N, K = w.shape
            _need(scales, torch.float32, "scales")
            if tuple(codes.shape) != codes_shape(N, max(K, TILE_K)) or scales.numel() != N:
                raise ValueError("codes/scales do not match w of shape %s" % (tuple(w.shape),))
            self.descs[i] = PackDesc(w.data_ptr(), codes.data_ptr(), scales.data_ptr(), N, K)
        self.items = items
        self.n = n
        self.device = items[0][0].device

    def __call__(self, stream=None):
        s = ctypes.c_void_p(stream if stream is not None
                            else _stream_handle(self.device))
        _check(lib().sherry_pack_grouped(ctypes.cast(self.descs, ctypes.c_void_p), self.n, s),
               "sherry_pack_grouped")


def pack_grouped(ws):
    """Packs a list of float32 [N, K] CUDA matrices in one launch; returns
    [(codes, scales)] as pack() would."""
    outs = [(torch.empty(codes_shape(w.shape[0], max(w.shape[1], TILE_K)), dtype=torch.int32,
                         device=w.device),
             torch.empty(w.shape[0], dtype=torch.float32, device=w.device)) for w in ws]
    GroupedPack([(w, c, s) for w, (c, s) in zip(ws, outs)])()
    return outs


def _codes_shape(codes, N):
    _need(codes, torch.int32, "codes")
    if codes.dim() != 4 or codes.shape[2] != 5 or codes.shape[3] != GROUP:
        raise ValueError("codes must have shape [ceil(N/32), K/128, 5, 32]")
    if codes.shape[0] != (N + GROUP - 1) // GROUP:
        raise ValueError("codes hold %d row groups, N = %d needs %d"
                         % (codes.shape[0], N, (N + GROUP - 1) // GROUP))
    return N, codes.shape[1] * TILE_K


def gemv(codes, scales, x, y=None, ws=None):
    """y[B, N] = scales * (W . x^T); x int8 [B, K] (or [K])."""
    _need(scales, torch.float32, "scales")
    N, K = _codes_shape(codes, scales.numel())
    _need(x, torch.int8, "x")
    x2 = x.view(1, -1) if x.dim() == 1 else x
    B = x2.shape[0]
    if y is None:
        y = torch.empty((B, N), dtype=torch.float32, device=x.device)
    nb = gemv_workspace_bytes(N, K, B)
    ws = workspace(nb, x.device) if ws is None else ws
    _check(lib().sherry_gemv(_ptr(codes), _ptr(scales), _ptr(x2), _ptr(y), N, K, B, _ptr(ws),
                             ws.numel(), _stream(x)), "sherry_gemv")
    return y


STATIC_SCRATCH_BYTES = 4 << 20


def gemv_static(codes, scales, x, y=None):
    """As gemv, with the library's fixed scratch array instead of a workspace
    (sherry_gemv_static: the C call allocates nothing; y is allocated here
    only when not given)."""
    _need(scales, torch.float32, "scales")
    N, K = _codes_shape(codes, scales.numel())
    _need(x, torch.int8, "x")
    x2 = x.view(1, -1) if x.dim() == 1 else x
    B = x2.shape[0]
    if y is None:
        y = torch.empty((B, N), dtype=torch.float32, device=x.device)
    _check(lib().sherry_gemv_static(_ptr(codes), _ptr(scales), _ptr(x2), _ptr(y), N, K, B,
                                    _stream(x)), "sherry_gemv_static")
    return y


def gemv_acc(codes, x, N, acc=None, ws=None):
    """Exact int32 accumulators acc[B, N] = W . x^T."""
    N, K = _codes_shape(codes, N)
    _need(x, torch.int8, "x")
    x2 = x.view(1, -1) if x.dim() == 1 else x
    B = x2.shape[0]
    if acc is None:
        acc = torch.empty((B, N), dtype=torch.int32, device=x.device)
    nb = gemv_workspace_bytes(N, K, B)
    ws = workspace(nb, x.device) if ws is None else ws
    _check(lib().sherry_gemv_acc(_ptr(codes), _ptr(x2), _ptr(acc), N, K, B, _ptr(ws), ws.numel(),
                                 _stream(x)), "sherry_gemv_acc")
    return acc


def gemv_grouped(items, B, ws=None):
    """items: list of (codes, scales, x [B, K], y [B, N]); runs every GEMV in one pass."""
    n = len(items)
    descs = (GemvDesc * n)()
    total = 0
    dev = None
    for i, (codes, scales, x, y) in enumerate(items):
        _need(scales, torch.float32, "scales")
        N, K = _codes_shape(codes, scales.numel())
        _need(x, torch.int8, "x")
        _need(y, torch.float32, "y")
        descs[i] = GemvDesc(codes.data_ptr(), scales.data_ptr(), x.data_ptr(), y.data_ptr(), N, K)
        total += gemv_workspace_bytes(N, K, B)
        dev = x.device
    ws = workspace(total, dev) if ws is None else ws
    _check(lib().sherry_gemv_grouped(ctypes.cast(descs, ctypes.c_void_p), n, B, _ptr(ws),
                                     ws.numel(), _stream(items[0][2])), "sherry_gemv_grouped")


def quantize_act(x, q=None, s=None):
    """Per-token absmax int8 quantization of bf16 activations x [B, K]:
    returns (q int8 [B, K], s fp32 [B]) with x ~ s[:, None] * q."""
    _need(x, torch.bfloat16, "x")
    x2 = x.view(1, -1) if x.dim() == 1 else x
    B, K = x2.shape
    if q is None:
        q = torch.empty((B, K), dtype=torch.int8, device=x.device)
    if s is None:
        s = torch.empty((B,), dtype=torch.float32, device=x.device)
    _check(lib().sherry_quantize_act(_ptr(x2), B, K, _ptr(q), _ptr(s), _stream(x)),
           "sherry_quantize_act")
    return q, s


def gemv_bf16_workspace_bytes(N, K, B):
    return int(lib().sherry_gemv_bf16_workspace_bytes(N, K, B))


def gemv_bf16(codes, scales, x, y=None, ws=None):
    """y[B, N] = scales * s_x * (W . q^T) for bf16 activations x [B, K] quantized per token."""
    _need(scales, torch.float32, "scales")
    N, K = _codes_shape(codes, scales.numel())
    _need(x, torch.bfloat16, "x")
    x2 = x.view(1, -1) if x.dim() == 1 else x
    B = x2.shape[0]
    if y is None:
        y = torch.empty((B, N), dtype=torch.float32, device=x.device)
    nb = gemv_bf16_workspace_bytes(N, K, B)
    ws = workspace(nb, x.device) if ws is None else ws
    _check(lib().sherry_gemv_bf16(_ptr(codes), _ptr(scales), _ptr(x2), _ptr(y), N, K, B, _ptr(ws),
                                  ws.numel(), _stream(x)), "sherry_gemv_bf16")
    return y


def gemv_bf16_grouped(items, B, ws=None):
    """items: list of (codes, scales, x bf16 [B, K], y [B, N]); one pass over all GEMVs."""
    n = len(items)
    descs = (GemvDesc * n)()  # same field layout as sherry_gemv_bf16_desc
    total = 0
    dev = None
    for i, (codes, scales, x, y) in enumerate(items):
        _need(scales, torch.float32, "scales")
        N, K = _codes_shape(codes, scales.numel())
        _need(x, torch.bfloat16, "x")
        _need(y, torch.float32, "y")
        descs[i] = GemvDesc(codes.data_ptr(), scales.data_ptr(), x.data_ptr(), y.data_ptr(), N, K)
        total += gemv_bf16_workspace_bytes(N, K, B)
        dev = x.device
    ws = workspace(total, dev) if ws is None else ws
    _check(lib().sherry_gemv_bf16_grouped(ctypes.cast(descs, ctypes.c_void_p), n, B, _ptr(ws),
                                          ws.numel(), _stream(items[0][2])),
           "sherry_gemv_bf16_grouped")


def _rows(t, name):
    _need(t, torch.float32, name)
    return t.view(1, -1) if t.dim() == 1 else t


def quantize_f32(x, q=None, s=None):
    """Per-token absmax int8 quantization of fp32 activations x [B, K]
    (K a multiple of 128): returns (q int8 [B, K], s fp32 [B])."""
    x2 = _rows(x, "x")
    B, K = x2.shape
    q = torch.empty((B, K), dtype=torch.int8, device=x.device) if q is None else q
    s = torch.empty((B,), dtype=torch.float32, device=x.device) if s is None else s
    _check(lib().sherry_quantize_f32(_ptr(x2), B, K, _ptr(q), _ptr(s), _stream(x)),
           "sherry_quantize_f32")
    return q, s


def quantize_swiglu(g, u, q=None, s=None):
    """quantize_f32 of h = silu(g) * u, formed inside the front-end."""
    g2, u2 = _rows(g, "g"), _rows(u, "u")
    if g2.shape != u2.shape:
        raise ValueError("g and u differ in shape")
    B, K = g2.shape
    q = torch.empty((B, K), dtype=torch.int8, device=g.device) if q is None else q
    s = torch.empty((B,), dtype=torch.float32, device=g.device) if s is None else s
    _check(lib().sherry_quantize_swiglu(_ptr(g2), _ptr(u2), B, K, _ptr(q), _ptr(s), _stream(g)),
           "sherry_quantize_swiglu")
    return q, s


def gemv_f32_workspace_bytes(N, K, B):
    return int(lib().sherry_gemv_f32_workspace_bytes(N, K, B))


def gemv_f32(codes, scales, x, y=None, ws=None):
    """y[B, N] = scales * s_x * (W . q^T) for fp32 activations x [B, K] quantized per token."""
    _need(scales, torch.float32, "scales")
    N, K = _codes_shape(codes, scales.numel())
    x2 = _rows(x, "x")
    B = x2.shape[0]
    y = torch.empty((B, N), dtype=torch.float32, device=x.device) if y is None else y
    ws = workspace(gemv_f32_workspace_bytes(N, K, B), x.device) if ws is None else ws
    _check(lib().sherry_gemv_f32(_ptr(codes), _ptr(scales), _ptr(x2), _ptr(y), N, K, B, _ptr(ws),
                                 ws.numel(), _stream(x)), "sherry_gemv_f32")
    return y


def gemv_swiglu(codes, scales, g, u, y=None, ws=None):
    """gemv_f32 on h = silu(g) * u (the down projection of a gated MLP); g, u fp32 [B, K]."""
    _need(scales, torch.float32, "scales")
    N, K = _codes_shape(codes, scales.numel())
    g2, u2 = _rows(g, "g"), _rows(u, "u")
    if g2.shape != u2.shape:
        raise ValueError("g and u differ in shape")
    B = g2.shape[0]
    y = torch.empty((B, N), dtype=torch.float32, device=g.device) if y is None else y
    ws = workspace(gemv_f32_workspace_bytes(N, K, B), g.device) if ws is None else ws
    _check(lib().sherry_gemv_swiglu(_ptr(codes), _ptr(scales), _ptr(g2), _ptr(u2), _ptr(y), N, K, B,
                                    _ptr(ws), ws.numel(), _stream(g)), "sherry_gemv_swiglu")
    return y


class GroupedGemvF32:
    """Pre-marshalled grouped GEMV on fp32 activations (sherry_gemv_f32_grouped):
    items are (codes, scales, x fp32 [B, K], u fp32 [B, K] or None, y [B, N])."""

    def __init__(self, items, B, ws=None):
        n = len(items)
        self.descs = (F32Desc * n)()
        total = 0
        for i, (codes, scales, x, u, y) in enumerate(items):
            _need(scales, torch.float32, "scales")
            N, K = _codes_shape(codes, scales.numel())
            _need(x, torch.float32, "x")
            if u is not None:
                _need(u, torch.float32, "u")
            _need(y, torch.float32, "y")
            self.descs[i] = F32Desc(codes.data_ptr(), scales.data_ptr(), x.data_ptr(),
                                    u.data_ptr() if u is not None else None, y.data_ptr(), N, K)
            total += gemv_f32_workspace_bytes(N, K, B)
        self.items = items
        dev = items[0][2].device
        self.ws = torch.empty(max(total, 256), dtype=torch.uint8, device=dev) if ws is None else ws
        self.args = (ctypes.cast(self.descs, ctypes.c_void_p), n, B, _ptr(self.ws),
                     self.ws.numel())
        self.device = dev

    def __call__(self, stream=None):
        s = ctypes.c_void_p(stream if stream is not None
                            else _stream_handle(self.device))
        _check(lib().sherry_gemv_f32_grouped(*self.args, s), "sherry_gemv_f32_grouped")


def gemv_f32_grouped(items, B, ws=None):
    """items: list of (codes, scales, x fp32 [B, K], u fp32 [B, K] or None, y [B, N])."""
    GroupedGemvF32(items, B, ws)()


class GroupedGemv:
    """Pre-marshalled grouped GEMV: descriptors and workspace are built once, and
    each call only passes them to the library (used where per-call Python cost
    matters, e.g. timing a decode step)."""

    def __init__(self, items, B, ws=None):
        n = len(items)
        self.descs = (GemvDesc * n)()
        total = 0
        for i, (codes, scales, x, y) in enumerate(items):
            _need(scales, torch.float32, "scales")
            N, K = _codes_shape(codes, scales.numel())
            _need(x, torch.int8, "x")
            _need(y, torch.float32, "y")
            self.descs[i] = GemvDesc(codes.data_ptr(), scales.data_ptr(), x.data_ptr(),
                                     y.data_ptr(), N, K)
            total += gemv_workspace_bytes(N, K, B)
        self.items = items  # keep the tensors alive
        self.n, self.B = n, B
        dev = items[0][2].device
        self.ws = torch.empty(max(total, 256), dtype=torch.uint8, device=dev) if ws is None else ws
        self.args = (ctypes.cast(self.descs, ctypes.c_void_p), n, B, _ptr(self.ws),
                     self.ws.numel())
        self.device = dev

    def __call__(self, stream=None):
        s = ctypes.c_void_p(stream if stream is not None
                            else _stream_handle(self.device))
        _check(lib().sherry_gemv_grouped(*self.args, s), "sherry_gemv_grouped")

    def prepare(self, stream=None):
        s = ctypes.c_void_p(stream if stream is not None
                            else _stream_handle(self.device))
        _check(lib().sherry_gemv_prepare(*self.args, s), "sherry_gemv_prepare")

    def run(self, stream=None):
        s = ctypes.c_void_p(stream if stream is not None
                            else _stream_handle(self.device))
        _check(lib().sherry_gemv_run(*self.args, s), "sherry_gemv_run")


class GroupedGemvBf16:
    """Pre-marshalled grouped GEMV on bf16 activations (sherry_gemv_bf16_grouped):
    items are (codes, scales, x bf16 [B, K], y [B, N])."""

    def __init__(self, items, B, ws=None):
        n = len(items)
        self.descs = (GemvDesc * n)()  # same field layout as sherry_gemv_bf16_desc
        total = 0
        for i, (codes, scales, x, y) in enumerate(items):
            _need(scales, torch.float32, "scales")
            N, K = _codes_shape(codes, scales.numel())
            _need(x, torch.bfloat16, "x")
            _need(y, torch.float32, "y")
            self.descs[i] = GemvDesc(codes.data_ptr(), scales.data_ptr(), x.data_ptr(),
                                     y.data_ptr(), N, K)
            total += gemv_bf16_workspace_bytes(N, K, B)
        self.items = items
        dev = items[0][2].device
        self.ws = torch.empty(max(total, 256), dtype=torch.uint8, device=dev) if ws is None else ws
        self.args = (ctypes.cast(self.descs, ctypes.c_void_p), n, B, _ptr(self.ws),
                     self.ws.numel())
        self.device = dev

    def __call__(self, stream=None):
        s = ctypes.c_void_p(stream if stream is not None
                            else _stream_handle(self.device))
        _check(lib().sherry_gemv_bf16_grouped(*self.args, s), "sherry_gemv_bf16_grouped")


def gemm(codes, scales, x, y=None):
    """y[M, N] = scales * (x . W^T); x int8 [M, K]."""
    _need(scales, torch.float32, "scales")
    N, K = _codes_shape(codes, scales.numel())
    _need(x, torch.int8, "x")
    M = x.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    _check(lib().sherry_gemm(_ptr(codes), _ptr(scales), _ptr(x), _ptr(y), M, N, K, _stream(x)),
           "sherry_gemm")
    return y


def gemm_acc(codes, x, N, acc=None):
    """Exact int32 accumulators acc[M, N] = x . W^T."""
    N, K = _codes_shape(codes, N)
    _need(x, torch.int8, "x")
    M = x.shape[0]
    if acc is None:
        acc = torch.empty((M, N), dtype=torch.int32, device=x.device)
    _check(lib().sherry_gemm_acc(_ptr(codes), _ptr(x), _ptr(acc), M, N, K, _stream(x)),
           "sherry_gemm_acc")
    return acc


def device_error():
    """Synchronise and return (and clear) the device-side error word (0 = none)."""
    return int(lib().sherry_device_error())


def set_wait_limit(cycles):
    """Limit (SM clock cycles) of the kernels' bounded barrier waits, for
    kernels launched afterwards by this process; 0 restores the default."""
    _check(lib().sherry_set_wait_limit(int(cycles)), "sherry_set_wait_limit")


# ----------------------------------------------------------------------------- comparison formats
CMP_I2 = 1  # 2 bits per weight, aligned
CMP_T3 = 2  # three weights in five bits
_CMP_TILE_WORDS = {CMP_I2: 8, CMP_T3: 5}


def cmp_tiles(fmt, K):
    if fmt == CMP_I2:
        return K // TILE_K
    return 2 * ((K + 191) // 192)


def cmp_transcode(fmt, codes, N):
    """Sherry codes of an N x K matrix -> the same matrix in comparison format
    fmt, int32 [ceil(N/32), tiles, words, 32] holding the uint32 words."""
    N, K = _codes_shape(codes, N)
    shape = ((N + 31) // 32, cmp_tiles(fmt, K), _CMP_TILE_WORDS[fmt], 32)
    out = torch.empty(shape, dtype=torch.int32, device=codes.device)
    assert out.numel() * 4 == lib().sherry_cmp_packed_bytes(fmt, N, K)
    _check(lib().sherry_cmp_transcode(fmt, _ptr(codes), N, K, _ptr(out), _stream(codes)),
           "sherry_cmp_transcode")
    return out


def cmp_gemv_acc(fmt, codes, x, N, K, acc=None):
    """Exact int32 acc[B, N] of a comparison-format matrix against int8 x [B, K]."""
    _need(x, torch.int8, "x")
    x2 = x.view(1, -1) if x.dim() == 1 else x
    B = x2.shape[0]
    if acc is None:
        acc = torch.empty((B, N), dtype=torch.int32, device=x.device)
    nb = lib().sherry_cmp_workspace_bytes(fmt, N, K, B)
    ws = workspace(max(nb, 256), x.device)
    _check(lib().sherry_cmp_gemv_acc(fmt, _ptr(codes), _ptr(x2), _ptr(acc), N, K, B, _ptr(ws),
                                     ws.numel(), _stream(x)), "sherry_cmp_gemv_acc")
    return acc


class GroupedCmpGemv:
    """Pre-marshalled grouped GEMV on comparison-format matrices: items are
    (codes in format fmt, scales, x int8 [B, K], y [B, N], K)."""

    def __init__(self, fmt, items, B):
        n = len(items)
        self.descs = (GemvDesc * n)()
        total = 0
        for i, (codes, scales, x, y, K) in enumerate(items):
            _need(scales, torch.float32, "scales")
            _need(x, torch.int8, "x")
            _need(y, torch.float32, "y")
            N = scales.numel()
            self.descs[i] = GemvDesc(codes.data_ptr(), scales.data_ptr(), x.data_ptr(),
                                     y.data_ptr(), N, K)
            total += lib().sherry_cmp_workspace_bytes(fmt, N, K, B)
        self.items = items
        dev = items[0][2].device
        self.ws = torch.empty(max(total, 256), dtype=torch.uint8, device=dev)
        self.args = (fmt, ctypes.cast(self.descs, ctypes.c_void_p), n, B, _ptr(self.ws),
                     self.ws.numel())
        self.device = dev

    def __call__(self, stream=None):
        s = ctypes.c_void_p(stream if stream is not None
                            else _stream_handle(self.device))
        _check(lib().sherry_cmp_gemv_grouped(*self.args, s), "sherry_cmp_gemv_grouped")


def probe_mma_i8(iters, stream=None):
    """Launch the tensor-core int8 probe; returns the number of CTAs (one per
    SM).  Each CTA runs iters * 4 MMAs of 128 x 256 x 32."""
    ctas = ctypes.c_int(0)
    s = ctypes.c_void_p(stream if stream is not None else torch.cuda.current_stream().cuda_stream)
    _check(lib().sherry_probe_mma_i8(int(iters), ctypes.byref(ctas), s), "sherry_probe_mma_i8")
    return ctas.value
