"""The C ABI library loads, exports every declared entry point, and rejects bad
arguments on the host before touching a GPU (no CUDA device needed)."""
import ctypes
import os
import re

import pytest

from bit_gemv_sherry_b200 import sherry as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sherry.h")
FAKE = ctypes.c_void_p(0x100000)      # never dereferenced: checks fail first
FAKE_WS = ctypes.c_void_p(0x200000)   # 256-aligned fake workspace


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sherry_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_function():
    L = S.lib()
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n


def test_status_strings_and_version():
    L = S.lib()
    for code in range(8):
        assert L.sherry_status_string(code)
    assert L.sherry_version() >= 100


def test_packed_and_workspace_sizes():
    assert S.packed_bytes(256, 1024) == 256 * 1024 * 5 // 32
    assert S.packed_bytes(1, 1024) == 32 * 1024 * 5 // 32      # rows padded to a 32-row group
    assert S.codes_shape(33, 2048) == (2, 16, 5, 32)
    assert S.packed_bytes(3, 100) == 0
    assert S.packed_bytes(0, 128) == 0
    # re-ordered activations (rows of K padded to 512; B >= 3 pads the batch
    # rows to groups of 4, or of 8 above B = 4) + partial sums and counters
    # up to 4 chunks per row: re-ordered activations only, no split-K region
    assert S.gemv_workspace_bytes(100, 384, 3) == 4 * 512
    assert S.gemv_workspace_bytes(100, 384, 4) == 4 * 512
    assert S.gemv_workspace_bytes(100, 384, 5) == 8 * 512
    assert S.gemv_workspace_bytes(100, 384, 9) == 16 * 512
    assert S.gemv_workspace_bytes(100, 384, 16) == 16 * 512
    assert S.gemv_workspace_bytes(40, 1024, 2) == 2 * 8 * 128
    assert S.gemv_workspace_bytes(2048, 2048, 1) == 2048
    # up to 16 chunks per row: one K-part, re-ordered activations only
    assert S.gemv_workspace_bytes(2048, 8192, 1) == 4 * 64 * 32
    assert S.gemv_workspace_bytes(100, 8192, 3) == 4 * 4 * 64 * 32
    # 34 chunks per row -> 3 K-parts: activations, then partial sums [B][N] and one
    # counter per 32-row unit, rounded to 256 bytes
    assert S.gemv_workspace_bytes(2048, 17408, 1) == 4 * 136 * 32 + 256 * ((4 * (2048 + 64) + 255) // 256)
    assert S.gemv_workspace_bytes(100, 17408, 3) == 4 * 4 * 136 * 32 + 256 * ((4 * (300 + 4) + 255) // 256)
    assert S.gemv_workspace_bytes(16, 128, 0) == 0


def test_pack_argument_checks():
    L = S.lib()
    assert L.sherry_pack(None, 4, 128, FAKE, FAKE, None) == 1
    assert L.sherry_pack(FAKE, 0, 128, FAKE, FAKE, None) == 2
    assert L.sherry_pack(FAKE, 4, 100, FAKE, FAKE, None) == 2
    assert L.sherry_pack(FAKE, 4, 131072 + 128, FAKE, FAKE, None) == 2
    assert L.sherry_pack(ctypes.c_void_p(0x100004), 4, 128, FAKE, FAKE, None) == 3


def test_pack_grouped_argument_checks():
    L = S.lib()
    d = (S.PackDesc * 2)()
    d[0] = S.PackDesc(0x100000, 0x100000, 0x100000, 4, 128)
    d[1] = S.PackDesc(0x100000, 0x100000, None, 4, 128)
    p = ctypes.cast(d, ctypes.c_void_p)
    assert L.sherry_pack_grouped(None, 1, None) == 1
    assert L.sherry_pack_grouped(p, 0, None) == 2
    assert L.sherry_pack_grouped(p, 129, None) == 4
    assert L.sherry_pack_grouped(p, 2, None) == 1      # desc 1 has no scales
    d[1] = S.PackDesc(0x100000, 0x100000, 0x100000, 4, 200)
    assert L.sherry_pack_grouped(p, 2, None) == 2      # K not a multiple of 128
    d[1] = S.PackDesc(0x100008, 0x100000, 0x100000, 4, 128)
    assert L.sherry_pack_grouped(p, 2, None) == 3      # w not 16-byte aligned


def test_gemv_argument_checks():
    L = S.lib()
    ws = 1 << 20
    assert L.sherry_gemv(None, FAKE, FAKE, FAKE, 4, 128, 1, FAKE_WS, ws, None) == 1
    assert L.sherry_gemv(FAKE, None, FAKE, FAKE, 4, 128, 1, FAKE_WS, ws, None) == 1
    assert L.sherry_gemv(FAKE, FAKE, FAKE, FAKE, 0, 128, 1, FAKE_WS, ws, None) == 2
    assert L.sherry_gemv(FAKE, FAKE, FAKE, FAKE, 4, 130, 1, FAKE_WS, ws, None) == 2
    assert L.sherry_gemv(FAKE, FAKE, FAKE, FAKE, 4, 128, 0, FAKE_WS, ws, None) == 2
    assert L.sherry_gemv(FAKE, FAKE, FAKE, FAKE, 4, 128, 17, FAKE_WS, ws, None) == 4
    assert L.sherry_gemv(FAKE, FAKE, ctypes.c_void_p(0x100002), FAKE, 4, 128, 1, FAKE_WS, ws,
                         None) == 3
    assert L.sherry_gemv(FAKE, FAKE, FAKE, FAKE, 4, 128, 1, None, ws, None) == 7
    assert L.sherry_gemv(FAKE, FAKE, FAKE, FAKE, 4, 128, 1, ctypes.c_void_p(0x200010), ws,
                         None) == 3
    assert L.sherry_gemv(FAKE, FAKE, FAKE, FAKE, 4, 1024, 2, FAKE_WS, 1024, None) == 7
    assert L.sherry_gemv(FAKE, FAKE, FAKE, FAKE, 4, 1024, 2, FAKE_WS,
                         S.gemv_workspace_bytes(4, 1024, 2) - 4, None) == 7
    assert L.sherry_gemv_acc(FAKE, FAKE, None, 4, 128, 1, FAKE_WS, ws, None) == 1


def test_gemv_static_argument_checks():
    L = S.lib()
    assert L.sherry_gemv_static(None, FAKE, FAKE, FAKE, 4, 128, 1, None) == 1
    assert L.sherry_gemv_static(FAKE, FAKE, FAKE, FAKE, 4, 130, 1, None) == 2
    assert L.sherry_gemv_static(FAKE, FAKE, FAKE, FAKE, 4, 128, 17, None) == 4
    # beyond the 4 MiB static scratch: rejected on the host with both sizes in the message
    # 2 MiB of activations plus 6.4 MB of K-part sums: beyond the 4 MiB array
    assert L.sherry_gemv_static(FAKE, FAKE, FAKE, FAKE, 100000, 131072, 16, None) == 7
    assert b"4194304" in L.sherry_last_error()


def test_activation_front_end_argument_checks():
    L = S.lib()
    assert L.sherry_quantize_act(None, 1, 128, FAKE, FAKE, None) == 1
    assert L.sherry_quantize_act(FAKE, 1, 12, FAKE, FAKE, None) == 2        # K % 8
    assert L.sherry_quantize_act(FAKE, 0, 128, FAKE, FAKE, None) == 2
    assert L.sherry_quantize_act(ctypes.c_void_p(0x100008), 1, 128, FAKE, FAKE, None) == 3
    ws = 1 << 20
    assert L.sherry_gemv_bf16(FAKE, FAKE, None, FAKE, 4, 128, 1, FAKE_WS, ws, None) == 1
    assert L.sherry_gemv_bf16(FAKE, FAKE, ctypes.c_void_p(0x100008), FAKE, 4, 128, 1, FAKE_WS, ws,
                              None) == 3                                  # bf16 x: 16-byte aligned
    assert L.sherry_gemv_bf16(FAKE, FAKE, FAKE, FAKE, 4, 128, 17, FAKE_WS, ws, None) == 4
    # the activation scales take 64 more words than the int8 workspace
    assert S.gemv_bf16_workspace_bytes(2048, 2048, 1) == S.gemv_workspace_bytes(2048, 2048, 1) + 256
    assert L.sherry_gemv_bf16(FAKE, FAKE, FAKE, FAKE, 4, 1024, 2, FAKE_WS,
                              S.gemv_workspace_bytes(4, 1024, 2), None) == 7


def test_fp32_front_end_argument_checks():
    L = S.lib()
    odd = ctypes.c_void_p(0x100008)
    assert L.sherry_quantize_f32(None, 1, 128, FAKE, FAKE, None) == 1
    assert L.sherry_quantize_f32(FAKE, 1, 136, FAKE, FAKE, None) == 2        # K % 128
    assert L.sherry_quantize_f32(FAKE, 0, 128, FAKE, FAKE, None) == 2
    assert L.sherry_quantize_f32(FAKE, 65537, 128, FAKE, FAKE, None) == 4
    assert L.sherry_quantize_f32(odd, 1, 128, FAKE, FAKE, None) == 3
    assert L.sherry_quantize_swiglu(FAKE, None, 1, 128, FAKE, FAKE, None) == 1
    assert L.sherry_quantize_swiglu(FAKE, odd, 1, 128, FAKE, FAKE, None) == 3
    ws = 1 << 20
    assert L.sherry_gemv_f32(FAKE, FAKE, None, FAKE, 4, 128, 1, FAKE_WS, ws, None) == 1
    assert L.sherry_gemv_f32(FAKE, FAKE, odd, FAKE, 4, 128, 1, FAKE_WS, ws, None) == 3
    assert L.sherry_gemv_f32(FAKE, FAKE, FAKE, FAKE, 4, 128, 17, FAKE_WS, ws, None) == 4
    assert L.sherry_gemv_swiglu(FAKE, FAKE, FAKE, None, FAKE, 4, 128, 1, FAKE_WS, ws, None) == 1
    assert L.sherry_gemv_swiglu(FAKE, FAKE, FAKE, odd, FAKE, 4, 128, 1, FAKE_WS, ws, None) == 3
    assert L.sherry_gemv_swiglu(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 100, 1, FAKE_WS, ws, None) == 2
    # the activation scales take 64 more words than the int8 workspace, as for bf16
    assert S.gemv_f32_workspace_bytes(2048, 8192, 1) == S.gemv_workspace_bytes(2048, 8192, 1) + 256
    assert L.sherry_gemv_f32(FAKE, FAKE, FAKE, FAKE, 4, 1024, 2, FAKE_WS,
                             S.gemv_workspace_bytes(4, 1024, 2), None) == 7
    d = (S.F32Desc * 2)()
    d[0] = S.F32Desc(0x100000, 0x100000, 0x100000, None, 0x100000, 16, 128)
    d[1] = S.F32Desc(0x100000, 0x100000, None, 0x100000, 0x100000, 16, 128)
    p = ctypes.cast(d, ctypes.c_void_p)
    assert L.sherry_gemv_f32_grouped(None, 1, 1, FAKE_WS, ws, None) == 1
    assert L.sherry_gemv_f32_grouped(p, 0, 1, FAKE_WS, ws, None) == 2
    assert L.sherry_gemv_f32_grouped(p, 129, 1, FAKE_WS, ws, None) == 4
    assert L.sherry_gemv_f32_grouped(p, 2, 1, FAKE_WS, ws, None) == 1    # desc 1 has no x
    d[1] = S.F32Desc(0x100000, 0x100000, 0x100000, 0x100008, 0x100000, 16, 128)
    assert L.sherry_gemv_f32_grouped(p, 2, 1, FAKE_WS, ws, None) == 3    # desc 1's u unaligned


def test_grouped_argument_checks():
    L = S.lib()
    d = (S.GemvDesc * 2)()
    d[0] = S.GemvDesc(0x100000, 0x100000, 0x100000, 0x100000, 16, 128)
    d[1] = S.GemvDesc(0x100000, 0, 0x100000, 0x100000, 16, 128)
    p = ctypes.cast(d, ctypes.c_void_p)
    assert L.sherry_gemv_grouped(None, 1, 1, FAKE_WS, 1 << 20, None) == 1
    assert L.sherry_gemv_grouped(p, 0, 1, FAKE_WS, 1 << 20, None) == 2
    assert L.sherry_gemv_grouped(p, 129, 1, FAKE_WS, 1 << 20, None) == 4
    assert L.sherry_gemv_grouped(p, 2, 1, FAKE_WS, 1 << 20, None) == 1    # desc 1 has no scales
    d[1] = S.GemvDesc(0x100000, 0x100000, 0x100000, 0x100000, 16, 200)
    assert L.sherry_gemv_grouped(p, 2, 1, FAKE_WS, 1 << 20, None) == 2


def test_gemm_argument_checks():
    L = S.lib()
    assert L.sherry_gemm(None, FAKE, FAKE, FAKE, 4, 4, 128, None) == 1
    assert L.sherry_gemm(FAKE, FAKE, FAKE, FAKE, 0, 4, 128, None) == 2
    assert L.sherry_gemm(FAKE, FAKE, FAKE, FAKE, 4, 4, 64, None) == 2
    assert L.sherry_gemm(FAKE, FAKE, ctypes.c_void_p(0x100008), FAKE, 4, 4, 128, None) == 3
    assert L.sherry_gemm_acc(FAKE, FAKE, None, 4, 4, 128, None) == 1


def test_python_binding_rejects_cpu_tensors():
    import torch
    with pytest.raises(TypeError):
        S.pack(torch.zeros(4, 128))


def test_wait_limit_setting_is_checked_and_restorable():
    L = S.lib()
    assert L.sherry_set_wait_limit(-1) == 2
    assert L.sherry_set_wait_limit(1000) == 0
    assert L.sherry_set_wait_limit(0) == 0


def test_cmp_argument_checks_on_the_host():
    L = S.lib()
    assert L.sherry_cmp_packed_bytes(1, 32, 1024) == 32 * 1024 * 2 // 8
    assert L.sherry_cmp_packed_bytes(2, 32, 1920) == 32 * 1920 * 5 // 3 // 8
    assert L.sherry_cmp_packed_bytes(3, 32, 1024) == 0 and L.sherry_cmp_packed_bytes(1, 32, 100) == 0
    assert L.sherry_cmp_workspace_bytes(1, 64, 2048, 1) == 0          # I2 reads x in place
    assert L.sherry_cmp_workspace_bytes(2, 64, 2048, 2) == 4 * 64 * ((2 * 22 * 32 + 63) // 64)
    acc = FAKE
    assert L.sherry_cmp_gemv_acc(3, FAKE, FAKE, acc, 32, 512, 1, FAKE_WS, 1 << 20, None) == 4
    assert L.sherry_cmp_gemv_acc(1, FAKE, FAKE, acc, 32, 512, 3, FAKE_WS, 1 << 20, None) == 4
    assert L.sherry_cmp_gemv_acc(1, FAKE, FAKE, acc, 32, 384, 1, FAKE_WS, 1 << 20, None) == 2
    assert L.sherry_cmp_gemv_acc(1, None, FAKE, acc, 32, 512, 1, FAKE_WS, 1 << 20, None) == 1
    assert L.sherry_cmp_gemv_acc(1, ctypes.c_void_p(0x100004), FAKE, acc, 32, 512, 1, FAKE_WS,
                                 1 << 20, None) == 3
    assert L.sherry_cmp_gemv_acc(2, FAKE, FAKE, acc, 32, 512, 1, FAKE_WS, 16, None) == 7
    assert L.sherry_cmp_transcode(5, FAKE, 32, 512, FAKE, None) == 4
    assert L.sherry_cmp_transcode(1, FAKE, 32, 500, FAKE, None) == 2
