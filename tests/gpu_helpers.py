"""Shared helpers of the GPU parity tests (data movement only)."""
import numpy as np
import torch


def dev_codes(codes_np):
    return torch.from_numpy(np.ascontiguousarray(codes_np).view(np.int32)).cuda()


def host_codes(codes_t):
    return codes_t.cpu().numpy().view(np.uint32)


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def rows_subset(codes_np, rows):
    """Codes of a subset of output rows, re-grouped ([ceil(n/32)][T][5][32] layout)."""
    rows = np.asarray(rows)
    out = np.zeros(((len(rows) + 31) // 32, codes_np.shape[1], 5, 32), np.uint32)
    for j, r in enumerate(rows):
        out[j // 32, :, :, j % 32] = codes_np[r // 32, :, :, r % 32]
    return out


def assert_y_matches(y_gpu, y_ref):
    """y_gpu = fl32(s * acc) with one rounding; y_ref = s * acc exact in double.

    Bit-exact equality with the fp32 rounding of the exact value is required;
    the relative error is reported against the 1e-6 bound as well.
    """
    y = np.asarray(y_gpu, np.float32)
    ref32 = np.asarray(y_ref, np.float64).astype(np.float32)
    rel = np.abs(y.astype(np.float64) - y_ref) / np.maximum(np.abs(y_ref), 1e-300)
    rel[(y_ref == 0) & (y == 0)] = 0.0
    assert np.all(rel <= 1e-6), rel.max()
    assert np.array_equal(y, ref32)
