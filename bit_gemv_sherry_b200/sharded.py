"""Row-sharded decode GEMV across the ranks of a process group.

Output rows are independent (each y[b][n] is one row of codes against x), so
a matrix too large for one GPU, or a layer split for latency, can be cut by
rows: every rank holds a contiguous run of whole 32-row groups of the code
layout (a contiguous slice of the codes buffer) with their scales, runs the
library's GEMV on the replicated activations, and one all-gather of y
completes the product.  The all-gather is the only exchange; it moves
4 * B * N bytes per call (NCCL over NVLink on GPUs; gloo on CPU in tests).

The split is balanced by groups: with G = ceil(N / 32) groups and W ranks,
rank r holds groups [r * G // W, (r + 1) * G // W).  Ranks with fewer groups
pad their y to the largest share, so the gather has equal parts; the result
is re-assembled in row order (a view at B = 1 when every share is equal).
"""
import torch

from . import sherry as S

GROUP = 32  # rows per group of the code layout


def group_range(N, rank, world):
    """Groups [g0, g1) held by `rank` of `world` for an N-row matrix."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank %d not in a world of %d" % (rank, world))
    G = (N + GROUP - 1) // GROUP
    return rank * G // world, (rank + 1) * G // world


def row_range(N, rank, world):
    """Output rows [n0, n1) held by `rank` (whole groups; the last one may be partial)."""
    g0, g1 = group_range(N, rank, world)
    return min(N, g0 * GROUP), min(N, g1 * GROUP)


def max_share_rows(N, world):
    """Rows of the largest share, padded to whole groups (the gather's part size)."""
    G = (N + GROUP - 1) // GROUP
    return -(-G // world) * GROUP


def shard(codes, scales, rank, world):
    """This rank's slice of a packed matrix: (codes [g1-g0][T][5][32], scales [n1-n0],
    (n0, n1)).  `codes` is laid out as sherry_pack writes it; both slices are views."""
    N = scales.numel()
    g0, g1 = group_range(N, rank, world)
    n0, n1 = row_range(N, rank, world)
    return codes[g0:g1], scales[n0:n1], (n0, n1)


class ShardedGemv:
    """y[B][N] = s (.) (W . x^T) with W's rows spread over the ranks of `group`.

    codes, scales: this rank's shard (see `shard`); N: rows of the whole
    matrix.  `local_gemv(codes, scales, x, y)` computes the shard's y; the
    default is the library's sherry_gemv (the CUDA path).  Call with the same
    x on every rank; every rank gets the whole y.
    """

    def __init__(self, codes, scales, N, K, B, group=None, local_gemv=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.N, self.K, self.B = N, K, B
        self.n0, self.n1 = row_range(N, self.rank, self.world)
        self.codes, self.scales = codes, scales
        self.part = max_share_rows(N, self.world)
        self.local_gemv = local_gemv or S.gemv
        dev = scales.device
        # this rank's part of the gather, padded to the largest share
        self.y_part = torch.zeros((B, self.part), dtype=torch.float32, device=dev)
        # gathered parts, [world * B][part] (rank-major, as the collective concatenates)
        self.y_all = torch.empty((self.world * B, self.part), dtype=torch.float32, device=dev)
        self.shares = [row_range(N, r, self.world) for r in range(self.world)]
        self.equal = all(n1 - n0 == self.part for n0, n1 in self.shares)

    def __call__(self, x):
        rows = self.n1 - self.n0
        if rows > 0:
            if self.B == 1:   # the part's first `rows` values are contiguous: write in place
                self.local_gemv(self.codes, self.scales, x, self.y_part[:, :rows])
            else:
                y = self.local_gemv(self.codes, self.scales, x, None)
                self.y_part[:, :rows].copy_(y)
        self.dist.all_gather_into_tensor(self.y_all, self.y_part, group=self.group)
        if self.equal and self.B == 1:
            return self.y_all.view(1, self.N)
        # [world][B][part] -> [B][N]: each rank's valid rows, in rank order
        parts = self.y_all.view(self.world, self.B, self.part)
        return torch.cat([parts[r, :, :n1 - n0] for r, (n0, n1) in enumerate(self.shares)], dim=1)
