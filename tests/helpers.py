"""Test-side helpers: input construction only (no arithmetic of the method).

`ternary_latents` builds fp32 latent weights whose 3:4 prune is known in
advance: kept entries have |w| in [1, 1.5), the designated zero of each block
has |w| < 0.5.  The expected ternary matrix is the input pattern itself.
"""
import itertools
import json
import os

import numpy as np

VALID_BLOCKS = [b for b in itertools.product((-1, 0, 1), repeat=4) if b.count(0) == 1]


def random_ternary(N, K, rng):
    """Random 3:4 ternary matrix [N, K] (exactly one zero per 4-block)."""
    T = rng.choice([-1, 1], size=(N, K)).astype(np.int8)
    zpos = rng.integers(0, 4, size=(N, K // 4))
    T.reshape(N, K // 4, 4)[np.arange(N)[:, None], np.arange(K // 4)[None, :], zpos] = 0
    return T


def ternary_latents(T, rng):
    """fp32 latents whose prune gives exactly T."""
    mag = rng.uniform(1.0, 1.5, size=T.shape)
    small = rng.uniform(0.0, 0.5, size=T.shape) * rng.choice([-1, 1], size=T.shape)
    return np.where(T == 0, small, T * mag).astype(np.float32)


def load_tiles(golden_dir):
    with open(os.path.join(golden_dir, "tiles.json")) as f:
        spec = json.load(f)
    tiles = []
    for t in spec["tiles"]:
        lat = np.zeros((32, 4), np.float32)
        dense = []
        for j in range(32):
            if t.get("cyclic"):
                blk = [1.0] * 4
                blk[j % 4] = 0.0
            else:
                blk = t["overrides"].get(str(j), t["default"]) if "overrides" in t else t["default"]
            lat[j] = blk
            pat = t["dense_block_pattern"][j % len(t["dense_block_pattern"])]
            pat = t.get("dense_overrides", {}).get(str(j), pat)
            dense.extend({"+": 1, "-": -1, "0": 0}[c] for c in pat)
        tiles.append(dict(
            name=t["name"], latent=lat.reshape(128), dense=np.array(dense, np.int8),
            words=[int(w, 16) for w in t["words"]],
            scale=np.float32(t["scale_num"] / t["scale_den"])))
    return tiles


def ulp_diff_f32(a, b):
    """Distance in units in the last place between float32 arrays of one sign."""
    ai = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    bi = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    return np.abs(ai - bi)
