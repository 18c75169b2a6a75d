"""Shapes of the synthetic workloads (LLaMA-3.2-1B/3B linear layers).

(N out, K in) per projection.  These are plain data; no arithmetic of the
method lives here.
"""
# LLaMA-3.2-1B: hidden 2048, 8 KV heads x 64 = 512, MLP 8192.
LLAMA_1B_LAYERS = [
    ("q", 2048, 2048), ("k", 512, 2048), ("v", 512, 2048), ("o", 2048, 2048),
    ("gate", 8192, 2048), ("up", 8192, 2048), ("down", 2048, 8192),
]
# LLaMA-3.2-3B: hidden 3072, 8 KV heads x 128 = 1024, MLP 8192.
LLAMA_3B_LAYERS = [
    ("q", 3072, 3072), ("k", 1024, 3072), ("v", 1024, 3072), ("o", 3072, 3072),
    ("gate", 8192, 3072), ("up", 8192, 3072), ("down", 3072, 8192),
]
# Prefill GEMMs: (M tokens, N out, K in).
PREFILL_GEMMS = [("gate_up_like", 2048, 8192, 2048), ("down_like", 2048, 2048, 8192)]

PROJ_INDEX = {name: i for i, (name, _, _) in enumerate(LLAMA_1B_LAYERS)}


def layer_seed(layer, proj_index, base=0):
    """Weight seed of projection `proj_index` of decoder layer `layer`."""
    return base + layer * 7 + proj_index


def decode_stack(n_layers=16):
    """The 1B-shaped decode stack: list of (layer, name, N, K, weight_seed)."""
    out = []
    for layer in range(n_layers):
        for pi, (name, n, k) in enumerate(LLAMA_1B_LAYERS):
            out.append((layer, name, n, k, layer_seed(layer, pi)))
    return out
