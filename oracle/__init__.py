"""Plain CPU oracle for the Sherry 1.25-bit ternary format (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding) never touches it.  See ``sherry_oracle.c`` for the definitions
and the readings of the paper it follows.
"""
from .oracle import (  # noqa: F401
    build,
    packed_bytes,
    prune_block,
    block_code,
    code_weights,
    pack,
    unpack,
    quantize_act,
    quantize_f32,
    swiglu,
    gemv_act,
    bf16_bits,
    gemv_acc,
    gemv,
    gemm_acc,
    gemm,
    num_threads,
    set_num_threads,
    FMT_I2,
    FMT_T3,
    cmp_tiles,
    cmp_packed_bytes,
    t3_code,
    t3_weights,
    cmp_encode,
    cmp_unpack,
    cmp_gemv_acc,
)
