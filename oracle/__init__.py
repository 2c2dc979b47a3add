"""fp64 CPU oracle for the video-DiT attention forward pass.

TEST INFRASTRUCTURE ONLY.  Imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py``; the product package never
imports it, and it shares no code with the CUDA library.
"""
from .oracle import (  # noqa: F401
    MASK_BLOCK_CAUSAL,
    MASK_BLOCK_SPARSE,
    MASK_CROSS,
    MASK_FULL,
    attention,
    build,
    max_threads,
    rms_norm,
    round_to_bf16_bits,
    SPARSE_BLOCK,
)
