"""vdit_attn: bf16 video-DiT attention forward for B200 (sm_100a).

The compute path is the C-ABI library ``libvdit_attn.so`` built from
``csrc/``; :mod:`.binding` marshals torch tensors into its calls and raises if
the library is missing.  :mod:`.workloads` draws the seeded synthetic inputs.
"""
from .workloads import (  # noqa: F401
    MASK_BLOCK_CAUSAL,
    MASK_CROSS,
    MASK_FULL,
    WORKLOADS,
    workload_inputs,
)
from .flops import allowed_pairs, attn_flops, attn_min_bytes  # noqa: F401
