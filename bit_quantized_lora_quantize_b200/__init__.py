"""Frozen-NF4 linear layer with a LoRA adapter (QLoRA's data-parallel hot
path) for NVIDIA B200 (sm_100a).

The product is the C-ABI library ``libqlora.so`` (include/qlora.h) built from
``csrc/`` by ``build.py``; ``qlora`` is its thin Python binding and
``synthetic`` the seeded input generator used by tests and the benchmark;
``dp`` the data-parallel gradient bucket and ``paged`` the paged AdamW of the
adapters.
"""

from .qlora import (  # noqa: F401
    CODES,
    LIB_PATH,
    PackedNF4,
    QloraError,
    lib,
    new_workspace,
    qlora_check_status,
    qlora_codebook,
    qlora_get_wait_timeout,
    qlora_set_wait_timeout,
    qlora_silu_gate_bwd,
    qlora_silu_gate_fwd,
    qlora_dequantize_nf4,
    qlora_linear_bwd,
    qlora_linear_fwd,
    qlora_nf4_codebook,
    qlora_profile_start,
    qlora_profile_stop,
    qlora_quantize_nf4,
    qlora_workspace_bytes,
)
