"""QLoRA NF4 frozen-base linear layer on B200 (sm_100a).

The hot path lives in libqlora_nf4.so (C ABI: include/qlora_nf4.h), built
in-tree by ``bit_nf4_quantized_19_b200.build``.  This package only marshals
torch tensors into that ABI; importing it does not load the library, calling
any op does, and fails loudly if the library is missing.
"""
from .api import (  # noqa: F401
    NF4Weight,
    nf4_levels,
    nf4_bytes,
    nf4_empty,
    nf4_empty_single,
    nf4_quantize,
    nf4_dequant,
    nf4_merge,
    workspace_bytes,
    make_workspace,
    pack_keep_mask,
    linear_fwd,
    linear_bwd,
    device_status,
    selftest_wait_timeout,
    set_wait_limit_us,
    set_gemm_pairing,
    gemm_units,
    profile_enable,
    profile_read,
)

__all__ = [
    "NF4Weight", "nf4_levels", "nf4_bytes", "nf4_empty", "nf4_empty_single", "nf4_quantize", "nf4_dequant", "nf4_merge",
    "workspace_bytes", "make_workspace", "pack_keep_mask", "linear_fwd", "linear_bwd", "device_status",
    "selftest_wait_timeout", "set_wait_limit_us", "set_gemm_pairing", "gemm_units", "profile_enable", "profile_read",
]
