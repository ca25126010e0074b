"""Hybrid Linear Attention (HLA) over Gated DeltaNet on NVIDIA B200 (sm_100a).

The hot path lives in ``libhla.so`` (hand-written CUDA for sm_100a behind a C ABI,
``include/hla.h``); this package is its thin ctypes binding.  PyTorch is used only
for device memory and streams.
"""
from ._hla import (  # noqa: F401
    Cache,
    HlaConfig,
    HlaError,
    cache_bytes,
    decode_workspace_bytes,
    gdn_chunk_transitions,
    hla_decode_step,
    hla_decode_step_static,
    hla_check_bounded_wait,
    hla_device_status,
    hla_prefill,
    hla_profile_enable,
    hla_profile_read,
    hla_routing,
    lib,
    make_config,
    prefill_workspace_bytes,
)
