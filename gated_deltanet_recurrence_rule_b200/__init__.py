"""Gated DeltaNet recurrence (the gated delta rule) on NVIDIA B200 (sm_100a).

The compute lives in ``libgdn.so`` (hand-written CUDA behind a C ABI declared
in ``include/gdn.h``); this package is the thin Python binding over it plus
the seeded input generator.  Importing the package does not load the CUDA
library; the first call does, and fails loudly if it is missing.
"""
from .api import (  # noqa: F401
    GDN_INPUT_PREPARED,
    GDN_INPUT_RAW,
    GDNError,
    decode_step,
    decode_tokens,
    get_device_status,
    lib_path,
    prefill,
    prefill_backward,
    prefill_backward_workspace_size,
    prefill_launch_count,
    prefill_uses_tensor_cores,
    prefill_workspace_size,
)

__all__ = ["prefill", "prefill_backward", "decode_step", "decode_tokens", "prefill_workspace_size",
           "prefill_backward_workspace_size", "prefill_launch_count", "prefill_uses_tensor_cores",
           "get_device_status", "GDNError", "GDN_INPUT_PREPARED", "GDN_INPUT_RAW", "lib_path"]
