"""Gated DeltaNet recurrence (the gated delta rule) on NVIDIA B200 (sm_100a).

The compute lives in ``libgdn.so`` (hand-written CUDA behind a C ABI declared
in ``include/gdn.h``); this package is the thin Python binding over it plus
the seeded input generator.  Importing the package does not load the CUDA
library; the first call does, and fails loudly if it is missing.
"""
from .api import (  # noqa: F401
    GDNError,
    decode_step,
    get_device_status,
    lib_path,
    prefill,
    prefill_uses_tensor_cores,
    prefill_workspace_size,
)

__all__ = ["prefill", "decode_step", "prefill_workspace_size", "prefill_uses_tensor_cores", "get_device_status", "GDNError",
           "lib_path"]
