"""B200-native Mamba-2 SSD scan: chunked forward and decode step (sm_100a).

The compute lives in libssd.so (C ABI in include/ssd.h); ``ssd`` is its
Python binding.  ``inputs`` holds the seeded synthetic workloads.
"""
from . import inputs  # noqa: F401
from .ssd import (  # noqa: F401
    SSDError,
    alloc_workspace,
    chunk_scan_fwd,
    load_library,
    read_device_status,
    step,
    workspace_size,
)
