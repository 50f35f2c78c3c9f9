"""fp64 CPU oracle for the Mamba-2 SSD scan and decode step.

TEST INFRASTRUCTURE ONLY: imported by the test suite, the smoke check and the
benchmark's CPU-baseline leg, never by the CUDA path.  See ``ssd_oracle.py``.
"""
from .ssd_oracle import (  # noqa: F401
    build_oracle,
    conv1d_silu,
    gated_rmsnorm,
    oracle_library_path,
    scan,
    scan_bwd,
    scan_states,
    scan_varlen,
    softplus,
    step,
)
