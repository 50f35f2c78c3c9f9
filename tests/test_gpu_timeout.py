"""The device-side timeout path of the tensor-core scan, run without any fault.

Every wait of the tensor-path kernels is bounded: after its budget it raises
a CTA-wide abort flag, every other wait of the CTA gives up at once, the CTA
lets the copies and MMAs it already issued finish, releases its tensor
memory, records SSD_ERR_DEVICE_TIMEOUT in the workspace's status word and
returns.  The test hook ssd_set_test_fault(1) makes one expected arrival
never happen (the chunk-output kernel does not request its first C and B
tiles) and shortens every wait to about 2^21 cycles, so that path runs in a
few milliseconds.  The GPU stays usable: the next normal call on it matches
the oracle.
"""
import math
import time

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import TOL_BF16, compare, run_scan
from state_space_sequence_scan_b200 import ssd
from state_space_sequence_scan_b200.inputs import ScanConfig, make_scan_inputs

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_is_reported():
    cfg = ScanConfig("timeout", 1, 600, 4, 64, 128, 2, 128, "bf16", "ones", "normal", seed=81)
    inp = make_scan_inputs(cfg)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    ws = ssd.alloc_workspace(ssd.workspace_size(1, 600, 4, 64, 128, 2, 128, torch.bfloat16, "tensor"), "cuda")
    ssd.set_test_fault(1)
    try:
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        ssd.chunk_scan_fwd(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                           init_state=d["init_state"], chunk_size=128, path="tensor", workspace=ws)
        status = ssd.read_device_status(ws)          # synchronises the stream
        elapsed = time.perf_counter() - t0
    finally:
        ssd.set_test_fault(0)
    assert status == 6, "expected SSD_ERR_DEVICE_TIMEOUT, got %d" % status
    # every wait gave up through the abort flag: the call ended in well under
    # the 2^32-cycle budget of a single normal wait (about 2 s)
    assert elapsed < 0.5, "the timed-out call took %.3f s" % elapsed
    # the context is intact: a normal call on the same GPU matches the oracle
    y, fs = run_scan(inp, 128, path="tensor")
    yr, fr = oracle.scan(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"],
                         init_state=inp["init_state"])
    compare(y, yr, TOL_BF16, "after the timeout y")
    compare(fs, fr, TOL_BF16, "after the timeout final_state")
