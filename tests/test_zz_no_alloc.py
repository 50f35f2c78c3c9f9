"""The allocation-free scan entry point, checked against the workspace one.

ssd_chunk_scan_fwd_noalloc serves callers that cannot allocate device memory
(code where cudaMalloc is forbidden or unsafe, or that only receives its input
and output buffers): its scratch is a fixed device array inside libssd.so.
Both entry points run the same deterministic kernels on the same inputs, so
their outputs must agree bit for bit; a difference would mean the shared array
carried something over from an earlier call.  This file is collected last so
that a run stopping at the first failure has already run every other test; it
also passes on its own in a fresh process.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from state_space_sequence_scan_b200 import ssd
from state_space_sequence_scan_b200.inputs import ScanConfig, make_scan_inputs

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    lib = ssd.load_library()
    f = lib.ssd_chunk_scan_fwd_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 10 + [ctypes.c_int64] * 7 + [ctypes.c_float, ctypes.c_float, ctypes.c_int,
                                                                  ctypes.c_int, ctypes.c_void_p]
    return f


def _call_noalloc(f, d, y, fs, Q, path=0):
    b, L, H, P = d["x"].shape
    G, N = d["B"].shape[2], d["B"].shape[3]
    p = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return f(p(d["x"]), p(d["dt_raw"]), p(d["dt_bias"]), p(d["A"]), p(d["B"]), p(d["C"]), p(d["D"]),
             p(d["init_state"]), p(y), p(fs), b, L, H, P, N, G, Q, 0.0, math.inf, ssd.DTYPES[d["x"].dtype], path,
             stream)


# (dtype, path) pairs: the tensor-core path (bf16, auto) and the SIMT path's
# carve-up of the shared array, with bf16 and with fp32 inputs
CASES = [("bf16", "auto", 128), ("bf16", "simt", 100), ("f32", "simt", 64)]


@pytest.mark.parametrize("dtype,path,Q", CASES)
def test_noalloc_matches_workspace_entry_twice(dtype, path, Q):
    f = _noalloc_fn()
    cfg = ScanConfig("noalloc", 2, 1000, 8, 64, 128, 2, Q, dtype, "ones", "normal", seed=21)
    d = {k: (v.cuda() if v is not None else None) for k, v in make_scan_inputs(cfg).items()}
    y_ref, fs_ref = ssd.chunk_scan_fwd(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                                       init_state=d["init_state"], chunk_size=Q, path=path)
    y_ref = y_ref.cpu().numpy()
    fs_ref = fs_ref.cpu().numpy()
    for _ in range(2):                      # the shared array keeps the previous call's contents
        y = torch.full((2, 1000, 8, 64), float("nan"), device="cuda")
        fs = torch.full((2, 8, 128, 64), float("nan"), device="cuda")
        assert _call_noalloc(f, d, y, fs, Q, ssd.PATHS[path]) == 0
        torch.cuda.synchronize()
        assert np.array_equal(y.cpu().numpy(), y_ref), "noalloc y differs from the workspace entry's"
        assert np.array_equal(fs.cpu().numpy(), fs_ref), "noalloc final_state differs from the workspace entry's"


def test_noalloc_allocates_nothing():
    """After one warm-up call (which resolves the array's address), a call
    leaves the device's free memory and PyTorch's allocator untouched."""
    f = _noalloc_fn()
    cfg = ScanConfig("noalloc_mem", 1, 700, 4, 64, 128, 1, 128, "bf16", "ones", "zero", seed=23)
    d = {k: (v.cuda() if v is not None else None) for k, v in make_scan_inputs(cfg).items()}
    y = torch.empty(1, 700, 4, 64, device="cuda")
    fs = torch.empty(1, 4, 128, 64, device="cuda")
    assert _call_noalloc(f, d, y, fs, 128) == 0
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for _ in range(3):
        assert _call_noalloc(f, d, y, fs, 128) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0, "device free memory changed by %d bytes" % (free0 - free1)


def test_noalloc_rejects_oversized_work():
    f = _noalloc_fn()
    # shapes only: the size check runs on the host before anything is enqueued
    x = torch.empty(8, 4096, 80, 64, dtype=torch.bfloat16, device="cuda")
    Bm = torch.empty(8, 4096, 1, 128, dtype=torch.bfloat16, device="cuda")
    h = torch.empty(80, device="cuda")
    d = dict(x=x, dt_raw=torch.empty(8, 4096, 80, device="cuda"), dt_bias=h, A=h, B=Bm, C=Bm, D=h, init_state=None)
    y = torch.empty(8, 4096, 80, 64, device="cuda")
    assert _call_noalloc(f, d, y, None, 256) == 2
