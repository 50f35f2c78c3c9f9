"""Shared helpers for the GPU parity tests (test code, not product code)."""
import math

import numpy as np
import torch

import oracle
from state_space_sequence_scan_b200 import ssd

# Tolerances: max|gpu - oracle| / RMS(oracle), per output tensor.
TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def tol_for(dtype) -> float:
    return TOL_F32 if dtype in (torch.float32, "f32") else TOL_BF16


def path_supported(inp, chunk_size, path) -> bool:
    """Whether the library accepts this shape on this path (host-side query)."""
    b, L, H, P = inp["x"].shape
    G, N = inp["B"].shape[2], inp["B"].shape[3]
    try:
        ssd.workspace_size(b, L, H, P, N, G, chunk_size, inp["x"].dtype, path)
        return True
    except ssd.SSDError:
        return False


def to_dev(inp, device="cuda"):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def run_scan(inp, chunk_size, path="auto", dt_limit=(0.0, math.inf), check_status=True):
    d = to_dev(inp)
    b, L, H, P = d["x"].shape
    G, N = d["B"].shape[2], d["B"].shape[3]
    ws = ssd.alloc_workspace(ssd.workspace_size(b, L, H, P, N, G, chunk_size, d["x"].dtype, path), "cuda")
    y, fs = ssd.chunk_scan_fwd(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                               init_state=d["init_state"], chunk_size=chunk_size, dt_limit=dt_limit,
                               path=path, workspace=ws)
    if check_status:
        st = ssd.read_device_status(ws)
        assert st == 0, "device status %d" % st
    torch.cuda.synchronize()
    return y.cpu().double().numpy(), fs.cpu().double().numpy()


def compare(got, ref, tol, what=""):
    rel_max, rel_l2 = oracle.ssd_oracle.max_err_over_rms(got, ref)
    assert np.isfinite(got).all(), "%s: non-finite output" % what
    assert rel_max <= tol, "%s: max|err|/RMS = %.3e > %.1e (rel L2 %.3e)" % (what, rel_max, tol, rel_l2)
    return rel_max, rel_l2


def sample_chains(inp, chains):
    """Slices (b, h) chains out of a scan input: each becomes batch 1, one
    head, one group (the head's own group's B and C).  Pure indexing."""
    H = inp["x"].shape[2]
    G = inp["B"].shape[2]
    out = []
    for (bi, h) in chains:
        g = h // (H // G)
        sub = dict(x=inp["x"][bi:bi + 1, :, h:h + 1], dt_raw=inp["dt_raw"][bi:bi + 1, :, h:h + 1],
                   dt_bias=inp["dt_bias"][h:h + 1], A=inp["A"][h:h + 1], D=inp["D"][h:h + 1],
                   B=inp["B"][bi:bi + 1, :, g:g + 1], C=inp["C"][bi:bi + 1, :, g:g + 1],
                   init_state=None if inp["init_state"] is None else inp["init_state"][bi:bi + 1, h:h + 1])
        out.append(sub)
    return out
