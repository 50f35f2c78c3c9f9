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


def stack_chains(inp, chains):
    """The (b, h) chains of a scan input as the heads of one batch row, each
    head its own group (its chain's B and C): one oracle call threads over all
    of them.  Pure indexing."""
    H = inp["x"].shape[2]
    G = inp["B"].shape[2]
    bs = [bi for bi, _ in chains]
    hs = [h for _, h in chains]
    gs = [h // (H // G) for h in hs]
    out = dict(x=torch.stack([inp["x"][bi, :, h] for bi, h in chains], 1)[None],
               dt_raw=torch.stack([inp["dt_raw"][bi, :, h] for bi, h in chains], 1)[None],
               B=torch.stack([inp["B"][bi, :, g] for bi, g in zip(bs, gs)], 1)[None],
               C=torch.stack([inp["C"][bi, :, g] for bi, g in zip(bs, gs)], 1)[None],
               dt_bias=inp["dt_bias"][hs], A=inp["A"][hs], D=inp["D"][hs])
    out["init_state"] = None if inp["init_state"] is None else torch.stack(
        [inp["init_state"][bi, h] for bi, h in chains], 0)[None]
    return {k: (v.contiguous() if isinstance(v, torch.Tensor) else v) for k, v in out.items()}


class StreamingCompare:
    """max|gpu - oracle| / RMS(oracle) over a tensor checked in pieces: the
    largest error and the sum of squares are accumulated, the bar applied to
    the whole."""

    def __init__(self, tol, what):
        self.tol, self.what = tol, what
        self.maxerr, self.sumsq, self.n = 0.0, 0.0, 0

    def add(self, got, ref):
        got = np.asarray(got, dtype=np.float64)
        ref = np.asarray(ref, dtype=np.float64)
        assert got.shape == ref.shape, (got.shape, ref.shape)
        assert np.isfinite(got).all(), "%s: non-finite output" % self.what
        self.maxerr = max(self.maxerr, float(np.max(np.abs(got - ref))) if got.size else 0.0)
        self.sumsq += float(np.sum(ref * ref))
        self.n += ref.size

    def check(self):
        rms = math.sqrt(self.sumsq / max(self.n, 1))
        rel = self.maxerr / rms if rms > 0 else self.maxerr
        assert rel <= self.tol, "%s: max|err|/RMS = %.3e > %.1e" % (self.what, rel, self.tol)
        return rel


def spread_chains(batch, heads, per_batch, stride=13):
    """per_batch heads of every batch row, spread over all heads and over the
    head positions inside a group (row bi starts at a different offset)."""
    out = []
    for bi in range(batch):
        for j in range(per_batch):
            out.append((bi, (bi * stride + j * max(1, heads // per_batch) + j) % heads))
    return sorted(set(out))
