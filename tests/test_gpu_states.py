"""GPU parity of the chunk-boundary states (ssd_chunk_scan_fwd_states)
against the fp64 oracle's.

nnterp guide "Mamba-2", "The state after every token": the chunk scan holds
the state at every chunk boundary, states[:, c] is the state after token
min((c+1) Q, L) - 1 and states[:, -1] equals the final state.  Each
boundary state is the final state of a prefix of the sequence, so each one
meets the final-state bar on its own: max|gpu - oracle| / RMS(oracle) over
the [b, H, N, P] state of that boundary <= 1e-4 (fp32 inputs), <= 2e-2 (bf16
inputs).  (Over the whole [b, nc, H, N, P] tensor one RMS would not do: a
burst of large dt makes some boundaries' states tens of times the others'.)
The last chunk state and the final state come from the same registers, so
they must agree bit for bit, and y must not change when the states are
requested.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (TOL_BF16, compare, path_supported, run_scan, sample_chains, spread_chains, stack_chains,
                         to_dev, tol_for)
from state_space_sequence_scan_b200 import ssd
from state_space_sequence_scan_b200.inputs import SCAN_CONFIGS, ScanConfig, make_scan_inputs

pytestmark = pytest.mark.gpu


def run_states(inp, Q, path="auto"):
    d = to_dev(inp)
    b, L, H, P = d["x"].shape
    G, N = d["B"].shape[2], d["B"].shape[3]
    eff = "simt" if (path == "auto" and Q % 128) else path
    ws = ssd.alloc_workspace(ssd.workspace_size(b, L, H, P, N, G, Q, d["x"].dtype, eff), "cuda")
    y, fs, cs = ssd.chunk_scan_fwd_states(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                                          init_state=d["init_state"], chunk_size=Q, path=path, workspace=ws)
    assert ssd.read_device_status(ws) == 0
    torch.cuda.synchronize()
    return y.cpu().double().numpy(), fs.cpu().double().numpy(), cs.cpu().double().numpy()


def compare_states(got, ref, tol, what=""):
    """The final-state bar at every boundary c: states[:, c] against its own RMS."""
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), "%s: non-finite states" % what
    for c in range(ref.shape[1]):
        compare(got[:, c], ref[:, c], tol, "%s, boundary %d" % (what, c))


def oracle_states(inp, Q):
    return oracle.scan_states(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"],
                              chunk_size=Q, init_state=inp["init_state"])


CASES = [
    # b, L, H, P, N, G, Q, dtype, init
    (2, 700, 4, 64, 128, 2, 128, "bf16", "normal"),
    (1, 549, 8, 64, 128, 1, 256, "bf16", "normal"),
    (2, 3 * 64 + 5, 4, 64, 128, 2, 64, "f32", "normal"),
    (3, 77, 2, 16, 16, 1, 7, "f32", "zero"),
    (1, 50, 2, 8, 4, 2, 1, "f32", "normal"),             # every token a boundary
]


@pytest.mark.parametrize("path", ["auto", "simt", "tensor"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "b%d_L%d_H%d_P%d_N%d_G%d_Q%d_%s_%s" % c)
def test_chunk_states_parity(case, path):
    b, L, H, P, N, G, Q, dtype, init = case
    cfg = ScanConfig("states", b, L, H, P, N, G, Q, dtype, "normal", init, seed=50 + L)
    inp = make_scan_inputs(cfg)
    if not path_supported(inp, Q, path) or (path == "tensor" and Q % 128):
        pytest.skip("the %s path does not give the states of this shape" % path)
    y, fs, cs = run_states(inp, Q, path)
    yr, fr, sr = oracle_states(inp, Q)
    tol = tol_for(inp["x"].dtype)
    assert cs.shape == sr.shape == (b, (L + Q - 1) // Q, H, N, P)
    compare_states(cs, sr, tol, "chunk states")
    compare(y, yr, tol, "y")
    assert np.array_equal(cs[:, -1], fs)                   # same registers, same bits
    y0, fs0 = run_scan(inp, Q, path="simt" if (path == "auto" and Q % 128) else path)
    assert np.array_equal(y, y0) and np.array_equal(fs, fs0)


def test_skip_token_holds_the_state():
    """The guide's check on the GPU: dt = 0 at token 3 (chunk size 1) leaves
    the state after token 3 equal to the state after token 2, exactly."""
    cfg = ScanConfig("skip", 1, 10, 4, 16, 16, 2, 1, "f32", "normal", "normal", seed=61)
    inp = make_scan_inputs(cfg)
    inp["dt_raw"][:, 3, :] = -1.0e4                        # softplus underflows to exactly 0
    _, _, cs = run_states(inp, 1, "simt")
    assert np.array_equal(cs[:, 3], cs[:, 2])
    assert not np.array_equal(cs[:, 4], cs[:, 3])


def test_tensor_path_needs_whole_blocks():
    """The tensor path has no state inside a 128-token block: chunk size 64
    with states is refused on it before anything runs (auto moves to SIMT)."""
    cfg = ScanConfig("q64", 1, 256, 2, 64, 128, 1, 64, "bf16", "normal", "zero", seed=62)
    d = to_dev(make_scan_inputs(cfg))
    with pytest.raises(ssd.SSDError) as e:
        ssd.chunk_scan_fwd_states(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                                  chunk_size=64, path="tensor")
    assert e.value.status == 2


@pytest.mark.parametrize("name", ["c2_2p7b", "c3_long"])
def test_full_size_sampled_chain_states(name):
    """The whole workload on the tensor path with the states (c3: units of 47
    blocks, the split path); the oracle evaluates sampled chains together:
    64 spread over all batch rows and heads of c2, every fifth head of c3."""
    cfg = SCAN_CONFIGS[name]
    inp = make_scan_inputs(cfg)
    Q = cfg.chunk_size
    y, fs, cs = run_states(inp, Q, "tensor")
    assert np.isfinite(cs).all()
    assert np.array_equal(cs[:, -1], fs)
    chains = spread_chains(cfg.batch, cfg.nheads, 8) if cfg.batch > 1 else [(0, h) for h in range(0, cfg.nheads, 5)]
    for c0 in range(0, len(chains), 16):
        part = chains[c0:c0 + 16]
        _, fr, sr = oracle_states(stack_chains(inp, part), Q)
        for j, (bi, h) in enumerate(part):
            compare_states(cs[bi:bi + 1, :, h:h + 1], sr[:, :, j:j + 1], TOL_BF16,
                           "%s chain %s chunk states" % (name, (bi, h)))
            compare(fs[bi:bi + 1, h:h + 1], fr[:, j:j + 1], TOL_BF16, "%s chain %s final_state" % (name, (bi, h)))
