"""GPU parity of the chunked scan (through the C ABI) against the fp64 oracle.

Bar: max|gpu - oracle| / RMS(oracle) <= 1e-4 for fp32 inputs and <= 2e-2 for
bf16 inputs (oracle fed the same bf16-rounded values), separately for y and
for final_state.  Small cases span several chunks/tiles and a ragged tail;
the full-size workloads are checked on sampled (batch, head) chains, each of
which the oracle evaluates alone (chains are independent).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (TOL_BF16, TOL_F32, StreamingCompare, compare, path_supported, run_scan, sample_chains,
                         spread_chains, stack_chains, to_dev, tol_for)
from state_space_sequence_scan_b200 import ssd
from state_space_sequence_scan_b200.inputs import SCAN_CONFIGS, ScanConfig, make_scan_inputs

pytestmark = pytest.mark.gpu

PATHS = ["auto", "simt", "tensor"]
BF16_PATHS = ["simt", "tensor"]


def _oracle(inp, dt_limit=(0.0, math.inf)):
    return oracle.scan(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"],
                       init_state=inp["init_state"], dt_limit=dt_limit)


def _check(inp, Q, path, dt_limit=(0.0, math.inf), what=""):
    if not path_supported(inp, Q, path):
        pytest.skip("the %s path does not cover this shape/dtype" % path)
    y, fs = run_scan(inp, Q, path=path, dt_limit=dt_limit)
    yr, fr = _oracle(inp, dt_limit)
    tol = tol_for(inp["x"].dtype)
    compare(y, yr, tol, what + " y")
    compare(fs, fr, tol, what + " final_state")
    return y, fs


@pytest.mark.parametrize("path", PATHS)
def test_tiny_fp32_config(path):
    cfg = SCAN_CONFIGS["c0_tiny_fp32"]
    _check(make_scan_inputs(cfg), cfg.chunk_size, path, what=cfg.name)


CASES = [
    # b, L, H, P, N, G, Q, dtype, init
    (2, 3 * 64 + 5, 4, 64, 128, 2, 64, "f32", "normal"),
    (2, 3 * 64 + 5, 4, 64, 128, 2, 64, "bf16", "normal"),
    (1, 2 * 256 + 37, 8, 64, 128, 1, 256, "bf16", "normal"),
    (2, 700, 6, 64, 128, 3, 128, "bf16", "zero"),
    (1, 300, 4, 32, 64, 4, 100, "f32", "normal"),        # G = H, odd chunk
    (3, 77, 2, 16, 16, 1, 7, "f32", "normal"),
    (1, 50, 2, 8, 4, 2, 1, "f32", "normal"),             # chunk 1: every token a boundary
    (1, 129, 2, 64, 128, 1, 128, "bf16", "normal"),      # one token past a chunk
    (2, 1, 4, 64, 128, 1, 256, "bf16", "normal"),        # one token
]


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("case", CASES, ids=lambda c: "b%d_L%d_H%d_P%d_N%d_G%d_Q%d_%s_%s" % c)
def test_small_parity(case, path):
    b, L, H, P, N, G, Q, dt, init = case
    cfg = ScanConfig("case", b, L, H, P, N, G, Q, dt, "normal", init, seed=sum(c for c in case if isinstance(c, int)) % 997)
    _check(make_scan_inputs(cfg), Q, path, what=str(case))


@pytest.mark.parametrize("path", BF16_PATHS)
def test_dt_limit_clamp(path):
    cfg = ScanConfig("clamp", 2, 300, 4, 64, 128, 2, 64, "bf16", "ones", "normal", seed=11)
    inp = make_scan_inputs(cfg)
    _check(inp, 64, path, dt_limit=(0.02, 0.3), what="clamp")


@pytest.mark.parametrize("path", BF16_PATHS)
def test_c1_130m_full(path):
    cfg = SCAN_CONFIGS["c1_130m"]
    _check(make_scan_inputs(cfg), cfg.chunk_size, path, what=cfg.name)


@pytest.mark.parametrize("path", BF16_PATHS)
def test_c2_full_size_64_chains(path):
    """The 2.7B-shaped layer, whole (the launch the benchmark times), against
    the oracle on 64 chains spread over all 8 batch rows, over the heads and
    over every head position inside the group; the bar over all of them."""
    cfg = SCAN_CONFIGS["c2_2p7b"]
    inp = make_scan_inputs(cfg)
    y, fs = run_scan(inp, cfg.chunk_size, path=path)
    assert np.isfinite(y).all() and np.isfinite(fs).all()
    chains = spread_chains(cfg.batch, cfg.nheads, 8)
    assert len(chains) == 64
    yr, fr = _oracle(stack_chains(inp, chains))
    cy, cf = StreamingCompare(TOL_BF16, "c2 y"), StreamingCompare(TOL_BF16, "c2 final_state")
    for j, (bi, h) in enumerate(chains):
        cy.add(y[bi, :, h], yr[0, :, j])
        cf.add(fs[bi, h], fr[0, j])
    cy.check()
    cf.check()


def test_c3_full_size_every_chain():
    """The long-context layer (one 65536-token row, 80 heads in 8 groups, 11
    units of 47 blocks each on the tensor path), every (batch, head) chain
    against the oracle, 16 chains per oracle call; the bar over the whole
    y and final_state."""
    cfg = SCAN_CONFIGS["c3_long"]
    inp = make_scan_inputs(cfg)
    d = to_dev(inp)
    b, L, H, P = d["x"].shape
    G, N = d["B"].shape[2], d["B"].shape[3]
    ws = ssd.alloc_workspace(ssd.workspace_size(b, L, H, P, N, G, cfg.chunk_size, d["x"].dtype, "tensor"), "cuda")
    y, fs = ssd.chunk_scan_fwd(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                               init_state=d["init_state"], chunk_size=cfg.chunk_size, path="tensor", workspace=ws)
    assert ssd.read_device_status(ws) == 0
    y = y.cpu().numpy()
    fs = fs.cpu().numpy()
    del d, ws
    cy, cf = StreamingCompare(TOL_BF16, "c3 y"), StreamingCompare(TOL_BF16, "c3 final_state")
    for h0 in range(0, H, 16):
        chains = [(0, h) for h in range(h0, min(H, h0 + 16))]
        yr, fr = _oracle(stack_chains(inp, chains))
        for j, (bi, h) in enumerate(chains):
            cy.add(y[bi, :, h], yr[0, :, j])
            cf.add(fs[bi, h], fr[0, j])
    cy.check()
    cf.check()


def test_diag_sub_blocks_straddle_the_exp_cap():
    """Per-token log decays of about -2 make the 31-step decay across a
    diagonal 32x32 sub-block straddle the cap (64) of the factored form:
    inside one 128-token block some sub-blocks take the factored path and
    some the one-exp-per-element path.  A = -1 and dt_raw chosen so that
    dt (the softplus of dt_raw + dt_bias) is 1.9 .. 2.3."""
    cfg = ScanConfig("cap", 2, 700, 4, 64, 128, 2, 128, "bf16", "ones", "normal", seed=71)
    inp = make_scan_inputs(cfg)
    g = torch.Generator().manual_seed(71)
    dt = 1.9 + 0.4 * torch.rand(cfg.batch, cfg.seqlen, cfg.nheads, generator=g, dtype=torch.float64)
    inp["A"][:] = -1.0
    inp["dt_bias"][:] = 0.0
    inp["dt_raw"] = (dt + torch.log(-torch.expm1(-dt))).float()       # softplus^-1(dt)
    # the decays really straddle the cap inside blocks (the kernel's flag test in fp32)
    da = -dt.float()
    cum = torch.cumsum(da.view(cfg.batch, -1, cfg.nheads), 1)
    spans = []
    for t0 in range(0, cfg.seqlen - 31, 32):
        spans.append((cum[:, t0] - cum[:, t0 + 31]).flatten())
    spans = torch.cat(spans)
    assert (spans <= 64).any() and (spans > 64).any()
    _check(inp, 128, "tensor", what="exp cap")
    _check(inp, 128, "simt", what="exp cap")


def test_chunk_size_invariance_fp32():
    cfg = ScanConfig("inv", 1, 512, 4, 64, 128, 2, 64, "f32", "normal", "normal", seed=5)
    inp = make_scan_inputs(cfg)
    ys = [run_scan(inp, Q, path="simt") for Q in (1, 16, 64, 200, 512)]
    yr, fr = _oracle(inp)
    y0, f0 = ys[2]
    for y, f in ys:
        compare(y, yr, TOL_F32, "y vs oracle")
        compare(f, fr, TOL_F32, "final_state vs oracle")
        compare(y, y0, TOL_F32, "y across chunk sizes")
        compare(f, f0, TOL_F32, "final_state across chunk sizes")


@pytest.mark.parametrize("path", BF16_PATHS)
def test_split_and_carry(path):
    cfg = ScanConfig("split", 2, 1000, 4, 64, 128, 1, 128, "bf16", "ones", "normal", seed=6)
    inp = make_scan_inputs(cfg)
    y, fs = run_scan(inp, 128, path=path)
    T1 = 389
    first = {k: (v[:, :T1] if k in ("x", "dt_raw", "B", "C") else v) for k, v in inp.items()}
    y1, h1 = run_scan(first, 128, path=path)
    second = {k: (v[:, T1:] if k in ("x", "dt_raw", "B", "C") else v) for k, v in inp.items()}
    second["init_state"] = torch.from_numpy(h1).float()
    y2, h2 = run_scan(second, 128, path=path)
    yr, fr = _oracle(inp)
    compare(np.concatenate([y1, y2], axis=1), yr, TOL_BF16, "split y")
    compare(h2, fr, TOL_BF16, "split final_state")
    compare(y, yr, TOL_BF16, "whole y")


def test_skip_token():
    """dt = 0 exactly (softplus underflow): the token writes nothing and decays
    nothing, so the rest of the sequence sees what it would without it."""
    cfg = ScanConfig("skip", 1, 300, 4, 64, 128, 1, 64, "f32", "ones", "normal", seed=7)
    inp = make_scan_inputs(cfg)
    t = 130
    inp["dt_raw"][:, t] = -1.0e4
    y, fs = run_scan(inp, 64)
    cut = {k: (torch.cat([v[:, :t], v[:, t + 1:]], 1) if k in ("x", "dt_raw", "B", "C") else v)
           for k, v in inp.items()}
    yc, fc = run_scan(cut, 64)
    compare(np.delete(y, t, axis=1), yc, TOL_F32, "skip y")
    compare(fs, fc, TOL_F32, "skip final_state")


@pytest.mark.parametrize("path", BF16_PATHS)
def test_memoryless_and_nonfinite_guard(path):
    """Huge |A| and dt >= 0.01: every exponent underflows to 0; output must
    stay finite and equal dt_t (C_t.B_t) x_t + D x_t."""
    cfg = ScanConfig("memless", 1, 600, 4, 64, 128, 1, 256, "bf16", "ones", "normal", seed=8)
    inp = make_scan_inputs(cfg)
    inp["A"][:] = -1.0e5
    y, fs = run_scan(inp, 256, path=path, dt_limit=(0.01, math.inf))
    yr, fr = _oracle(inp, (0.01, math.inf))
    compare(y, yr, TOL_BF16, "memoryless y")
    compare(fs, fr, TOL_BF16, "memoryless final")


@pytest.mark.parametrize("path", BF16_PATHS)
def test_deterministic(path):
    cfg = SCAN_CONFIGS["c1_130m"].with_(seqlen=1024)
    inp = make_scan_inputs(cfg)
    a = run_scan(inp, cfg.chunk_size, path=path)
    b = run_scan(inp, cfg.chunk_size, path=path)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


@pytest.mark.parametrize("path", BF16_PATHS)
def test_groups_replicated_equal(path):
    cfg = ScanConfig("grp", 1, 400, 4, 64, 128, 1, 128, "bf16", "ones", "normal", seed=9)
    inp = make_scan_inputs(cfg)
    y1, f1 = run_scan(inp, 128, path=path)
    rep = dict(inp)
    rep["B"] = inp["B"].repeat_interleave(4, dim=2).contiguous()
    rep["C"] = inp["C"].repeat_interleave(4, dim=2).contiguous()
    y4, f4 = run_scan(rep, 128, path=path)
    compare(y4, y1, 1e-6, "G=H vs G=1 y")
    compare(f4, f1, 1e-6, "G=H vs G=1 final")


def test_positive_A_is_reported():
    cfg = ScanConfig("posA", 1, 64, 2, 16, 16, 1, 16, "f32", "ones", "zero", seed=10)
    inp = make_scan_inputs(cfg)
    inp["A"][1] = 0.5
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    ws = ssd.alloc_workspace(ssd.workspace_size(1, 64, 2, 16, 16, 1, 16, torch.float32), "cuda")
    ssd.chunk_scan_fwd(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"], chunk_size=16,
                       workspace=ws)
    assert ssd.read_device_status(ws) == 7
    inp["A"][1] = -0.5
    d["A"] = inp["A"].cuda()
    ssd.chunk_scan_fwd(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"], chunk_size=16,
                       workspace=ws)
    assert ssd.read_device_status(ws) == 0                 # the status word is cleared per call


def test_empty_sequence_and_batch():
    H, P, N = 4, 64, 128
    init = torch.randn(2, H, N, P, device="cuda")
    x = torch.zeros(2, 0, H, P, device="cuda", dtype=torch.bfloat16)
    B = torch.zeros(2, 0, 1, N, device="cuda", dtype=torch.bfloat16)
    z = torch.zeros(H, device="cuda")
    y, fs = ssd.chunk_scan_fwd(x, torch.zeros(2, 0, H, device="cuda"), z, -torch.ones(H, device="cuda"), B, B.clone(),
                               torch.ones(H, device="cuda"), init_state=init, chunk_size=256)
    torch.cuda.synchronize()
    assert y.shape == (2, 0, H, P) and torch.equal(fs, init)
    x0 = torch.zeros(0, 10, H, P, device="cuda", dtype=torch.bfloat16)
    B0 = torch.zeros(0, 10, 1, N, device="cuda", dtype=torch.bfloat16)
    y0, f0 = ssd.chunk_scan_fwd(x0, torch.zeros(0, 10, H, device="cuda"), z, -torch.ones(H, device="cuda"), B0,
                                B0.clone(), torch.ones(H, device="cuda"), chunk_size=256)
    assert y0.shape == (0, 10, H, P) and f0.shape == (0, H, N, P)


def test_130m_shapes_match_pages():
    """Shapes the nnterp guide prints for mamba2-130m on a 10-token prompt."""
    cfg = ScanConfig("shapes", 1, 10, 24, 64, 128, 1, 256, "bf16", "ones", "zero", seed=12)
    inp = make_scan_inputs(cfg)
    y, fs = run_scan(inp, 256)
    assert y.shape == (1, 10, 24, 64) and fs.shape == (1, 24, 128, 64)
    yr, fr = _oracle(inp)
    compare(y, yr, TOL_BF16, "130m 10-token y")
    compare(fs, fr, TOL_BF16, "130m 10-token final")


@pytest.mark.parametrize("Q", [64, 128, 256])
def test_tensor_path_chunk_sizes(Q):
    """The tensor path over each chunk size it accepts, against the oracle."""
    cfg = ScanConfig("tcq", 2, 3 * 256 + 77, 4, 64, 128, 2, Q, "bf16", "normal", "normal", seed=30 + Q)
    _check(make_scan_inputs(cfg), Q, "tensor", what="tensor Q=%d" % Q)


def test_tensor_path_units():
    """Long sequences split into several units per (batch, head): the state
    passed between units must equal the oracle's."""
    cfg = ScanConfig("units", 1, 8192 + 45, 2, 64, 128, 1, 256, "bf16", "ones", "normal", seed=40)
    _check(make_scan_inputs(cfg), 256, "tensor", what="tensor units")


def test_tensor_path_range_guard():
    """An fp16 operand the tensor path forms out of range is reported, never
    silently wrong.  x itself enters W.X as bf16 (no range limit there); the
    operands formed in fp16 are w.x (for the state) and the carried state.
    x = 1e30 at one token overflows them: the call reports
    SSD_ERR_PRECONDITION.  x = 1e6 at one token is either computed within
    the bar or reported."""
    cfg = ScanConfig("range", 1, 256, 2, 64, 128, 1, 128, "bf16", "ones", "zero", seed=41)
    inp = make_scan_inputs(cfg)
    ws = ssd.alloc_workspace(ssd.workspace_size(1, 256, 2, 64, 128, 1, 128, torch.bfloat16, "tensor"), "cuda")
    for big in (1.0e30, 1.0e6):
        case = dict(inp)
        case["x"] = inp["x"].clone()
        case["x"][0, 10, 0, 3] = big
        d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in case.items()}
        y, fs = ssd.chunk_scan_fwd(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                                   chunk_size=128, path="tensor", workspace=ws)
        st = ssd.read_device_status(ws)
        if big > 1e20:
            assert st == 7
            continue
        assert st in (0, 7)
        if st == 0:
            yr, fr = _oracle(case)
            compare(y.cpu().double().numpy(), yr, TOL_BF16, "x = 1e6 y")
            compare(fs.cpu().double().numpy(), fr, TOL_BF16, "x = 1e6 final_state")


