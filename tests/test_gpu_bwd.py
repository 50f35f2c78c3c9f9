"""GPU parity of the deterministic backward (ssd_chunk_scan_bwd) against the
fp64 oracle's reverse mode of the recurrence (oracle.scan_bwd, pinned by
finite differences in test_oracle_bwd.py).

Bars, per gradient tensor, with bf16 or fp32 inputs alike (both sides read
the same values, bf16 widening to fp32 exactly, and the GPU computes in fp32
throughout):
  * max|gpu - oracle| / RMS(oracle) <= 2e-4 on the small layers (up to about
    1M elements per tensor), <= 1e-3 on the full-size 130m layer;
  * relative L2 error <= 1e-5 for the per-element gradients (x, dt_raw, B, C,
    init_state).  The per-head gradients dA, d(dt_bias), dD are sums over all
    of a head's tokens whose terms cancel: their fp32 error scales with the
    sum of the terms' sizes, not with the result (the chunked form in fp32 on
    the CPU already gives dA a 1.5e-5 relative error on a 200-token, 2-head
    layer whose dA is [-0.45, 0.96]), so they carry the max bar only.
Derived from the arithmetic: the chunked form evaluated in fp32 on the CPU
lands at 1e-6 to 2.3e-5 max/RMS on 300-600-token rows (Q = 64, 256).  The
maximum over a tensor grows with its size: on the full-size layer's dx (12.6M
elements) the GPU reaches 2.7e-4 max/RMS at a relative L2 error of 1.4e-6, so
its max bar is 1e-3 and the L2 bar carries the precision.  Determinism: two
calls give the same bits.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import compare, to_dev
from state_space_sequence_scan_b200 import ssd
from state_space_sequence_scan_b200.inputs import SCAN_CONFIGS, ScanConfig, make_grad_inputs, make_scan_inputs

pytestmark = pytest.mark.gpu

TOL_BWD = 2e-4
TOL_BWD_FULL = 1e-3
TOL_BWD_L2 = 1e-5
KEYS = ("x", "dt_raw", "dt_bias", "A", "B", "C", "D", "init_state")


def run_bwd(inp, grads, Q, dt_limit=(0.0, math.inf), with_dfinal=True):
    d = to_dev(inp)
    dy = grads["dy"].cuda()
    df = grads["dfinal"].cuda() if with_dfinal else None
    b, L, H, P = d["x"].shape
    G, N = d["B"].shape[2], d["B"].shape[3]
    ws = ssd.alloc_workspace(ssd.bwd_workspace_size(b, L, H, P, N, G, Q, d["x"].dtype), "cuda")
    g = ssd.chunk_scan_bwd(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"], dy,
                           dfinal_state=df, init_state=d["init_state"], chunk_size=Q, dt_limit=dt_limit,
                           workspace=ws)
    assert ssd.read_device_status(ws) == 0
    torch.cuda.synchronize()
    return {k: v.cpu().double().numpy() for k, v in g.items()}


def oracle_bwd(inp, grads, dt_limit=(0.0, math.inf), with_dfinal=True):
    return oracle.scan_bwd(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"],
                           grads["dy"], dfinal=grads["dfinal"] if with_dfinal else None,
                           init_state=inp["init_state"], dt_limit=dt_limit)


PER_ELEMENT = ("x", "dt_raw", "B", "C", "init_state")


def check_all(got, ref, what, tol=TOL_BWD):
    for k in KEYS:
        _, l2 = compare(got[k], ref[k], tol, "%s: d%s" % (what, k))
        if k in PER_ELEMENT:
            assert l2 <= TOL_BWD_L2, "%s: d%s: relative L2 %.3e > %.0e" % (what, k, l2, TOL_BWD_L2)


CASES = [
    # b, L, H, P, N, G, Q, dtype, init, dfinal
    (1, 64, 4, 16, 16, 1, 16, "f32", "zero", False),      # the tiny fp32 layer
    (2, 300, 4, 64, 128, 2, 64, "f32", "normal", True),   # ragged last chunk, several pair tiles
    (2, 300, 4, 64, 128, 2, 256, "bf16", "normal", True),
    (1, 200, 2, 32, 64, 2, 100, "f32", "zero", True),     # Q not a multiple of the 64-token tile; G = H
    (2, 130, 3, 8, 8, 3, 7, "f32", "normal", True),       # small Q, many chunks
    (1, 1, 2, 16, 16, 1, 64, "f32", "normal", True),      # one token
    (1, 257, 4, 64, 128, 4, 256, "bf16", "normal", False),  # one token into the second chunk
    (1, 96, 8, 64, 128, 2, 1, "f32", "normal", True),     # Q = 1: a chunk per token
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b%d_L%d_H%d_P%d_N%d_G%d_Q%d_%s_%s_%s" % c)
def test_backward_parity(case):
    b, L, H, P, N, G, Q, dtype, init, with_df = case
    cfg = ScanConfig("bwd", b, L, H, P, N, G, Q, dtype, d_dist="normal", init=init, seed=90 + L)
    inp = make_scan_inputs(cfg)
    grads = make_grad_inputs(cfg)
    got = run_bwd(inp, grads, Q, with_dfinal=with_df)
    ref = oracle_bwd(inp, grads, with_dfinal=with_df)
    check_all(got, ref, str(case))


def test_backward_time_step_limit():
    """Tokens clamped strictly outside [lo, hi] pass no gradient to dt_raw."""
    cfg = ScanConfig("bwd_clamp", 2, 200, 4, 64, 128, 2, 64, "f32", "normal", "normal", seed=95)
    inp = make_scan_inputs(cfg)
    grads = make_grad_inputs(cfg)
    lim = (0.02, 0.05)
    got = run_bwd(inp, grads, 64, dt_limit=lim)
    ref = oracle_bwd(inp, grads, dt_limit=lim)
    check_all(got, ref, "clamped")
    assert np.array_equal(got["dt_raw"] == 0.0, ref["dt_raw"] == 0.0)


def test_backward_is_deterministic():
    cfg = ScanConfig("bwd_det", 2, 1000, 8, 64, 128, 2, 256, "bf16", "normal", "normal", seed=96)
    inp = make_scan_inputs(cfg)
    grads = make_grad_inputs(cfg)
    g1 = run_bwd(inp, grads, 256)
    g2 = run_bwd(inp, grads, 256)
    for k in KEYS:
        assert np.array_equal(g1[k], g2[k]), k


def test_backward_no_tokens():
    """seqlen 0: the seed passes to the initial state unchanged, the per-head sums are 0."""
    cfg = ScanConfig("bwd_empty", 2, 0, 4, 16, 16, 1, 16, "f32", "normal", "normal", seed=97)
    inp = make_scan_inputs(cfg)
    grads = make_grad_inputs(cfg)
    got = run_bwd(inp, grads, 16)
    assert np.array_equal(got["init_state"], grads["dfinal"].double().numpy())
    for k in ("A", "D", "dt_bias"):
        assert np.all(got[k] == 0.0)


def test_backward_130m_layer():
    """The 130m-shaped layer at full size (b 4, L 2048, H 24, bf16), every
    gradient against the oracle."""
    cfg = SCAN_CONFIGS["c1_130m"]
    inp = make_scan_inputs(cfg)
    grads = make_grad_inputs(cfg)
    got = run_bwd(inp, grads, cfg.chunk_size)
    ref = oracle_bwd(inp, grads)
    check_all(got, ref, "c1_130m", tol=TOL_BWD_FULL)


# ---- packed rows (ssd_chunk_scan_bwd_varlen) ---------------------------------

def _packed_ids(b, L, Q, rng, mean_len):
    """Document ids with random lengths down to one token, a start exactly on
    a chunk boundary and on a 64-token pair-tile edge, and a one-token
    document at tokens 5..5."""
    seq = np.zeros((b, L), np.int32)
    for bi in range(b):
        cuts = set(int(c) for c in rng.integers(1, L, size=max(1, L // mean_len)))
        cuts.update({c for c in (Q, 64, 5, 6) if 0 < c < L})
        doc = 0
        for t in range(L):
            if t in cuts:
                doc += 1
            seq[bi, t] = doc
    return seq


def run_bwd_packed(inp, grads, Q, seq):
    d = to_dev(inp)
    b, L, H, P = d["x"].shape
    G, N = d["B"].shape[2], d["B"].shape[3]
    ws = ssd.alloc_workspace(ssd.bwd_workspace_size(b, L, H, P, N, G, Q, d["x"].dtype), "cuda")
    g = ssd.chunk_scan_bwd(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"], grads["dy"].cuda(),
                           dfinal_state=grads["dfinal"].cuda(), init_state=d["init_state"], chunk_size=Q,
                           workspace=ws, seq_idx=torch.from_numpy(seq).cuda())
    assert ssd.read_device_status(ws) == 0
    torch.cuda.synchronize()
    return {k: v.cpu().double().numpy() for k, v in g.items()}


PACKED_CASES = [
    # b, L, H, P, N, G, Q, dtype, mean document length
    (2, 300, 4, 64, 128, 2, 64, "f32", 40),
    (2, 300, 4, 64, 128, 2, 256, "bf16", 70),
    (1, 200, 2, 32, 64, 2, 100, "f32", 25),
    (2, 130, 3, 8, 8, 3, 7, "f32", 9),
    (1, 257, 4, 64, 128, 1, 128, "f32", 3),      # documents of about three tokens
]


@pytest.mark.parametrize("case", PACKED_CASES, ids=lambda c: "b%d_L%d_H%d_P%d_N%d_G%d_Q%d_%s_doc%d" % c)
def test_backward_packed_rows(case):
    """Every gradient of a packed row against the oracle's reverse mode with
    the same document ids (pinned by finite differences of the packed forward
    and by 'a packed row's gradients are its documents' own')."""
    b, L, H, P, N, G, Q, dt, mean_len = case
    cfg = ScanConfig("bwdp", b, L, H, P, N, G, Q, dt, "normal", "normal", seed=sum(case[:7]) % 1009)
    inp = make_scan_inputs(cfg)
    grads = make_grad_inputs(cfg)
    seq = _packed_ids(b, L, Q, np.random.default_rng(L + Q), mean_len)
    got = run_bwd_packed(inp, grads, Q, seq)
    ref = oracle.scan_bwd(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"],
                          grads["dy"], dfinal=grads["dfinal"], init_state=inp["init_state"], seq_idx=seq)
    check_all(got, ref, "packed %s" % (case,))


def test_backward_packed_constant_ids_is_the_plain_backward():
    """One document per row: the packed backward equals the plain one bit for
    bit (every mask passes), and two packed calls give the same bits."""
    cfg = ScanConfig("bwdc", 2, 300, 4, 64, 128, 2, 64, "bf16", "normal", "normal", seed=913)
    inp = make_scan_inputs(cfg)
    grads = make_grad_inputs(cfg)
    seq = np.full((2, 300), 7, np.int32)
    a = run_bwd_packed(inp, grads, 64, seq)
    b_ = run_bwd_packed(inp, grads, 64, seq)
    plain = run_bwd(inp, grads, 64)
    for k in KEYS:
        assert np.array_equal(a[k], plain[k]), "d%s differs from the plain backward" % k
        assert np.array_equal(a[k], b_[k]), "d%s differs between two calls" % k


# ---- the tensor-core pair kernels (path "tensor") ----------------------------
# bf16 inputs, P 64, N 128, chunk sizes that are multiples of 128.  The block
# products run with fp16 operands: dy, the decay-weighted U = (C.B^T) L and
# V = (dy.x^T) L, G_c and H_in are rounded to 11 bits, so every product term
# carries up to 2^-10 relative error.  Derived bar: an output's error is
# about 2^-11 of its own size, and the gradients are heavy-tailed (dx on the
# 130m layer reaches 60x its RMS; an fp64 emulation of the kernels' roundings
# on it gives 1.2e-2 max/RMS on 8 heads), so the largest elements reach
# 2^-11 x 60 = 3e-2 of the RMS: max|gpu - oracle| / RMS <= 5e-2 per gradient,
# and relative L2 <= 2e-3 for the per-element ones (the emulation gives
# 2.2e-4, about 2^-12).
TOL_TC = 5e-2
TOL_TC_L2 = 2e-3

TC_CASES = [
    # b, L, H, G, Q, init, dfinal
    (2, 300, 4, 2, 256, True, True),
    (1, 1, 2, 1, 128, True, True),          # one token
    (2, 2, 2, 2, 256, False, True),         # two tokens
    (1, 128, 2, 1, 128, False, True),
    (1, 129, 2, 2, 128, True, False),
    (2, 640, 3, 3, 256, True, True),
    (1, 1000, 4, 1, 512, True, True),
]


def _tc_case(b, L, H, G, Q, init, seed):
    cfg = ScanConfig("bwdtc", b, L, H, 64, 128, G, Q, "bf16", "normal", "normal" if init else "zero", seed=seed)
    return cfg, make_scan_inputs(cfg), make_grad_inputs(cfg)


def run_bwd_tc(inp, grads, Q, with_dfinal=True, dt_limit=(0.0, math.inf)):
    d = to_dev(inp)
    b, L, H, P = d["x"].shape
    G, N = d["B"].shape[2], d["B"].shape[3]
    ws = ssd.alloc_workspace(ssd.bwd_workspace_size(b, L, H, P, N, G, Q, d["x"].dtype), "cuda")
    g = ssd.chunk_scan_bwd(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"], grads["dy"].cuda(),
                           dfinal_state=grads["dfinal"].cuda() if with_dfinal else None, init_state=d["init_state"],
                           chunk_size=Q, dt_limit=dt_limit, workspace=ws, path="tensor")
    assert ssd.read_device_status(ws) == 0
    torch.cuda.synchronize()
    return {k: v.cpu().double().numpy() for k, v in g.items()}


def check_tc(got, ref, what):
    for k in KEYS:
        if ref[k] is None:
            continue
        rel_max, rel_l2 = compare(got[k], ref[k], TOL_TC, "%s d%s" % (what, k))
        if k in ("x", "dt_raw", "B", "C", "init_state"):
            assert rel_l2 <= TOL_TC_L2, "%s d%s: relative L2 %.3e" % (what, k, rel_l2)


@pytest.mark.parametrize("case", TC_CASES, ids=lambda c: "b%d_L%d_H%d_G%d_Q%d_init%d_df%d" % c)
def test_backward_tensor_path(case):
    b, L, H, G, Q, init, dfin = case
    cfg, inp, grads = _tc_case(b, L, H, G, Q, init, seed=L + 11 * H + G)
    got = run_bwd_tc(inp, grads, Q, with_dfinal=dfin)
    ref = oracle_bwd(inp, grads, with_dfinal=dfin)
    check_tc(got, ref, "tensor %s" % (case,))


def test_backward_tensor_path_clamped_dt():
    cfg, inp, grads = _tc_case(2, 300, 4, 2, 256, True, seed=77)
    lim = (0.002, 0.05)
    got = run_bwd_tc(inp, grads, 256, dt_limit=lim)
    ref = oracle_bwd(inp, grads, dt_limit=lim)
    check_tc(got, ref, "tensor clamped")


def test_backward_tensor_path_130m_layer_and_determinism():
    """The full-size 130m layer on the tensor path against the oracle, and two
    calls give the same bits."""
    cfg = SCAN_CONFIGS["c1_130m"]
    inp = make_scan_inputs(cfg)
    grads = make_grad_inputs(cfg)
    a = run_bwd_tc(inp, grads, cfg.chunk_size)
    b_ = run_bwd_tc(inp, grads, cfg.chunk_size)
    for k in KEYS:
        if a[k] is not None:
            assert np.array_equal(a[k], b_[k]), "d%s differs between two calls" % k
    check_tc(a, oracle_bwd(inp, grads), "tensor c1_130m")


def test_backward_tensor_path_rejects_what_it_does_not_take():
    for dtype, P, Q in (("f32", 64, 256), ("bf16", 32, 256), ("bf16", 64, 64)):
        cfg = ScanConfig("bwdtcx", 1, 200, 2, P, 128, 1, Q, dtype, "normal", "zero", seed=3)
        inp, grads = make_scan_inputs(cfg), make_grad_inputs(cfg)
        with pytest.raises(ssd.SSDError, match="SSD_ERR_UNSUPPORTED"):
            run_bwd_tc(inp, grads, Q)


TC_PACKED_CASES = [
    # b, L, H, G, Q, mean document length
    (2, 300, 4, 2, 256, 40),
    (1, 257, 4, 1, 128, 3),          # documents of about three tokens
    (2, 640, 3, 3, 256, 100),
]


def run_bwd_packed_tc(inp, grads, Q, seq):
    d = to_dev(inp)
    b, L, H, P = d["x"].shape
    G, N = d["B"].shape[2], d["B"].shape[3]
    ws = ssd.alloc_workspace(ssd.bwd_workspace_size(b, L, H, P, N, G, Q, d["x"].dtype), "cuda")
    g = ssd.chunk_scan_bwd(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"], grads["dy"].cuda(),
                           dfinal_state=grads["dfinal"].cuda(), init_state=d["init_state"], chunk_size=Q,
                           workspace=ws, seq_idx=torch.from_numpy(seq).cuda(), path="tensor")
    assert ssd.read_device_status(ws) == 0
    torch.cuda.synchronize()
    return {k: v.cpu().double().numpy() for k, v in g.items()}


@pytest.mark.parametrize("case", TC_PACKED_CASES, ids=lambda c: "b%d_L%d_H%d_G%d_Q%d_doc%d" % c)
def test_backward_tensor_path_packed_rows(case):
    """Packed rows on the tensor path against the oracle's reverse mode with
    the same document ids, at the tensor path's bar."""
    b, L, H, G, Q, mean_len = case
    cfg, inp, grads = _tc_case(b, L, H, G, Q, True, seed=L + Q + mean_len)
    seq = _packed_ids(b, L, Q, np.random.default_rng(L + 3 * Q), mean_len)
    got = run_bwd_packed_tc(inp, grads, Q, seq)
    ref = oracle.scan_bwd(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"],
                          grads["dy"], dfinal=grads["dfinal"], init_state=inp["init_state"], seq_idx=seq)
    check_tc(got, ref, "tensor packed %s" % (case,))


def test_backward_tensor_path_constant_ids_is_unpacked():
    """One document per row: the packed tensor path equals the unpacked one
    bit for bit (every mask passes)."""
    cfg, inp, grads = _tc_case(2, 300, 4, 2, 256, True, seed=915)
    a = run_bwd_packed_tc(inp, grads, 256, np.full((2, 300), 3, np.int32))
    plain = run_bwd_tc(inp, grads, 256)
    for k in KEYS:
        assert np.array_equal(a[k], plain[k]), "d%s differs from the unpacked tensor path" % k
