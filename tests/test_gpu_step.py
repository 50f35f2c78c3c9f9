"""GPU parity of the decode step (through the C ABI) against the fp64 oracle,
and agreement of a loop of steps with the chunked forward (the step-vs-forward
protocol of the state-spaces/mamba issue page: run forward on a sequence,
then the same sequence one step at a time from the same starting state)."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import TOL_BF16, TOL_F32, compare, run_scan
from state_space_sequence_scan_b200 import ssd
from state_space_sequence_scan_b200.inputs import STEP_CONFIGS, ScanConfig, StepConfig, make_scan_inputs, make_step_inputs

pytestmark = pytest.mark.gpu


def _run_steps(inp, T, dt_limit=(0.0, math.inf)):
    d = {k: v.cuda() for k, v in inp.items()}
    state = d["state"].clone()
    ys = []
    for t in range(T):
        # per-token tensors as fresh (16-byte aligned) allocations
        xt, dtt, Bt, Ct = (d[k][t].clone() for k in ("x", "dt_raw", "B", "C"))
        ys.append(ssd.step(xt, dtt, d["dt_bias"], d["A"], Bt, Ct, d["D"], state, dt_limit=dt_limit))
    torch.cuda.synchronize()
    return torch.stack(ys).cpu().double().numpy(), state.cpu().double().numpy()


def _oracle_steps(inp, T, dt_limit=(0.0, math.inf)):
    st = inp["state"].double().numpy().copy()
    ys = [oracle.step(inp["x"][t], inp["dt_raw"][t], inp["dt_bias"], inp["A"], inp["B"][t], inp["C"][t], inp["D"], st,
                      dt_limit=dt_limit) for t in range(T)]
    return np.stack(ys), st


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [(4, 8, 64, 128, 2), (3, 6, 16, 16, 3), (2, 4, 4, 7, 1), (2, 2, 256, 32, 1)])
def test_step_parity_small(shape, dtype):
    b, H, P, N, G = shape
    cfg = StepConfig("s", b, H, P, N, G, 6, dtype, "normal", seed=b * 7 + P)
    inp = make_step_inputs(cfg)
    y, st = _run_steps(inp, 6)
    yr, sr = _oracle_steps(inp, 6)
    tol = TOL_F32
    compare(y, yr, tol, "step y")
    compare(st, sr, tol, "step state")


def test_decode_config_steps():
    """The decode workload (batch 256, 80 heads) for 8 steps on every chain."""
    cfg = STEP_CONFIGS["c4_decode"]
    inp = make_step_inputs(cfg, steps=8)
    y, st = _run_steps(inp, 8)
    yr, sr = _oracle_steps(inp, 8)
    compare(y, yr, TOL_F32, "decode y")
    compare(st, sr, TOL_F32, "decode state")


def test_decode_512_steps_sampled_rows():
    """All 512 steps at full batch on the GPU; the oracle follows 3 batch rows."""
    cfg = STEP_CONFIGS["c4_decode"]
    inp = make_step_inputs(cfg)
    y, st = _run_steps(inp, cfg.steps)
    rows = [0, 131, 255]
    sub = {k: (v[:, rows] if k in ("x", "dt_raw", "B", "C") else (v[rows] if k == "state" else v))
           for k, v in inp.items()}
    yr, sr = _oracle_steps(sub, cfg.steps)
    compare(y[:, rows], yr, TOL_F32, "decode 512 y")
    compare(st[rows], sr, TOL_F32, "decode 512 state")


def test_step_clamp_and_inplace():
    cfg = StepConfig("c", 2, 4, 64, 128, 2, 3, "bf16", "ones", seed=3)
    inp = make_step_inputs(cfg)
    y, st = _run_steps(inp, 3, dt_limit=(0.05, 0.2))
    yr, sr = _oracle_steps(inp, 3, dt_limit=(0.05, 0.2))
    compare(y, yr, TOL_F32, "clamped y")
    compare(st, sr, TOL_F32, "clamped state")


@pytest.mark.parametrize("dtype,tol", [("f32", TOL_F32), ("bf16", TOL_BF16)])
def test_steps_equal_forward(dtype, tol):
    """A loop of ssd_step from init_state equals ssd_chunk_scan_fwd over the
    same tokens, and the state the loop leaves equals final_state."""
    b, L, H, P, N, G = 2, 300, 4, 64, 128, 2
    cfg = ScanConfig("sf", b, L, H, P, N, G, 64, dtype, "normal", "normal", seed=13)
    inp = make_scan_inputs(cfg)
    y_fwd, f_fwd = run_scan(inp, 64)
    d = {k: v.cuda() for k, v in inp.items()}
    state = d["init_state"].clone()
    ys = []
    for t in range(L):
        ys.append(ssd.step(d["x"][:, t].clone(), d["dt_raw"][:, t].clone(), d["dt_bias"], d["A"],
                           d["B"][:, t].clone(), d["C"][:, t].clone(), d["D"], state))
    y_steps = torch.stack(ys, 1).cpu().double().numpy()
    compare(y_steps, y_fwd, tol, "steps vs forward y")
    compare(state.cpu().double().numpy(), f_fwd, tol, "steps vs forward state")


def test_step_deterministic():
    cfg = StepConfig("det", 8, 16, 64, 128, 8, 4, "bf16", "ones", seed=2)
    inp = make_step_inputs(cfg)
    a = _run_steps(inp, 4)
    b = _run_steps(inp, 4)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_step_rejects_misaligned_token_slices():
    """B for step t sliced out of a [T,b,G,N] bf16 buffer with N=7 starts 28t
    bytes in: the call refuses it (16-byte alignment) before any launch."""
    cfg = StepConfig("mis", 2, 4, 4, 7, 1, 2, "bf16", "ones", seed=1)
    d = {k: v.cuda() for k, v in make_step_inputs(cfg).items()}
    with pytest.raises(ssd.SSDError) as ei:
        ssd.step(d["x"][1], d["dt_raw"][1], d["dt_bias"], d["A"], d["B"][1], d["C"][1], d["D"], d["state"])
    assert ei.value.status == 3
