"""The conv1d and the scan in the combined arrangement (ssd_conv_scan_fwd)
against the split arrangement (ssd_conv1d_silu_split, then
ssd_chunk_scan_fwd) and against the oracle's conv followed by its scan.

The HF transformers issue "mamba2 mixer different outputs" traces a
difference between the training and inference fast paths to the fused
conv + scan kernel against the two kernels one after the other.  Here both
arrangements evaluate the same conv arithmetic and round each x, B, C value to
bf16 the same way, so they must agree bit for bit; the combined one must also
match the oracle's chain within the bf16 bar.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import TOL_BF16, compare
from state_space_sequence_scan_b200 import ssd
from state_space_sequence_scan_b200.inputs import ScanConfig, make_scan_inputs

pytestmark = pytest.mark.gpu


def _layer(b, L, H, G, seed, init="normal"):
    """Scan inputs of a bf16 layer (P 64, N 128) plus xbc and the conv's
    weights: xbc ~ N(0, 1) in bf16, weights N(0, 1/4), biases N(0, 0.01)."""
    P, N = 64, 128
    cfg = ScanConfig("convscan", b, L, H, P, N, G, 256, "bf16", "normal", init, seed=seed)
    inp = make_scan_inputs(cfg)
    g = torch.Generator().manual_seed(seed + 1)
    Cd = H * P + 2 * G * N
    xbc = torch.randn(b, L, Cd, generator=g).to(torch.bfloat16)
    w = (torch.randn(Cd, 4, generator=g) / 2).float()
    bias = (0.1 * torch.randn(Cd, generator=g)).float()
    return inp, xbc, w, bias


def _both(inp, xbc, w, bias, H, G, Q):
    """(y, final_state) of the split and of the combined arrangement."""
    P, N = 64, 128
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    xd, wd, bd = xbc.cuda(), w.cuda(), bias.cuda()
    x, B, C = ssd.conv1d_silu_split(xd, wd, bd, H, P, G, N)
    ys, fs = ssd.chunk_scan_fwd(x, d["dt_raw"], d["dt_bias"], d["A"], B, C, d["D"], init_state=d["init_state"],
                                chunk_size=Q, path="tensor")
    b, L = xbc.shape[0], xbc.shape[1]
    ws = ssd.alloc_workspace(ssd.workspace_size(b, L, H, P, N, G, Q, torch.bfloat16, "tensor"), "cuda")
    yc, fc = ssd.conv_scan_fwd(xd, wd, bd, d["dt_raw"], d["dt_bias"], d["A"], d["D"], H, P, G, N,
                               init_state=d["init_state"], chunk_size=Q, workspace=ws)
    assert ssd.read_device_status(ws) == 0
    assert ssd.read_device_status(None) == 0
    return ys.cpu().numpy(), fs.cpu().numpy(), yc.cpu().numpy(), fc.cpu().numpy()


# b, L, H, G, Q: ragged last blocks, one block, a token into a second block,
# G = 1, G < H and G = H, and long rows that split into several units (the
# unit-state kernel then convolves too, and each unit's first block takes its
# 3 earlier rows from the unit before)
CASES = [
    (2, 300, 4, 2, 256),
    (1, 1, 2, 1, 128),
    (2, 2, 2, 2, 64),
    (1, 128, 2, 1, 128),
    (1, 129, 2, 2, 64),
    (2, 77, 3, 3, 256),
    (1, 8192, 2, 1, 256),
    (2, 5000, 4, 2, 128),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b%d_L%d_H%d_G%d_Q%d" % c)
def test_combined_equals_split_bit_for_bit(case):
    b, L, H, G, Q = case
    inp, xbc, w, bias = _layer(b, L, H, G, seed=L + 7 * H + G)
    ys, fs, yc, fc = _both(inp, xbc, w, bias, H, G, Q)
    assert np.array_equal(yc, ys), "combined y differs from split: max %.3e" % float(np.max(np.abs(yc - ys)))
    assert np.array_equal(fc, fs), "combined final_state differs from split"


@pytest.mark.parametrize("case", [CASES[0], CASES[6]], ids=lambda c: "b%d_L%d_H%d_G%d_Q%d" % c)
def test_combined_equals_split_without_an_initial_state(case):
    """No initial state (the 130m and 2.7B layers' case): both arrangements
    start every chain from zeros, bit for bit alike."""
    b, L, H, G, Q = case
    inp, xbc, w, bias = _layer(b, L, H, G, seed=L + 5 * H + G, init="zero")
    assert inp["init_state"] is None
    ys, fs, yc, fc = _both(inp, xbc, w, bias, H, G, Q)
    assert np.array_equal(yc, ys), "combined y differs from split: max %.3e" % float(np.max(np.abs(yc - ys)))
    assert np.array_equal(fc, fs), "combined final_state differs from split"


@pytest.mark.parametrize("case", CASES[:4], ids=lambda c: "b%d_L%d_H%d_G%d_Q%d" % c)
def test_combined_against_the_oracle_chain(case):
    """The oracle's conv (fp64, rounded to bf16 as both arrangements store
    x, B, C) followed by its scan."""
    b, L, H, G, Q = case
    P, N = 64, 128
    inp, xbc, w, bias = _layer(b, L, H, G, seed=3 * L + H)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    yc, fc = ssd.conv_scan_fwd(xbc.cuda(), w.cuda(), bias.cuda(), d["dt_raw"], d["dt_bias"], d["A"], d["D"],
                               H, P, G, N, init_state=d["init_state"], chunk_size=Q)
    conv = oracle.conv1d_silu(xbc.float().numpy(), w.numpy(), bias.numpy())
    conv = torch.from_numpy(conv).float().to(torch.bfloat16).float().numpy()
    HP, GN = H * P, G * N
    x = conv[..., :HP].reshape(b, L, H, P)
    B = conv[..., HP:HP + GN].reshape(b, L, G, N)
    C = conv[..., HP + GN:].reshape(b, L, G, N)
    yr, fr = oracle.scan(x, inp["dt_raw"].numpy(), inp["dt_bias"].numpy(), inp["A"].numpy(), B, C,
                         inp["D"].numpy(), init_state=inp["init_state"].numpy())
    compare(yc.cpu().double().numpy(), yr, TOL_BF16, "combined y")
    compare(fc.cpu().double().numpy(), fr, TOL_BF16, "combined final_state")


def test_combined_130m_layer_full_size():
    """The 130m-shaped layer (b 4, L 2048, H 24, G 1) at full size, bit for
    bit against the split arrangement."""
    inp, xbc, w, bias = _layer(4, 2048, 24, 1, seed=130)
    ys, fs, yc, fc = _both(inp, xbc, w, bias, 24, 1, 256)
    assert np.array_equal(yc, ys)
    assert np.array_equal(fc, fs)


def test_combined_rejects_what_it_does_not_take():
    inp, xbc, w, bias = _layer(1, 200, 2, 1, seed=5)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    args = (d["dt_raw"], d["dt_bias"], d["A"], d["D"], 2, 64, 1, 128)
    with pytest.raises(ssd.SSDError, match="SSD_ERR_UNSUPPORTED"):
        ssd.conv_scan_fwd(xbc.cuda(), w[:, :3].contiguous().cuda(), bias.cuda(), *args)   # width 3
    with pytest.raises(ssd.SSDError, match="SSD_ERR_UNSUPPORTED"):
        ssd.conv_scan_fwd(xbc.cuda(), w.cuda(), bias.cuda(), *args, chunk_size=100)       # SIMT-only chunk


def test_combined_long_context_layer_full_size():
    """The long-context layer (b 1, L 65536, H 80, G 8: 11 units of 47 blocks,
    so unit_state convolves too and every unit's first block reads its 3
    earlier rows from the unit before), bit for bit against the split
    arrangement."""
    inp, xbc, w, bias = _layer(1, 65536, 80, 8, seed=65)
    ys, fs, yc, fc = _both(inp, xbc, w, bias, 80, 8, 256)
    assert np.array_equal(yc, ys), "combined y differs from split: max %.3e" % float(np.max(np.abs(yc - ys)))
    assert np.array_equal(fc, fs)
