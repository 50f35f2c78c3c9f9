"""Pins of the oracle's steps either side of the scan: the causal depthwise
conv1d with SiLU before it, the gated RMS norm after it (readings in
oracle/ssd_oracle.c).  Each is checked against library routines and
properties the mathematics fixes, never against a retyping of itself."""
import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle


def _silu(u):
    return u * expit(u)


@pytest.mark.parametrize("K", [1, 2, 4])
def test_conv_equals_numpy_convolve(K):
    """Per channel: the causal 'full' convolution's first L values, with the
    kernel reversed (w[c, K-1] multiplies the current token), then SiLU."""
    rng = np.random.default_rng(K)
    b, L, Cd = 2, 13, 6
    x = rng.standard_normal((b, L, Cd)).astype(np.float32)
    w = rng.standard_normal((Cd, K)).astype(np.float32)
    bias = rng.standard_normal(Cd).astype(np.float32)
    got = oracle.conv1d_silu(x, w, bias)
    for bi in range(b):
        for c in range(Cd):
            pre = np.convolve(x[bi, :, c].astype(np.float64), w[c, ::-1].astype(np.float64))[:L] + bias[c]
            assert np.allclose(got[bi, :, c], _silu(pre), rtol=1e-13, atol=1e-13)


def test_conv_impulse_response_and_causality():
    """A unit impulse at t0 on one channel (no bias) reads out the kernel:
    pre-activation w[c, K-1-(t-t0)] for t0 <= t < t0+K, zero elsewhere; and
    nothing before t0 moves."""
    K, L, Cd, t0, c = 4, 12, 3, 5, 1
    w = np.arange(1, Cd * K + 1, dtype=np.float32).reshape(Cd, K) / 10
    x = np.zeros((1, L, Cd), np.float32)
    x[0, t0, c] = 1.0
    out = oracle.conv1d_silu(x, w, np.zeros(Cd, np.float32))
    for t in range(L):
        pre = w[c, K - 1 - (t - t0)] if t0 <= t < t0 + K else 0.0
        assert out[0, t, c] == pytest.approx(float(_silu(np.float64(pre))), abs=1e-14)
    assert np.all(out[0, :, [0, 2]] == 0.0)                # other channels untouched
    x2 = x.copy()
    x2[0, t0:, :] += 3.0
    out2 = oracle.conv1d_silu(x2, w, np.zeros(Cd, np.float32))
    assert np.array_equal(out[0, :t0], out2[0, :t0])


def test_gated_norm_equals_torch_rms_norm():
    rng = np.random.default_rng(3)
    T, D, grp, eps = 7, 12, 4, 1e-5
    y = rng.standard_normal((T, D)).astype(np.float32)
    z = rng.standard_normal((T, D)).astype(np.float32)
    wt = rng.uniform(0.5, 1.5, D).astype(np.float32)
    got = oracle.gated_rmsnorm(y, z, wt, grp, eps)
    v = torch.from_numpy(y).double() * torch.nn.functional.silu(torch.from_numpy(z).double())
    ref = torch.nn.functional.rms_norm(v.view(T, D // grp, grp), (grp,), eps=eps).view(T, D)
    ref = (ref * torch.from_numpy(wt).double()).numpy()
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_gated_norm_invariants():
    """eps = 0, weight 1: every group's output has RMS exactly 1 and is blind
    to a positive scale of y; a zero gate gives zero; groups are independent."""
    rng = np.random.default_rng(4)
    T, D, grp = 5, 16, 8
    y = rng.standard_normal((T, D)).astype(np.float32)
    z = rng.standard_normal((T, D)).astype(np.float32) + 1.0
    one = np.ones(D, np.float32)
    out = oracle.gated_rmsnorm(y, z, one, grp, 0.0)
    rms = np.sqrt((out.reshape(T, D // grp, grp) ** 2).mean(axis=2))
    assert np.allclose(rms, 1.0, rtol=1e-12)
    assert np.allclose(oracle.gated_rmsnorm(4.0 * y, z, one, grp, 0.0), out, rtol=1e-12, atol=1e-12)
    assert np.all(oracle.gated_rmsnorm(y, np.zeros_like(z), one, grp, 1e-5) == 0.0)
    y2 = y.copy()
    y2[:, :grp] *= -7.0
    out2 = oracle.gated_rmsnorm(y2, z, one, grp, 0.0)
    assert np.array_equal(out2[:, grp:], out[:, grp:])
