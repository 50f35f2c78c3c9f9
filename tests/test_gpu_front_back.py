"""GPU parity of the steps either side of the scan (ssd_conv1d_silu_split,
ssd_gated_rmsnorm) against the fp64 oracle, and the three in a row.

Bars: fp32 outputs max|gpu - oracle| / RMS(oracle) <= 1e-5 (one fp32 fma
chain or sum per element); bf16 conv outputs within one bf16 rounding of the
oracle plus 1e-6 absolute per element (the kernel rounds an fp32 value once).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import TOL_BF16, compare
from state_space_sequence_scan_b200 import ssd

pytestmark = pytest.mark.gpu


def _conv_case(b, L, H, P, G, N, K, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    Cd = H * P + 2 * G * N
    xbc = torch.randn(b, L, Cd, generator=g).to(dtype)
    w = (torch.randn(Cd, K, generator=g) / math.sqrt(K)).float()
    bias = (0.1 * torch.randn(Cd, generator=g)).float()
    return xbc, w, bias


def _split(ref, b, L, H, P, G, N):
    HP, GN = H * P, G * N
    return (ref[..., :HP].reshape(b, L, H, P), ref[..., HP:HP + GN].reshape(b, L, G, N),
            ref[..., HP + GN:].reshape(b, L, G, N))


def _check_conv(got, ref, dtype, what):
    got = got.float().cpu().double().numpy()
    if dtype == torch.float32:
        compare(got, ref, 1e-5, what)
    else:
        err = np.abs(got - ref)
        assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 1e-6), "%s: max excess %.3e" % (
            what, float(np.max(err - 2.0 ** -8 * np.abs(ref))))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("K", [1, 2, 3, 4])
def test_conv1d_parity(K, dtype):
    b, L, H, P, G, N = 2, 77, 4, 16, 2, 16               # 77: a ragged last token tile
    xbc, w, bias = _conv_case(b, L, H, P, G, N, K, dtype, seed=K)
    x, B, C = ssd.conv1d_silu_split(xbc.cuda(), w.cuda(), bias.cuda(), H, P, G, N)
    torch.cuda.synchronize()
    ref = oracle.conv1d_silu(xbc.float().numpy(), w.numpy(), bias.numpy())
    for got, r, nm in zip((x, B, C), _split(ref, b, L, H, P, G, N), "xBC"):
        _check_conv(got, r, dtype, "conv K=%d %s" % (K, nm))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_conv1d_silu_over_its_range(dtype):
    """Weights (0, 0, 0, 1) and no bias make every output silu(x) of its own
    input; x spans [-100, 100] (the SiLU's exponential saturates at both
    ends) and tiny magnitudes.  fp32: within 1e-5 relative of the oracle (the
    fast exponential's error grows with |x|: about 6e-6 at |x| = 100), and
    1e-30 absolute where silu itself is below that; bf16: one rounding."""
    H, P, G, N = 2, 64, 1, 64
    Cd = H * P + 2 * G * N
    vals = np.concatenate([np.linspace(-100, 100, 4001), np.geomspace(1e-20, 1, 500), -np.geomspace(1e-20, 1, 500)])
    L = int(math.ceil(vals.size / Cd))
    flat = np.zeros(L * Cd)
    flat[:vals.size] = vals
    xbc = torch.from_numpy(flat.reshape(1, L, Cd)).to(dtype)
    w = torch.zeros(Cd, 4)
    w[:, 3] = 1.0
    bias = torch.zeros(Cd)
    x, B, C = ssd.conv1d_silu_split(xbc.cuda(), w.cuda(), bias.cuda(), H, P, G, N)
    ref = oracle.conv1d_silu(xbc.float().numpy(), w.numpy(), bias.numpy())
    for got, r, nm in zip((x, B, C), _split(ref, 1, L, H, P, G, N), "xBC"):
        g = got.float().cpu().double().numpy()
        if dtype == torch.float32:
            err = np.abs(g - r)
            bad = err > 1e-5 * np.abs(r) + 1e-30
            assert not bad.any(), "silu %s: %d values off, worst input %r (got %r, oracle %r)" % (
                nm, int(bad.sum()), *(float(a[bad][np.argmax((err - 1e-5 * np.abs(r))[bad])])
                                     for a in (_split(xbc.float().numpy(), 1, L, H, P, G, N)["xBC".index(nm)], g, r)))
        else:
            _check_conv(got, r, dtype, "silu range %s" % nm)


# (b, L, H, P, G, N): channel tiles of 128 with the x|B and B|C edges inside
# a tile and a partial last tile (Cd = 152); token tiles of 64 with a ragged
# tail; enough (batch, token tile) rows that each CTA walks its ring of
# stages several times over
TILE_CASES = [(3, 200, 3, 24, 1, 40), (2, 130, 2, 8, 3, 8), (4, 71040, 1, 64, 1, 32),
              (2, 1, 2, 8, 1, 8), (1, 2, 2, 8, 1, 8)]      # one and two tokens: all of the window is halo


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", TILE_CASES, ids=lambda c: "b%d_L%d_H%d_P%d_G%d_N%d" % c)
def test_conv1d_tile_edges(shape, dtype):
    b, L, H, P, G, N = shape
    K = 4
    xbc, w, bias = _conv_case(b, L, H, P, G, N, K, dtype, seed=L + H)
    x, B, C = ssd.conv1d_silu_split(xbc.cuda(), w.cuda(), bias.cuda(), H, P, G, N)
    assert ssd.read_device_status(None) == 0
    ref = oracle.conv1d_silu(xbc.float().numpy(), w.numpy(), bias.numpy())
    for got, r, nm in zip((x, B, C), _split(ref, b, L, H, P, G, N), "xBC"):
        _check_conv(got, r, dtype, "conv %s %s" % (shape, nm))


@pytest.mark.parametrize("zdtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("group", [16, 64, 256, 512, 1536])   # 512, 1536: the single-pass block kernel
def test_gated_rmsnorm_parity(group, zdtype):
    g = torch.Generator().manual_seed(group)
    T, D = 300, 3072                           # a multiple of every group size above
    y = torch.randn(T, D, generator=g)
    z = torch.randn(T, D, generator=g).to(zdtype)
    w = torch.rand(D, generator=g) + 0.5
    out = ssd.gated_rmsnorm(y.cuda(), z.cuda(), w.cuda(), group, 1e-5)
    ref = oracle.gated_rmsnorm(y.numpy(), z.float().numpy(), w.numpy(), group, 1e-5)
    compare(out.cpu().double().numpy(), ref, 1e-5, "gated norm group %d" % group)


def test_conv_scan_norm_in_a_row():
    """conv1d -> scan -> gated norm on the GPU against the oracle's three in
    a row (the oracle's scan fed the GPU conv's bf16 outputs, so the bar is
    the scan's)."""
    b, L, H, P, G, N, K = 2, 300, 4, 64, 2, 128, 4
    xbc, w, bias = _conv_case(b, L, H, P, G, N, K, torch.bfloat16, seed=9)
    gen = torch.Generator().manual_seed(10)
    dt_raw = torch.randn(b, L, H, generator=gen)
    dt_bias = torch.log(torch.expm1(torch.exp(torch.empty(H).uniform_(math.log(1e-3), math.log(0.1), generator=gen))))
    A = -torch.exp(torch.empty(H).uniform_(0.0, math.log(16.0), generator=gen))
    D = torch.ones(H)
    z = torch.randn(b, L, H * P, generator=gen).to(torch.bfloat16)
    wn = torch.rand(H * P, generator=gen) + 0.5
    dev = {k: v.cuda() for k, v in dict(dt_raw=dt_raw, dt_bias=dt_bias, A=A, D=D).items()}
    x, B, C = ssd.conv1d_silu_split(xbc.cuda(), w.cuda(), bias.cuda(), H, P, G, N)
    y, fs = ssd.chunk_scan_fwd(x, dev["dt_raw"], dev["dt_bias"], dev["A"], B, C, dev["D"], chunk_size=256)
    out = ssd.gated_rmsnorm(y.view(b * L, H * P), z.view(b * L, H * P).cuda(), wn.cuda(), P, 1e-5)
    torch.cuda.synchronize()
    yr, fr = oracle.scan(x.float().cpu().numpy(), dt_raw.numpy(), dt_bias.numpy(), A.numpy(), B.float().cpu().numpy(),
                         C.float().cpu().numpy(), D.numpy())
    outr = oracle.gated_rmsnorm(yr.reshape(b * L, H * P).astype(np.float32), z.float().view(b * L, H * P).numpy(),
                                wn.numpy(), P, 1e-5)
    compare(y.cpu().double().numpy(), yr, TOL_BF16, "y")
    compare(out.cpu().double().numpy(), outr, TOL_BF16, "normed y")


def test_full_size_conv_and_norm_of_the_2p7b_layer():
    """The 2.7B-shaped layer's conv (Cd = 80*64 + 2*128) and norm (per head,
    over its y) at full size, against the oracle."""
    b, L, H, P, G, N, K = 8, 4096, 80, 64, 1, 128, 4
    xbc, w, bias = _conv_case(b, L, H, P, G, N, K, torch.bfloat16, seed=11)
    x, B, C = ssd.conv1d_silu_split(xbc.cuda(), w.cuda(), bias.cuda(), H, P, G, N)
    torch.cuda.synchronize()
    ref = oracle.conv1d_silu(xbc.float().numpy(), w.numpy(), bias.numpy())
    for got, r, nm in zip((x, B, C), _split(ref, b, L, H, P, G, N), "xBC"):
        _check_conv(got, r, torch.bfloat16, "2.7B conv %s" % nm)
    g = torch.Generator().manual_seed(12)
    y = torch.randn(b * L, H * P, generator=g)
    z = torch.randn(b * L, H * P, generator=g).to(torch.bfloat16)
    wn = torch.rand(H * P, generator=g) + 0.5
    out = ssd.gated_rmsnorm(y.cuda(), z.cuda(), wn.cuda(), P, 1e-5)
    ref = oracle.gated_rmsnorm(y.numpy(), z.float().numpy(), wn.numpy(), P, 1e-5)
    compare(out.cpu().double().numpy(), ref, 1e-5, "2.7B gated norm")
