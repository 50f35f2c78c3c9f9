"""Pins for the fp64 oracle, against facts that do not come from the oracle.

Each test names what fixes the expected value:
  * the quadratic closed form of the scan (the SSD "matrix form": y_t as a
    causal sum over s <= t of (C_t . B_s) exp(sum_{r=s+1..t} dt_r A) dt_s x_s,
    plus the initial state carried by exp(sum_{r<=t} dt_r A), plus D x_t);
  * a two-token example worked out by hand from the per-token recurrence of
    the nnterp guide "Mamba-2" (opening paragraph);
  * the chunked evaluation (intra-chunk quadratic part plus states passed
    between chunks, "Mamba2" knowledge page), which must agree for every chunk
    size, chunk size 1 included (nnterp guide, "The state after every token");
  * the exact skip token dt = 0 (nnterp guide, "betas and decays are one
    argument"), split-and-carry (assigning state_input), decode-step
    continuity (nnterp guide, "The state between steps");
  * limits with textbook answers: no decay (causal linear attention as a
    prefix sum) and an instantly forgetting state (memoryless output);
  * linearity in (x, initial state) and the group-sharing of B and C.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from state_space_sequence_scan_b200.inputs import SCAN_CONFIGS, make_scan_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
INF = float("inf")


def _rand_case(seed, b=2, L=23, H=4, P=5, N=3, G=2, init=True, scale_dt=1.0):
    rng = np.random.default_rng(seed)
    f = lambda *s: rng.standard_normal(s).astype(np.float32)
    case = dict(
        x=f(b, L, H, P), dt_raw=(scale_dt * f(b, L, H)).astype(np.float32),
        dt_bias=(rng.uniform(-3, 0.5, H)).astype(np.float32),
        A=(-rng.uniform(0.2, 3.0, H)).astype(np.float32),
        B=f(b, L, G, N), C=f(b, L, G, N), D=rng.uniform(0.5, 1.5, H).astype(np.float32),
        init_state=(0.3 * f(b, H, N, P)) if init else None)
    return case


def _softplus_py(z):
    z = float(z)
    return max(z, 0.0) + math.log1p(math.exp(-abs(z)))


def _dt(case, lo=0.0, hi=INF):
    z = case["dt_raw"].astype(np.float64) + case["dt_bias"].astype(np.float64)[None, None, :]
    sp = np.vectorize(_softplus_py)(z)
    return np.clip(sp, lo, hi)


def _closed_form(case, lo=0.0, hi=INF):
    """Brute-force quadratic form, explicit loops over (t, s)."""
    x = case["x"].astype(np.float64)
    B = case["B"].astype(np.float64)
    C = case["C"].astype(np.float64)
    A = case["A"].astype(np.float64)
    D = case["D"].astype(np.float64)
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dt = _dt(case, lo, hi)
    H0 = (np.zeros((b, H, N, P)) if case["init_state"] is None
          else case["init_state"].astype(np.float64))
    y = np.zeros((b, L, H, P))
    fs = np.zeros((b, H, N, P))
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            la = dt[bi, :, h] * A[h]                     # log decay per token
            for t in range(L):
                acc = math.exp(la[: t + 1].sum()) * (C[bi, t, g] @ H0[bi, h])
                for s in range(t + 1):
                    decay = math.exp(la[s + 1: t + 1].sum())
                    acc = acc + (C[bi, t, g] @ B[bi, s, g]) * decay * dt[bi, s, h] * x[bi, s, h]
                y[bi, t, h] = acc + D[h] * x[bi, t, h]
            st = math.exp(la.sum()) * H0[bi, h]
            for s in range(L):
                st = st + math.exp(la[s + 1:].sum()) * dt[bi, s, h] * np.outer(B[bi, s, g], x[bi, s, h])
            fs[bi, h] = st
    return y, fs


def _chunked(case, Q, lo=0.0, hi=INF):
    """Chunked SSD in fp64: within-chunk cumsum of the log decay, masked
    decay-weighted C.B^T times x, chunk states B^T.(w x), serial state
    passing between chunks, and C.h + D.x."""
    x = case["x"].astype(np.float64)
    B = case["B"].astype(np.float64)
    C = case["C"].astype(np.float64)
    A = case["A"].astype(np.float64)
    D = case["D"].astype(np.float64)
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dt = _dt(case, lo, hi)
    y = np.zeros((b, L, H, P))
    fs = np.zeros((b, H, N, P))
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            Hs = (np.zeros((N, P)) if case["init_state"] is None
                  else case["init_state"][bi, h].astype(np.float64))
            for c0 in range(0, L, Q):
                sl = slice(c0, min(L, c0 + Q))
                q = sl.stop - sl.start
                cum = np.cumsum(dt[bi, sl, h] * A[h])
                seg = cum[:, None] - cum[None, :]
                mask = np.tril(np.ones((q, q), dtype=bool))
                Lmat = np.where(mask, np.exp(np.where(mask, seg, 0.0)), 0.0)
                Cc, Bc, xc = C[bi, sl, g], B[bi, sl, g], x[bi, sl, h]
                W = (Cc @ Bc.T) * Lmat * dt[bi, sl, h][None, :]
                ydiag = W @ xc
                yoff = np.exp(cum)[:, None] * (Cc @ Hs)
                y[bi, sl, h] = ydiag + yoff + D[h] * xc
                w = np.exp(cum[-1] - cum) * dt[bi, sl, h]
                Hs = math.exp(cum[-1]) * Hs + Bc.T @ (w[:, None] * xc)
            fs[bi, h] = Hs
    return y, fs


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


# --------------------------------------------------------------------------

def test_softplus_matches_textbook():
    for z in (-30.0, -5.0, -1.0, -1e-3, 0.0, 0.7, 3.0, 19.0):
        assert oracle.softplus(z) == pytest.approx(math.log(1.0 + math.exp(z)), rel=1e-14)
    assert oracle.softplus(0.0) == pytest.approx(math.log(2.0), rel=1e-15)
    assert oracle.softplus(60.0) == pytest.approx(60.0, rel=1e-15)
    assert oracle.softplus(-800.0) == 0.0           # underflows to an exact zero


@pytest.mark.parametrize("seed,G,init,limit", [
    (0, 1, False, (0.0, INF)),
    (1, 2, True, (0.0, INF)),
    (2, 4, True, (0.05, 0.6)),                       # clamp active on both ends
    (3, 1, True, (0.0, 0.2)),
])
def test_recurrence_equals_quadratic_closed_form(seed, G, init, limit):
    case = _rand_case(seed, G=G, init=init)
    y, fs = oracle.scan(**case, dt_limit=limit)
    y_ref, fs_ref = _closed_form(case, *limit)
    assert _rel(y, y_ref) < 1e-12
    assert _rel(fs, fs_ref) < 1e-12


def test_two_token_example_by_hand():
    """L=2, one head, P=N=1: every term written out."""
    case = dict(x=np.array([[[[0.5]], [[-1.25]]]], np.float32),
                dt_raw=np.array([[[0.25], [-0.75]]], np.float32),
                dt_bias=np.array([0.125], np.float32), A=np.array([-2.0], np.float32),
                B=np.array([[[[1.5]], [[-0.5]]]], np.float32),
                C=np.array([[[[0.75]], [[2.0]]]], np.float32),
                D=np.array([0.25], np.float32),
                init_state=np.array([[[[0.375]]]], np.float32))
    dt0 = math.log(1 + math.exp(0.25 + 0.125))
    dt1 = math.log(1 + math.exp(-0.75 + 0.125))
    h0 = math.exp(-2.0 * dt0) * 0.375 + dt0 * 1.5 * 0.5
    y0 = 0.75 * h0 + 0.25 * 0.5
    h1 = math.exp(-2.0 * dt1) * h0 + dt1 * (-0.5) * (-1.25)
    y1 = 2.0 * h1 + 0.25 * (-1.25)
    y, fs = oracle.scan(**case)
    assert y[0, 0, 0, 0] == pytest.approx(y0, rel=1e-14)
    assert y[0, 1, 0, 0] == pytest.approx(y1, rel=1e-14)
    assert fs[0, 0, 0, 0] == pytest.approx(h1, rel=1e-14)


@pytest.mark.parametrize("Q", [1, 2, 4, 8, 16, 64])
def test_chunk_size_invariance(Q):
    case = _rand_case(7, b=1, L=64, H=2, P=4, N=3, G=1, init=True)
    y, fs = oracle.scan(**case)
    yc, fsc = _chunked(case, Q)
    assert _rel(yc, y) < 1e-12
    assert _rel(fsc, fs) < 1e-12


def test_chunked_ragged_tail():
    case = _rand_case(8, b=2, L=3 * 8 + 5, H=2, P=3, N=4, G=2, init=False)
    y, fs = oracle.scan(**case)
    yc, fsc = _chunked(case, 8)
    assert _rel(yc, y) < 1e-12 and _rel(fsc, fs) < 1e-12


def test_split_and_carry_equals_whole():
    case = _rand_case(9, L=40, init=True)
    y, fs = oracle.scan(**case)
    T1 = 17
    first = {k: (v[:, :T1] if k in ("x", "dt_raw", "B", "C") else v) for k, v in case.items()}
    y1, h1 = oracle.scan(**first)
    second = {k: (v[:, T1:] if k in ("x", "dt_raw", "B", "C") else v) for k, v in case.items()}
    second["init_state"] = h1.astype(np.float32)
    # the carried state is rounded to fp32 to be fed back: compare to that precision
    y2, h2 = oracle.scan(**second)
    assert _rel(y1, y[:, :T1]) == 0.0
    assert _rel(y2, y[:, T1:]) < 1e-6
    assert _rel(h2, fs) < 1e-6


def test_decode_steps_equal_forward():
    case = _rand_case(10, b=3, L=12, H=4, P=3, N=5, G=2, init=True)
    y, fs = oracle.scan(**case)
    state = case["init_state"].astype(np.float64).copy()
    prev = state.copy()
    for t in range(12):
        yt = oracle.step(case["x"][:, t], case["dt_raw"][:, t], case["dt_bias"], case["A"],
                         case["B"][:, t], case["C"][:, t], case["D"], state)
        assert np.array_equal(yt, y[:, t])              # same loop body, same order
        assert not np.array_equal(state, prev)          # the state moved
        prev = state.copy()
    assert np.array_equal(state, fs)


def test_skip_token_is_exact():
    """dt = 0 at token t: no write and no decay; the state after t equals the
    state after t-1, so dropping the token changes nothing else."""
    case = _rand_case(11, b=1, L=16, init=True)
    t = 6
    case["dt_raw"][:, t, :] = -1.0e4                   # softplus underflows to exactly 0
    y, fs = oracle.scan(**case)
    cut = {k: (np.delete(v, t, axis=1) if k in ("x", "dt_raw", "B", "C") else v)
           for k, v in case.items()}
    y_cut, fs_cut = oracle.scan(**cut)
    assert np.array_equal(fs, fs_cut)
    assert np.array_equal(np.delete(y, t, axis=1), y_cut)
    # the skipped token still reads the state held since token t-1
    before = {k: (v[:, :t] if k in ("x", "dt_raw", "B", "C") else v) for k, v in case.items()}
    _, h_prev = oracle.scan(**before)
    G = case["B"].shape[2]
    for hh in range(case["x"].shape[2]):
        g = hh // (case["x"].shape[2] // G)
        expect = case["C"][0, t, g].astype(np.float64) @ h_prev[0, hh] + \
            float(case["D"][hh]) * case["x"][0, t, hh].astype(np.float64)
        assert np.allclose(y[0, t, hh], expect, rtol=1e-13, atol=1e-13)


def test_no_decay_is_causal_linear_attention():
    """A = 0: y_t = sum_{s<=t} dt_s (C_t . B_s) x_s + D x_t, evaluated as a
    running prefix sum of dt_s B_s x_s^T."""
    case = _rand_case(12, b=1, L=20, H=2, P=3, N=4, G=1, init=False)
    case["A"][:] = 0.0
    y, fs = oracle.scan(**case)
    dt = _dt(case)
    for h in range(2):
        outer = dt[0, :, h, None, None] * np.einsum("tn,tp->tnp", case["B"][0, :, 0].astype(np.float64),
                                                       case["x"][0, :, h].astype(np.float64))
        prefix = np.cumsum(outer, axis=0)
        ref = np.einsum("tn,tnp->tp", case["C"][0, :, 0].astype(np.float64), prefix) \
            + case["D"][h] * case["x"][0, :, h].astype(np.float64)
        assert _rel(y[0, :, h], ref) < 1e-13
        assert _rel(fs[0, h], prefix[-1]) < 1e-13


def test_memoryless_limit():
    """dt*A <= -1000 makes exp() exactly 0: y_t = dt_t (C_t.B_t) x_t + D x_t,
    final state = dt_L B_L x_L^T."""
    case = _rand_case(13, b=2, L=9, H=2, P=3, N=4, G=1, init=True)
    case["A"][:] = -1.0e5
    lim = (0.01, INF)
    y, fs = oracle.scan(**case, dt_limit=lim)
    dt = _dt(case, *lim)
    x64, B64, C64 = (case[k].astype(np.float64) for k in ("x", "B", "C"))
    cb = np.einsum("btn,btn->bt", C64[:, :, 0], B64[:, :, 0])
    ref = dt[..., None] * cb[:, :, None, None] * x64 + case["D"][None, None, :, None] * x64
    assert _rel(y, ref) < 1e-14
    ref_fs = dt[:, -1, :, None, None] * np.einsum("bn,bhp->bhnp", B64[:, -1, 0], x64[:, -1])
    assert _rel(fs, ref_fs) < 1e-14


def test_linear_in_x_and_initial_state():
    c1 = _rand_case(14, init=True)
    c2 = _rand_case(15, init=True)
    for k in ("dt_raw", "dt_bias", "A", "B", "C", "D"):
        c2[k] = c1[k]
    csum = dict(c1)
    csum["x"] = (c1["x"].astype(np.float64) + c2["x"]).astype(np.float32)
    csum["init_state"] = (c1["init_state"].astype(np.float64) + c2["init_state"]).astype(np.float32)
    # fp32 rounding of the sums: compare the oracle on the rounded sums to the
    # sum of the oracle outputs within that rounding
    y1, f1 = oracle.scan(**c1)
    y2, f2 = oracle.scan(**c2)
    ys, fss = oracle.scan(**csum)
    assert _rel(ys, y1 + y2) < 1e-6
    assert _rel(fss, f1 + f2) < 1e-6


def test_groups_share_b_and_c():
    """G=1 with B/C replicated over heads equals G=H; heads h of group g read
    B[:, :, g] with g = h // (H/G)."""
    case = _rand_case(16, H=4, G=1, init=True)
    y1, f1 = oracle.scan(**case)
    rep = dict(case)
    rep["B"] = np.repeat(case["B"], 4, axis=2)
    rep["C"] = np.repeat(case["C"], 4, axis=2)
    y4, f4 = oracle.scan(**rep)
    assert np.array_equal(y1, y4) and np.array_equal(f1, f4)
    # G=2, H=4: zero the second group's B and C -> heads 2,3 see no writes/reads
    c2 = _rand_case(17, H=4, G=2, init=False)
    c2["B"][:, :, 1] = 0.0
    c2["C"][:, :, 1] = 0.0
    y, f = oracle.scan(**c2)
    assert np.array_equal(f[:, 2:], np.zeros_like(f[:, 2:]))
    expect = c2["D"].astype(np.float64)[None, None, 2:, None] * c2["x"][:, :, 2:].astype(np.float64)
    assert np.array_equal(y[:, :, 2:], expect)
    assert np.abs(f[:, :2]).max() > 0


def test_decay_and_write_strength_signs():
    """Printed facts of the nnterp guide for realistic inputs: dt > 0 and the
    log decay A*dt <= 0 (table "The values" and the example's last line)."""
    cfg = SCAN_CONFIGS["c0_tiny_fp32"]
    inp = make_scan_inputs(cfg)
    case = {k: (v.float().numpy() if v is not None else None) for k, v in inp.items()}
    dt = _dt(case)
    assert dt.min() > 0
    assert (dt * case["A"][None, None, :]).max() <= 0


def test_golden_shapes_of_the_130m_layer():
    """Shapes printed by the nnterp guide for mamba2-130m on a 10-token prompt."""
    with open(os.path.join(GOLDEN, "nnterp_mamba2_130m_shapes.json")) as f:
        g = json.load(f)
    b, L = g["batch"], g["seq"]
    H, P, N, G = g["heads"], g["head_dim"], g["state_dim"], g["groups"]
    rng = np.random.default_rng(0)
    case = dict(x=rng.standard_normal((b, L, H, P)).astype(np.float32),
                dt_raw=rng.standard_normal((b, L, H)).astype(np.float32),
                dt_bias=np.zeros(H, np.float32), A=-np.ones(H, np.float32),
                B=rng.standard_normal((b, L, G, N)).astype(np.float32),
                C=rng.standard_normal((b, L, G, N)).astype(np.float32),
                D=np.ones(H, np.float32), init_state=None)
    y, fs = oracle.scan(**case)
    assert list(case["C"].shape) == g["C"] and list(case["B"].shape) == g["B"]
    assert list(case["x"].shape) == g["x"] and list(case["dt_raw"].shape) == g["dt"]
    assert list(y.shape) == g["y"] and list(fs.shape) == g["state"]


def _closed_form_states(case, lo=0.0, hi=INF):
    """Brute force: the state after every token, S_t = exp(sum_{r<=t} la_r) H0
    + sum_{s<=t} exp(sum_{s<r<=t} la_r) dt_s B_s x_s^T, explicit loops."""
    x = case["x"].astype(np.float64)
    B = case["B"].astype(np.float64)
    A = case["A"].astype(np.float64)
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dt = _dt(case, lo, hi)
    H0 = (np.zeros((b, H, N, P)) if case["init_state"] is None
          else case["init_state"].astype(np.float64))
    out = np.zeros((b, L, H, N, P))
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            la = dt[bi, :, h] * A[h]
            for t in range(L):
                st = math.exp(la[: t + 1].sum()) * H0[bi, h]
                for s in range(t + 1):
                    st = st + math.exp(la[s + 1: t + 1].sum()) * dt[bi, s, h] * np.outer(B[bi, s, g], x[bi, s, h])
                out[bi, t, h] = st
    return out


@pytest.mark.parametrize("seed,init", [(40, True), (41, False)])
def test_states_after_every_token_equal_closed_form(seed, init):
    """Chunk size 1: every token is a chunk boundary (nnterp guide, "The
    state after every token"), so states[:, t] is the state after token t."""
    case = _rand_case(seed, b=2, L=9, H=4, P=3, N=2, G=2, init=init)
    y, fs, st = oracle.scan_states(chunk_size=1, **case)
    ref = _closed_form_states(case)
    assert st.shape == ref.shape
    assert _rel(st, ref) < 1e-12
    y0, fs0 = oracle.scan(**case)
    assert np.array_equal(y, y0) and np.array_equal(fs, fs0)


@pytest.mark.parametrize("Q", [2, 3, 5, 23, 64])
def test_chunk_states_are_the_per_token_states_at_boundaries(Q):
    """states[:, c] is the state after token min((c+1) Q, L) - 1, the last one
    is final_state (the guide prints states[:, -1] == final as True)."""
    case = _rand_case(42, b=2, L=23, init=True)
    _, fs, st = oracle.scan_states(chunk_size=Q, **case)
    _, _, per_tok = oracle.scan_states(chunk_size=1, **case)
    L = case["x"].shape[1]
    nc = (L + Q - 1) // Q
    assert st.shape[1] == nc
    for c in range(nc):
        assert np.array_equal(st[:, c], per_tok[:, min((c + 1) * Q, L) - 1])
    assert np.array_equal(st[:, -1], fs)


def test_skip_token_holds_the_state():
    """The guide's check: with betas (dt) of token 3 set to 0, the state after
    token 3 equals the state after token 2 exactly."""
    case = _rand_case(43, b=1, L=10, init=False)
    case["dt_raw"][:, 3, :] = -1.0e4                   # softplus underflows to exactly 0
    _, _, held = oracle.scan_states(chunk_size=1, **case)
    assert np.array_equal(held[:, 3], held[:, 2])
    assert not np.array_equal(held[:, 4], held[:, 3])


def test_golden_states_shape_of_the_130m_layer():
    """Shape of the per-token states the nnterp guide prints for mamba2-130m
    on a 10-token prompt, and its states[:, -1] == final."""
    with open(os.path.join(GOLDEN, "nnterp_mamba2_130m_shapes.json")) as f:
        g = json.load(f)
    b, L = g["batch"], g["seq"]
    H, P, N, G = g["heads"], g["head_dim"], g["state_dim"], g["groups"]
    rng = np.random.default_rng(1)
    case = dict(x=rng.standard_normal((b, L, H, P)).astype(np.float32),
                dt_raw=rng.standard_normal((b, L, H)).astype(np.float32),
                dt_bias=np.zeros(H, np.float32), A=-np.ones(H, np.float32),
                B=rng.standard_normal((b, L, G, N)).astype(np.float32),
                C=rng.standard_normal((b, L, G, N)).astype(np.float32),
                D=np.ones(H, np.float32), init_state=None)
    _, fs, st = oracle.scan_states(chunk_size=1, **case)
    assert list(st.shape) == g["states_per_token"]
    assert np.array_equal(st[:, -1], fs)


def test_bad_shapes_raise():
    case = _rand_case(18)
    bad = dict(case)
    bad["B"] = case["B"][:, :, :1, :2]
    with pytest.raises(ValueError):
        oracle.scan(**bad)
    odd = _rand_case(19, H=3, G=2)
    with pytest.raises(ValueError):
        oracle.scan(**odd)


def _docs(rng, L, min_len=1, max_len=9):
    """Random document lengths covering L (some of length 1)."""
    lens = []
    while sum(lens) < L:
        lens.append(int(rng.integers(min_len, max_len + 1)))
    lens[-1] -= sum(lens) - L
    if lens[-1] == 0:
        lens.pop()
    return lens


@pytest.mark.parametrize("seed", [60, 61])
def test_packed_row_equals_separate_documents(seed):
    """Packing (the "Mamba2" knowledge page: sample packing for Mamba2): a row
    of documents gives, token for token, what each document gives alone from
    a zero state (the first from init_state), and its final state is the last
    document's.  Exactly: the reset writes the same zeros a fresh run starts
    from."""
    rng = np.random.default_rng(seed)
    case = _rand_case(seed, b=2, L=31, H=4, P=3, N=2, G=2, init=True)
    b, L = 2, 31
    seq = np.zeros((b, L), np.int32)
    bounds = []
    for bi in range(b):
        lens = _docs(rng, L)
        pos = 0
        for d, ln in enumerate(lens):
            seq[bi, pos:pos + ln] = 10 * d + bi                # ids need only differ from the neighbour's
            pos += ln
        bounds.append(lens)
    y, fs, st = oracle.scan_varlen(seq_idx=seq, chunk_size=4, **case)
    for bi in range(b):
        pos = 0
        for d, ln in enumerate(bounds[bi]):
            one = {k: (v[bi:bi + 1, pos:pos + ln] if k in ("x", "dt_raw", "B", "C") else v)
                   for k, v in case.items()}
            one["init_state"] = case["init_state"][bi:bi + 1] if d == 0 else None
            yd, fd = oracle.scan(**one)
            assert np.array_equal(y[bi:bi + 1, pos:pos + ln], yd)
            pos += ln
        assert np.array_equal(fs[bi:bi + 1], fd)
    assert np.array_equal(st[:, -1], fs)


def test_one_document_is_the_plain_scan():
    case = _rand_case(62, b=2, L=19, init=True)
    seq = np.full((2, 19), 7, np.int32)
    y, fs, st = oracle.scan_varlen(seq_idx=seq, chunk_size=5, **case)
    y0, fs0, st0 = oracle.scan_states(chunk_size=5, **case)
    assert np.array_equal(y, y0) and np.array_equal(fs, fs0) and np.array_equal(st, st0)
