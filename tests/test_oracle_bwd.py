"""Pins for the backward oracle (oracle.scan_bwd), CPU only.

The gradients are checked against things other than the backward code
itself:
  * directional finite differences of the forward oracle (itself pinned by
    test_oracle.py), with the exact float32 perturbation that reached it;
  * closed forms: dD = sum dy.x; with dy = 0 the seed dfinal reaches the
    initial state and every token through products of decays only;
  * the group sum: G = 1 equals G = H with B, C replicated and the per-head
    gradients of B, C added.
"""
import numpy as np
import pytest

import oracle

NAMES = ["x", "dt_raw", "dt_bias", "A", "B", "C", "D", "init_state"]


def make(b, L, H, P, N, G, seed, A_scale=1.0):
    rng = np.random.default_rng(seed)
    f = np.float32
    inp = {
        "x": rng.standard_normal((b, L, H, P)).astype(f),
        "dt_raw": rng.standard_normal((b, L, H)).astype(f),
        "dt_bias": rng.uniform(-3, 0, H).astype(f),
        "A": (-A_scale * np.exp(rng.uniform(0, np.log(16), H))).astype(f),
        "B": rng.standard_normal((b, L, G, N)).astype(f),
        "C": rng.standard_normal((b, L, G, N)).astype(f),
        "D": rng.normal(1, 0.1, H).astype(f),
        "init_state": rng.normal(0, 0.1, (b, H, N, P)).astype(f),
    }
    dy = rng.standard_normal((b, L, H, P)).astype(f)
    dfinal = rng.standard_normal((b, H, N, P)).astype(f)
    return inp, dy, dfinal


def loss(inp, dy, dfinal, limit):
    y, fs = oracle.scan(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"],
                        init_state=inp["init_state"], dt_limit=limit)
    return float(np.sum(y * dy.astype(np.float64)) + np.sum(fs * dfinal.astype(np.float64)))


def grads(inp, dy, dfinal, limit):
    return oracle.scan_bwd(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"], dy,
                           dfinal=dfinal, init_state=inp["init_state"], dt_limit=limit)


@pytest.mark.parametrize("limit", [(0.0, float("inf")), (0.02, 0.3)])
@pytest.mark.parametrize("name", NAMES)
def test_directional_finite_difference(name, limit):
    # 70 tokens: the oracle's recompute checkpoints (64 tokens) are crossed
    inp, dy, dfinal = make(2, 70, 4, 3, 5, 2, seed=11)
    g = grads(inp, dy, dfinal, limit)
    rng = np.random.default_rng(100 + NAMES.index(name))
    v = rng.standard_normal(inp[name].shape)
    # x, B, C, D and init_state enter linearly (no truncation error); dt and A
    # through exponentials, where the step sets the third-order term
    eps = 1e-3 if name in ("x", "B", "C", "D", "init_state") else 1e-4
    base = inp[name].astype(np.float64)
    plus, minus = dict(inp), dict(inp)
    plus[name] = (base + eps * v).astype(np.float32)
    minus[name] = (base - eps * v).astype(np.float32)
    # the perturbation that really reached the float32 inputs
    delta = plus[name].astype(np.float64) - minus[name].astype(np.float64)
    fd = loss(plus, dy, dfinal, limit) - loss(minus, dy, dfinal, limit)
    pred = float(np.sum(g[name] * delta))
    assert abs(fd - pred) <= 1e-6 * max(abs(pred), 1e-3 * float(np.sum(np.abs(g[name] * delta)))), (fd, pred)


def test_clamped_tokens_pass_no_gradient_to_dt_raw():
    inp, dy, dfinal = make(1, 30, 2, 3, 4, 1, seed=12)
    lo, hi = 0.05, 0.2
    g = grads(inp, dy, dfinal, (lo, hi))
    z = inp["dt_raw"].astype(np.float64) + inp["dt_bias"].astype(np.float64)
    sp = np.logaddexp(0.0, z)
    out = (sp < lo) | (sp > hi)
    assert out.any() and (~out).any()
    assert np.all(g["dt_raw"][out] == 0.0)
    assert np.all(g["dt_raw"][~out] != 0.0)


def test_dD_is_the_sum_of_dy_x():
    inp, dy, dfinal = make(2, 40, 3, 4, 5, 3, seed=13)
    g = grads(inp, dy, dfinal, (0.0, float("inf")))
    ref = np.einsum("blhp,blhp->h", dy.astype(np.float64), inp["x"].astype(np.float64))
    np.testing.assert_allclose(g["D"], ref, rtol=1e-12, atol=1e-12)


def test_final_state_seed_reaches_back_through_the_decays():
    """dy = 0: the loss is <dfinal, S_L> with S_L = (prod a) S_0 +
    sum_t dt_t (prod_{r>t} a_r) B_t x_t^T, so dinit = (prod a) dfinal,
    dx_t = dt_t (prod_{r>t} a_r) dfinal^T B_t, dB_t = the same with x_t, dC = 0."""
    b, L, H, P, N, G = 2, 9, 2, 3, 4, 2
    inp, _, dfinal = make(b, L, H, P, N, G, seed=14)
    dy = np.zeros((b, L, H, P), np.float32)
    g = grads(inp, dy, dfinal, (0.0, float("inf")))
    z = inp["dt_raw"].astype(np.float64) + inp["dt_bias"].astype(np.float64)
    dt = np.logaddexp(0.0, z)
    a = np.exp(dt * inp["A"].astype(np.float64))             # [b, L, H]
    after = np.ones_like(a)                                  # prod_{r>t} a_r
    for t in range(L - 2, -1, -1):
        after[:, t] = after[:, t + 1] * a[:, t + 1]
    df = dfinal.astype(np.float64)
    np.testing.assert_allclose(g["init_state"], np.prod(a, axis=1)[:, :, None, None] * df, rtol=1e-12, atol=1e-14)
    Bh = np.repeat(inp["B"].astype(np.float64), H // G, axis=2)   # [b, L, H, N]
    xh = inp["x"].astype(np.float64)
    dx = (dt * after)[..., None] * np.einsum("bhnp,blhn->blhp", df, Bh)
    np.testing.assert_allclose(g["x"], dx, rtol=1e-11, atol=1e-14)
    dBh = (dt * after)[..., None] * np.einsum("bhnp,blhp->blhn", df, xh)
    np.testing.assert_allclose(g["B"], dBh.reshape(b, L, G, H // G, N).sum(3), rtol=1e-11, atol=1e-14)
    assert np.all(g["C"] == 0.0)


def test_group_gradients_are_sums_over_the_heads_of_the_group():
    b, L, H, P, N = 1, 20, 4, 3, 5
    inp, dy, dfinal = make(b, L, H, P, N, 1, seed=15)
    g1 = grads(inp, dy, dfinal, (0.0, float("inf")))
    rep = dict(inp)
    rep["B"] = np.repeat(inp["B"], H, axis=2)
    rep["C"] = np.repeat(inp["C"], H, axis=2)
    gh = grads(rep, dy, dfinal, (0.0, float("inf")))
    np.testing.assert_allclose(g1["B"][:, :, 0], gh["B"].sum(axis=2), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(g1["C"][:, :, 0], gh["C"].sum(axis=2), rtol=1e-12, atol=1e-13)
    for k in ("x", "dt_raw", "A", "dt_bias", "D", "init_state"):
        np.testing.assert_allclose(g1[k], gh[k], rtol=1e-12, atol=1e-13)


def test_a_planted_sign_error_is_caught():
    """The finite-difference pin sees a flipped term: negate the A-direction
    gradient's decay part and the check fails."""
    inp, dy, dfinal = make(1, 20, 2, 3, 4, 1, seed=16)
    g = grads(inp, dy, dfinal, (0.0, float("inf")))
    v = np.ones(2)
    eps = 1e-3
    plus, minus = dict(inp), dict(inp)
    plus["A"] = (inp["A"] + eps * v).astype(np.float32)
    minus["A"] = (inp["A"] - eps * v).astype(np.float32)
    delta = plus["A"].astype(np.float64) - minus["A"].astype(np.float64)
    fd = loss(plus, dy, dfinal, (0.0, float("inf"))) - loss(minus, dy, dfinal, (0.0, float("inf")))
    assert abs(fd - float(np.sum(g["A"] * delta))) <= 1e-6 * abs(fd)
    assert abs(fd - float(np.sum(-g["A"] * delta))) > 1e-2 * abs(fd)


def test_split_and_carry_backward():
    """Backward over [T1, L) from dfinal gives the gradient of the state at T1;
    used as the seed of the backward over [0, T1) (which starts from
    init_state), the pieces equal the whole-sequence gradients (per-head sums
    added over the two segments)."""
    b, L, H, P, N, G, T1 = 2, 50, 4, 3, 5, 2, 23
    inp, dy, dfinal = make(b, L, H, P, N, G, seed=17)
    lim = (0.0, float("inf"))
    whole = grads(inp, dy, dfinal, lim)
    # the state at T1 from the forward oracle over the first segment
    first = {k: (v[:, :T1] if k in ("x", "dt_raw", "B", "C") else v) for k, v in inp.items()}
    _, s1 = oracle.scan(first["x"], first["dt_raw"], first["dt_bias"], first["A"], first["B"], first["C"],
                        first["D"], init_state=inp["init_state"], dt_limit=lim)
    second = {k: (v[:, T1:] if k in ("x", "dt_raw", "B", "C") else v) for k, v in inp.items()}
    second["init_state"] = s1.astype(np.float32)
    g2 = grads(second, dy[:, T1:], dfinal, lim)
    # the carried state is float32-rounded for the second segment: compare the
    # first segment with its own seed, exactly as the chain rule composes
    g1 = grads(first, dy[:, :T1], g2["init_state"].astype(np.float32), lim)
    np.testing.assert_allclose(np.concatenate([g1["x"], g2["x"]], axis=1), whole["x"], rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(np.concatenate([g1["B"], g2["B"]], axis=1), whole["B"], rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(np.concatenate([g1["C"], g2["C"]], axis=1), whole["C"], rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(np.concatenate([g1["dt_raw"], g2["dt_raw"]], axis=1), whole["dt_raw"], rtol=1e-5,
                               atol=1e-6)
    for k in ("A", "D", "dt_bias"):
        np.testing.assert_allclose(g1[k] + g2[k], whole[k], rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(g1["init_state"], whole["init_state"], rtol=1e-5, atol=1e-6)


def test_gradients_are_linear_in_the_seeds():
    inp, dy1, df1 = make(1, 30, 2, 3, 4, 1, seed=18)
    _, dy2, df2 = make(1, 30, 2, 3, 4, 1, seed=19)
    lim = (0.0, float("inf"))
    # seeds on a 1/64 grid: 0.5 a + 2 b is then exact in float32
    dy1, dy2, df1, df2 = (np.round(v * 64) / 64 for v in (dy1, dy2, df1, df2))
    dy1, dy2, df1, df2 = (v.astype(np.float32) for v in (dy1, dy2, df1, df2))
    g1 = grads(inp, dy1, df1, lim)
    g2 = grads(inp, dy2, df2, lim)
    dy12, df12 = 0.5 * dy1 + 2.0 * dy2, 0.5 * df1 + 2.0 * df2
    assert np.array_equal(dy12.astype(np.float64), 0.5 * dy1.astype(np.float64) + 2.0 * dy2.astype(np.float64))
    g12 = grads(inp, dy12, df12, lim)
    for k in NAMES:
        np.testing.assert_allclose(g12[k], 0.5 * g1[k] + 2.0 * g2[k], rtol=1e-11, atol=1e-12)


# ---- packed rows: seq_idx document ids, the state zeroed at every start

def packed_ids(b, L, seed):
    rng = np.random.default_rng(seed)
    ids = np.zeros((b, L), np.int32)
    for bi in range(b):
        cuts = np.sort(rng.choice(np.arange(1, L), size=4, replace=False))
        cuts[1] = cuts[0] + 1                 # a one-token document
        ids[bi] = np.searchsorted(cuts, np.arange(L), side="right")
    return ids


def loss_varlen(inp, dy, dfinal, ids):
    y, fs, _ = oracle.scan_varlen(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"],
                                  ids, init_state=inp["init_state"])
    return float(np.sum(y * dy.astype(np.float64)) + np.sum(fs * dfinal.astype(np.float64)))


def grads_varlen(inp, dy, dfinal, ids):
    return oracle.scan_bwd(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"], dy,
                           dfinal=dfinal, init_state=inp["init_state"], seq_idx=ids)


@pytest.mark.parametrize("name", NAMES)
def test_packed_directional_finite_difference(name):
    inp, dy, dfinal = make(2, 60, 4, 3, 5, 2, seed=41)
    ids = packed_ids(2, 60, seed=42)
    g = grads_varlen(inp, dy, dfinal, ids)
    v = np.random.default_rng(300 + NAMES.index(name)).standard_normal(inp[name].shape)
    eps = 1e-3 if name in ("x", "B", "C", "D", "init_state") else 1e-4
    base = inp[name].astype(np.float64)
    plus, minus = dict(inp), dict(inp)
    plus[name] = (base + eps * v).astype(np.float32)
    minus[name] = (base - eps * v).astype(np.float32)
    delta = plus[name].astype(np.float64) - minus[name].astype(np.float64)
    fd = loss_varlen(plus, dy, dfinal, ids) - loss_varlen(minus, dy, dfinal, ids)
    pred = float(np.sum(g[name] * delta))
    assert abs(fd - pred) <= 1e-6 * max(abs(pred), 1e-3 * float(np.sum(np.abs(g[name] * delta)))), (fd, pred)


def separate_documents(inp, dy, dfinal, ids):
    """The packed row's gradients assembled from each document's own
    backward: the first document starts from init_state, the others from
    zeros; only the last one's final state is the row's (dfinal seeds it)."""
    b, L, H, P = inp["x"].shape
    out = {"x": np.zeros((b, L, H, P)), "dt_raw": np.zeros((b, L, H)), "B": np.zeros(inp["B"].shape),
           "C": np.zeros(inp["C"].shape), "A": np.zeros(H), "dt_bias": np.zeros(H), "D": np.zeros(H),
           "init_state": np.zeros(inp["init_state"].shape)}
    for bi in range(b):
        starts = [0] + [t for t in range(1, L) if ids[bi, t] != ids[bi, t - 1]] + [L]
        for k in range(len(starts) - 1):
            t0, t1 = starts[k], starts[k + 1]
            doc = {n: (inp[n][bi:bi + 1, t0:t1] if n in ("x", "dt_raw", "B", "C") else inp[n])
                   for n in ("x", "dt_raw", "B", "C", "dt_bias", "A", "D")}
            s0 = inp["init_state"][bi:bi + 1] if k == 0 else None
            seed = dfinal[bi:bi + 1] if t1 == L else np.zeros_like(dfinal[bi:bi + 1])
            g = oracle.scan_bwd(doc["x"], doc["dt_raw"], doc["dt_bias"], doc["A"], doc["B"], doc["C"], doc["D"],
                                dy[bi:bi + 1, t0:t1], dfinal=seed, init_state=s0)
            for n in ("x", "dt_raw", "B", "C"):
                out[n][bi, t0:t1] = g[n][0]
            for n in ("A", "dt_bias", "D"):
                out[n] += g[n]
            if k == 0:
                out["init_state"][bi] = g["init_state"][0]
    return out


def test_packed_row_gradients_are_its_documents_gradients():
    inp, dy, dfinal = make(2, 60, 4, 3, 5, 2, seed=43)
    ids = packed_ids(2, 60, seed=44)
    g = grads_varlen(inp, dy, dfinal, ids)
    ref = separate_documents(inp, dy, dfinal, ids)
    for n in NAMES:
        np.testing.assert_allclose(g[n], ref[n], rtol=1e-12, atol=1e-13, err_msg=n)


def test_one_document_is_the_plain_backward():
    inp, dy, dfinal = make(1, 40, 2, 3, 4, 1, seed=45)
    g = grads_varlen(inp, dy, dfinal, np.full((1, 40), 7, np.int32))
    ref = grads(inp, dy, dfinal, (0.0, float("inf")))
    for n in NAMES:
        assert np.array_equal(g[n], ref[n]), n
