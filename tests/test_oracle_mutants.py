"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a private copy of the oracle's C source (a
dropped term, a wrong sign or index, swapped operands), compiles it on the
CPU, and checks that the closed-form pin rejects it.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

from test_oracle import _closed_form, _rand_case, _rel

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "ssd_oracle.c")

MUTANTS = {
    "drop_D_skip": ("yr[p] = yacc[p] + Dh * (double)xr[p];", "yr[p] = yacc[p];"),
    "decay_sign": ("const double a = exp(dt * A);", "const double a = exp(-dt * A);"),
    "no_dt_on_write": ("const double w = dt * (double)Br[n];\n            double *Sn",
                       "const double w = (double)Br[n];\n            double *Sn"),
    "group_index": ("const int64_t g = h / (H / G);", "const int64_t g = h % G;"),
    "B_C_swapped": ("const float *Br = J->B + ((bi * L + t) * G + g) * N;\n        const float *Cr = J->C",
                    "const float *Br = J->C + ((bi * L + t) * G + g) * N;\n        const float *Cr = J->B"),
    "no_bias": ("const double z = (double)J->dt_raw[(bi * L + t) * H + h] + bias;",
                "const double z = (double)J->dt_raw[(bi * L + t) * H + h];"),
    "decay_on_new_write": ("Sn[p] = a * Sn[p] + w * (double)xr[p];", "Sn[p] = a * (Sn[p] + w * (double)xr[p]);"),
    "state_transposed_read": ("const double *Sn = S + n * P;\n            for (p = 0; p < P; ++p) yacc[p] += c * Sn[p];",
                              "for (p = 0; p < P; ++p) yacc[p] += c * S[(p % N) * P + (n % P)];"),
    "no_init_state": ("for (n = 0; n < N * P; ++n) S[n] = (double)s0[n];",
                      "for (n = 0; n < N * P; ++n) S[n] = 0.0 * s0[n];"),
}


def _build(tmp_path, name, old, new):
    src = open(SRC).read()
    assert old in src, name
    src = src.replace(old, new)
    c = tmp_path / (name + ".c")
    c.write_text(src)
    so = tmp_path / (name + ".so")
    subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-std=c99", "-D_POSIX_C_SOURCE=200809L",
                           "-o", str(so), str(c), "-lm", "-lpthread"])
    return str(so)


def _scan_with(lib_path, case):
    lib = ctypes.CDLL(lib_path)
    f32p = ctypes.POINTER(ctypes.c_float)
    f64p = ctypes.POINTER(ctypes.c_double)
    lib.ssd_oracle_scan.restype = ctypes.c_int
    lib.ssd_oracle_scan.argtypes = [f32p] * 8 + [f64p, f64p] + [ctypes.c_int64] * 6 + [
        ctypes.c_double, ctypes.c_double, ctypes.c_int]
    arr = {k: (np.ascontiguousarray(v, np.float32) if v is not None else None) for k, v in case.items()}
    b, L, H, P = arr["x"].shape
    G, N = arr["B"].shape[2:]
    y = np.empty((b, L, H, P))
    fs = np.empty((b, H, N, P))
    p = lambda a: a.ctypes.data_as(f32p)
    rc = lib.ssd_oracle_scan(p(arr["x"]), p(arr["dt_raw"]), p(arr["dt_bias"]), p(arr["A"]), p(arr["B"]),
                             p(arr["C"]), p(arr["D"]),
                             p(arr["init_state"]) if arr["init_state"] is not None else f32p(),
                             y.ctypes.data_as(f64p), fs.ctypes.data_as(f64p), b, L, H, P, N, G,
                             0.0, float("inf"), 1)
    assert rc == 0
    return y, fs


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_planted_mistake(tmp_path, name):
    old, new = MUTANTS[name]
    so = _build(tmp_path, name, old, new)
    case = _rand_case(21, b=1, L=9, H=4, P=3, N=5, G=2, init=True)
    y, fs = _scan_with(so, case)
    y_ref, fs_ref = _closed_form(case)
    assert max(_rel(y, y_ref), _rel(fs, fs_ref)) > 1e-6, "planted mistake went unnoticed"


def test_unmutated_copy_passes(tmp_path):
    so = _build(tmp_path, "clean", "/* S <- a S + dt B x^T */", "/* S <- a S + dt B x^T */")
    case = _rand_case(21, b=1, L=9, H=4, P=3, N=5, G=2, init=True)
    y, fs = _scan_with(so, case)
    y_ref, fs_ref = _closed_form(case)
    assert max(_rel(y, y_ref), _rel(fs, fs_ref)) < 1e-12


# ---- the backward oracle: each planted mistake must fail the finite-difference pin
BWD_MUTANTS = {
    "bwd_drop_D": ("dxr[p] = dtt * acc + Dh * (double)dyr[p];", "dxr[p] = dtt * acc;"),
    "bwd_no_decay_carry": ("Gm[i] = start ? 0.0 : Gm[i] * at;", "Gm[i] = start ? 0.0 : Gm[i] * 1.0;"),
    "bwd_dA_no_dt": ("dA += dtt * at * gs;", "dA += at * gs;"),
    "bwd_ddt_no_A": ("dz = (bgx + A * at * gs)", "dz = (bgx + at * gs)"),
    "bwd_dC_previous_state": ("acc += Scur[n * P + p] * (double)dyr[p];", "acc += Sprev[n * P + p] * (double)dyr[p];"),
    "bwd_sigmoid_sign": ("? sigmoid_exact(z) : 0.0);", "? sigmoid_exact(-z) : 0.0);"),
    "bwd_dB_no_dt": ("dBr[n] = dtt * acc;", "dBr[n] = acc;"),
    "bwd_seed_ignored": ("for (i = 0; i < NP; ++i) Gm[i] = (double)J->dfinal[(bi * H + h) * NP + i];",
                         "for (i = 0; i < NP; ++i) Gm[i] = 0.0 * J->dfinal[(bi * H + h) * NP + i];"),
}


def _bwd_with(lib_path, inp, dy, dfinal):
    lib = ctypes.CDLL(lib_path)
    f32p = ctypes.POINTER(ctypes.c_float)
    f64p = ctypes.POINTER(ctypes.c_double)
    lib.ssd_oracle_scan_bwd.restype = ctypes.c_int
    lib.ssd_oracle_scan_bwd.argtypes = [f32p] * 10 + [f64p] * 8 + [ctypes.c_int64] * 6 + [
        ctypes.c_double, ctypes.c_double, ctypes.c_int]
    b, L, H, P = inp["x"].shape
    G, N = inp["B"].shape[2:]
    o = {"x": np.zeros((b, L, H, P)), "dt_raw": np.zeros((b, L, H)), "B_h": np.zeros((b, L, H, N)),
         "C_h": np.zeros((b, L, H, N)), "A_h": np.zeros((b, H)), "dt_bias_h": np.zeros((b, H)),
         "D_h": np.zeros((b, H)), "init_state": np.zeros((b, H, N, P))}
    p32 = lambda a: np.ascontiguousarray(a, np.float32).ctypes.data_as(f32p)
    keep = [np.ascontiguousarray(inp[k], np.float32) for k in ("x", "dt_raw", "dt_bias", "A", "B", "C", "D",
                                                              "init_state")]
    keep += [np.ascontiguousarray(dy, np.float32), np.ascontiguousarray(dfinal, np.float32)]
    rc = lib.ssd_oracle_scan_bwd(*[a.ctypes.data_as(f32p) for a in keep],
                                 *[o[k].ctypes.data_as(f64p) for k in ("x", "dt_raw", "B_h", "C_h", "A_h",
                                                                       "dt_bias_h", "D_h", "init_state")],
                                 b, L, H, P, N, G, 0.0, float("inf"), 1)
    assert rc == 0
    hpg = H // G
    return {"x": o["x"], "dt_raw": o["dt_raw"], "B": o["B_h"].reshape(b, L, G, hpg, N).sum(3),
            "C": o["C_h"].reshape(b, L, G, hpg, N).sum(3), "A": o["A_h"].sum(0), "dt_bias": o["dt_bias_h"].sum(0),
            "D": o["D_h"].sum(0), "init_state": o["init_state"]}


def _fd_misses(g, inp, dy, dfinal):
    """Names whose directional finite difference (of the pinned forward
    oracle) disagrees with g."""
    from test_oracle_bwd import NAMES, loss
    bad = []
    lim = (0.0, float("inf"))
    for name in NAMES:
        v = np.random.default_rng(200 + NAMES.index(name)).standard_normal(inp[name].shape)
        eps = 1e-3 if name in ("x", "B", "C", "D", "init_state") else 1e-4
        base = inp[name].astype(np.float64)
        plus, minus = dict(inp), dict(inp)
        plus[name] = (base + eps * v).astype(np.float32)
        minus[name] = (base - eps * v).astype(np.float32)
        delta = plus[name].astype(np.float64) - minus[name].astype(np.float64)
        fd = loss(plus, dy, dfinal, lim) - loss(minus, dy, dfinal, lim)
        pred = float(np.sum(g[name] * delta))
        if abs(fd - pred) > 1e-6 * max(abs(pred), 1e-3 * float(np.sum(np.abs(g[name] * delta)))):
            bad.append(name)
    return bad


@pytest.mark.parametrize("name", sorted(BWD_MUTANTS))
def test_backward_pin_rejects_planted_mistake(tmp_path, name):
    from test_oracle_bwd import make
    old, new = BWD_MUTANTS[name]
    so = _build(tmp_path, name, old, new)
    inp, dy, dfinal = make(1, 70, 4, 3, 5, 2, seed=31)
    assert _fd_misses(_bwd_with(so, inp, dy, dfinal), inp, dy, dfinal), "planted mistake went unnoticed"


def test_backward_unmutated_copy_passes(tmp_path):
    from test_oracle_bwd import make
    so = _build(tmp_path, "bwd_clean", "#define kSeg 64", "#define kSeg 64")
    inp, dy, dfinal = make(1, 70, 4, 3, 5, 2, seed=31)
    assert _fd_misses(_bwd_with(so, inp, dy, dfinal), inp, dy, dfinal) == []


PACKED_BWD_MUTANTS = {
    "bwd_gradient_crosses_start": ("Gm[i] = start ? 0.0 : Gm[i] * at;", "Gm[i] = Gm[i] * at;"),
    "bwd_decay_term_at_start": ("            if (!start)\n                for (i = 0; i < NP; ++i) gs",
                                "            if (1)\n                for (i = 0; i < NP; ++i) gs"),
}


@pytest.mark.parametrize("name", sorted(PACKED_BWD_MUTANTS))
def test_packed_backward_pin_rejects_planted_mistake(tmp_path, name, monkeypatch):
    """The separate-documents pin sees a backward that lets a gradient or a
    decay term cross a document start."""
    import oracle
    from oracle import ssd_oracle
    from test_oracle_bwd import make, packed_ids, separate_documents
    old, new = PACKED_BWD_MUTANTS[name]
    so = _build(tmp_path, name, old, new)
    inp, dy, dfinal = make(2, 60, 4, 3, 5, 2, seed=43)
    ids = packed_ids(2, 60, seed=44)
    ref = separate_documents(inp, dy, dfinal, ids)       # the clean oracle's per-document runs
    monkeypatch.setattr(ssd_oracle, "_lib", None)
    monkeypatch.setattr(ssd_oracle, "build_oracle", lambda force=False: so)
    g = oracle.scan_bwd(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"], dy,
                        dfinal=dfinal, init_state=inp["init_state"], seq_idx=ids)
    monkeypatch.setattr(ssd_oracle, "_lib", None)
    worst = max(float(np.max(np.abs(g[n] - ref[n])) / (np.sqrt(np.mean(ref[n] ** 2)) + 1e-300)) for n in ref)
    assert worst > 1e-6, "planted mistake went unnoticed"
