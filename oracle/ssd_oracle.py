"""Python face of the fp64 CPU oracle (``ssd_oracle.c``).

TEST INFRASTRUCTURE ONLY.  The test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may call this module; the CUDA path never
does, and this module imports nothing from the CUDA package.

Parity: pinned by tests/test_oracle.py against the quadratic closed form of
the scan, a hand-computed two-token example, and the invariants the nnterp
"Mamba-2" guide states (exact skip token, chunk-boundary continuity, decode
continuity) -- see the C file's header for the recurrence itself.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB_NAME = "libssd_oracle.so"
_lib = None


def oracle_library_path() -> str:
    return os.path.join(_HERE, _LIB_NAME)


def build_oracle(force: bool = False) -> str:
    """Compile ssd_oracle.c with gcc into oracle/libssd_oracle.so."""
    out = oracle_library_path()
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(_SRC):
        return out
    tmp = out + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-std=c99", "-D_POSIX_C_SOURCE=200809L",
           "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm", "-lpthread"]
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_oracle())
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        i64 = ctypes.c_int64
        lib.ssd_oracle_scan.restype = ctypes.c_int
        lib.ssd_oracle_scan.argtypes = [f32p] * 8 + [f64p, f64p] + [i64] * 6 + [
            ctypes.c_double, ctypes.c_double, ctypes.c_int]
        lib.ssd_oracle_scan_states.restype = ctypes.c_int
        lib.ssd_oracle_scan_states.argtypes = [f32p] * 8 + [f64p, f64p, f64p] + [i64] * 7 + [
            ctypes.c_double, ctypes.c_double, ctypes.c_int]
        i32p = ctypes.POINTER(ctypes.c_int32)
        lib.ssd_oracle_scan_varlen.restype = ctypes.c_int
        lib.ssd_oracle_scan_varlen.argtypes = [f32p] * 8 + [i32p, f64p, f64p, f64p] + [i64] * 7 + [
            ctypes.c_double, ctypes.c_double, ctypes.c_int]
        lib.ssd_oracle_conv1d_silu.restype = ctypes.c_int
        lib.ssd_oracle_conv1d_silu.argtypes = [f32p] * 3 + [f64p] + [i64] * 4
        lib.ssd_oracle_gated_rmsnorm.restype = ctypes.c_int
        lib.ssd_oracle_gated_rmsnorm.argtypes = [f32p] * 3 + [f64p] + [i64] * 3 + [ctypes.c_double]
        lib.ssd_oracle_step.restype = ctypes.c_int
        lib.ssd_oracle_step.argtypes = [f32p] * 7 + [f64p, f64p] + [i64] * 5 + [
            ctypes.c_double, ctypes.c_double, ctypes.c_int]
        lib.ssd_oracle_scan_bwd.restype = ctypes.c_int
        lib.ssd_oracle_scan_bwd.argtypes = [f32p] * 10 + [f64p] * 8 + [i64] * 6 + [
            ctypes.c_double, ctypes.c_double, ctypes.c_int]
        lib.ssd_oracle_scan_bwd_varlen.restype = ctypes.c_int
        lib.ssd_oracle_scan_bwd_varlen.argtypes = [f32p] * 8 + [i32p] + [f32p] * 2 + [f64p] * 8 + [i64] * 6 + [
            ctypes.c_double, ctypes.c_double, ctypes.c_int]
        lib.ssd_oracle_softplus.restype = ctypes.c_double
        lib.ssd_oracle_softplus.argtypes = [ctypes.c_double]
        _lib = lib
    return _lib


def _f32(a) -> np.ndarray:
    """Exact float32 copy of an input (torch tensors of bf16/f32, numpy)."""
    if hasattr(a, "detach"):  # torch tensor: widen bf16 exactly, move to host
        a = a.detach().to("cpu").float().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _p32(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def _p64(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def softplus(z: float) -> float:
    """The oracle's softplus, log(1 + e^z), evaluated in double."""
    return float(_load().ssd_oracle_softplus(float(z)))


def scan(x, dt_raw, dt_bias, A, B, C, D, init_state=None,
         dt_limit: Tuple[float, float] = (0.0, float("inf")),
         nthreads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """Sequential fp64 recurrence over a whole sequence.

    x [b,L,H,P], dt_raw [b,L,H], dt_bias/A/D [H], B/C [b,L,G,N],
    init_state [b,H,N,P] or None (zeros).  Returns (y [b,L,H,P] float64,
    final_state [b,H,N,P] float64).
    """
    x, dt_raw, dt_bias, A, B, C, D = (_f32(v) for v in (x, dt_raw, dt_bias, A, B, C, D))
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    if dt_raw.shape != (b, L, H) or B.shape != (b, L, G, N) or C.shape != B.shape:
        raise ValueError("oracle.scan: inconsistent shapes")
    if dt_bias.shape != (H,) or A.shape != (H,) or D.shape != (H,) or H % G:
        raise ValueError("oracle.scan: bad per-head parameter shapes or H % G != 0")
    s0 = None
    if init_state is not None:
        s0 = _f32(init_state)
        if s0.shape != (b, H, N, P):
            raise ValueError("oracle.scan: init_state must be [b,H,N,P]")
    y = np.empty((b, L, H, P), dtype=np.float64)
    fs = np.empty((b, H, N, P), dtype=np.float64)
    rc = _load().ssd_oracle_scan(
        _p32(x), _p32(dt_raw), _p32(dt_bias), _p32(A), _p32(B), _p32(C), _p32(D),
        _p32(s0) if s0 is not None else ctypes.POINTER(ctypes.c_float)(),
        _p64(y), _p64(fs), b, L, H, P, N, G,
        float(dt_limit[0]), float(dt_limit[1]), int(nthreads))
    if rc != 0:
        raise RuntimeError("ssd_oracle_scan failed with code %d" % rc)
    return y, fs


def scan_states(x, dt_raw, dt_bias, A, B, C, D, chunk_size: int, init_state=None,
                dt_limit: Tuple[float, float] = (0.0, float("inf")),
                nthreads: int = 0) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """As scan(), also returning the chunk-boundary states (nnterp guide
    "Mamba-2", "The state after every token"): states [b, ceil(L/Q), H, N, P]
    float64, states[:, c] the state after token min((c+1) Q, L) - 1, so
    states[:, -1] is final_state and Q = 1 gives the state after every token.
    """
    x, dt_raw, dt_bias, A, B, C, D = (_f32(v) for v in (x, dt_raw, dt_bias, A, B, C, D))
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    Q = int(chunk_size)
    if Q < 1:
        raise ValueError("oracle.scan_states: chunk_size must be >= 1")
    if dt_raw.shape != (b, L, H) or B.shape != (b, L, G, N) or C.shape != B.shape:
        raise ValueError("oracle.scan_states: inconsistent shapes")
    if dt_bias.shape != (H,) or A.shape != (H,) or D.shape != (H,) or H % G:
        raise ValueError("oracle.scan_states: bad per-head parameter shapes or H % G != 0")
    s0 = None
    if init_state is not None:
        s0 = _f32(init_state)
        if s0.shape != (b, H, N, P):
            raise ValueError("oracle.scan_states: init_state must be [b,H,N,P]")
    nc = (L + Q - 1) // Q
    y = np.empty((b, L, H, P), dtype=np.float64)
    fs = np.empty((b, H, N, P), dtype=np.float64)
    states = np.empty((b, nc, H, N, P), dtype=np.float64)
    rc = _load().ssd_oracle_scan_states(
        _p32(x), _p32(dt_raw), _p32(dt_bias), _p32(A), _p32(B), _p32(C), _p32(D),
        _p32(s0) if s0 is not None else ctypes.POINTER(ctypes.c_float)(),
        _p64(y), _p64(fs), _p64(states), b, L, H, P, N, G, Q,
        float(dt_limit[0]), float(dt_limit[1]), int(nthreads))
    if rc != 0:
        raise RuntimeError("ssd_oracle_scan_states failed with code %d" % rc)
    return y, fs, states


def scan_varlen(x, dt_raw, dt_bias, A, B, C, D, seq_idx, chunk_size: int = 1, init_state=None,
                dt_limit: Tuple[float, float] = (0.0, float("inf")),
                nthreads: int = 0) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Packed rows: seq_idx [b, L] int32 document ids; the state is zeroed
    before the first token of every document but a row's first (which starts
    from init_state).  Returns (y, final_state, chunk states) as scan_states."""
    x, dt_raw, dt_bias, A, B, C, D = (_f32(v) for v in (x, dt_raw, dt_bias, A, B, C, D))
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    Q = int(chunk_size)
    si = np.ascontiguousarray(np.asarray(seq_idx, dtype=np.int32))
    if si.shape != (b, L):
        raise ValueError("oracle.scan_varlen: seq_idx must be [b, L]")
    if Q < 1 or dt_raw.shape != (b, L, H) or B.shape != (b, L, G, N) or C.shape != B.shape:
        raise ValueError("oracle.scan_varlen: inconsistent shapes")
    s0 = None
    if init_state is not None:
        s0 = _f32(init_state)
    nc = (L + Q - 1) // Q
    y = np.empty((b, L, H, P), dtype=np.float64)
    fs = np.empty((b, H, N, P), dtype=np.float64)
    states = np.empty((b, nc, H, N, P), dtype=np.float64)
    rc = _load().ssd_oracle_scan_varlen(
        _p32(x), _p32(dt_raw), _p32(dt_bias), _p32(A), _p32(B), _p32(C), _p32(D),
        _p32(s0) if s0 is not None else ctypes.POINTER(ctypes.c_float)(),
        si.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
        _p64(y), _p64(fs), _p64(states), b, L, H, P, N, G, Q,
        float(dt_limit[0]), float(dt_limit[1]), int(nthreads))
    if rc != 0:
        raise RuntimeError("ssd_oracle_scan_varlen failed with code %d" % rc)
    return y, fs, states


def scan_bwd(x, dt_raw, dt_bias, A, B, C, D, dy, dfinal=None, init_state=None,
             dt_limit: Tuple[float, float] = (0.0, float("inf")), nthreads: int = 0, seq_idx=None) -> dict:
    """Gradients of <dy, y> + <dfinal, final_state> for scan(), or for
    scan_varlen() when seq_idx [b, L] is given (reverse mode of the
    recurrence; see ssd_oracle.c).  dy [b,L,H,P], dfinal [b,H,N,P] or
    None (zeros).  Returns float64 arrays keyed by input: x, dt_raw [b,L,H],
    dt_bias, A, D [H], B, C [b,L,G,N] (the heads of each group summed),
    init_state [b,H,N,P] (always, also when init_state is None)."""
    x, dt_raw, dt_bias, A, B, C, D, dy = (_f32(v) for v in (x, dt_raw, dt_bias, A, B, C, D, dy))
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    if dt_raw.shape != (b, L, H) or B.shape != (b, L, G, N) or C.shape != B.shape or dy.shape != x.shape:
        raise ValueError("oracle.scan_bwd: inconsistent shapes")
    if dt_bias.shape != (H,) or A.shape != (H,) or D.shape != (H,) or H % G:
        raise ValueError("oracle.scan_bwd: bad per-head parameter shapes or H % G != 0")
    null = ctypes.POINTER(ctypes.c_float)()
    s0 = _f32(init_state) if init_state is not None else None
    df = _f32(dfinal) if dfinal is not None else None
    for nm, v in (("init_state", s0), ("dfinal", df)):
        if v is not None and v.shape != (b, H, N, P):
            raise ValueError("oracle.scan_bwd: %s must be [b,H,N,P]" % nm)
    out = {
        "x": np.zeros((b, L, H, P)), "dt_raw": np.zeros((b, L, H)),
        "B_h": np.zeros((b, L, H, N)), "C_h": np.zeros((b, L, H, N)),
        "A_h": np.zeros((b, H)), "dt_bias_h": np.zeros((b, H)), "D_h": np.zeros((b, H)),
        "init_state": np.zeros((b, H, N, P)),
    }
    si = None
    if seq_idx is not None:
        si = np.ascontiguousarray(np.asarray(seq_idx, dtype=np.int32))
        if si.shape != (b, L):
            raise ValueError("oracle.scan_bwd: seq_idx must be [b, L]")
    rc = _load().ssd_oracle_scan_bwd_varlen(
        _p32(x), _p32(dt_raw), _p32(dt_bias), _p32(A), _p32(B), _p32(C), _p32(D),
        _p32(s0) if s0 is not None else null,
        si.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)) if si is not None else ctypes.POINTER(ctypes.c_int32)(),
        _p32(dy), _p32(df) if df is not None else null,
        _p64(out["x"]), _p64(out["dt_raw"]), _p64(out["B_h"]), _p64(out["C_h"]), _p64(out["A_h"]),
        _p64(out["dt_bias_h"]), _p64(out["D_h"]), _p64(out["init_state"]), b, L, H, P, N, G,
        float(dt_limit[0]), float(dt_limit[1]), int(nthreads))
    if rc != 0:
        raise RuntimeError("ssd_oracle_scan_bwd failed with code %d" % rc)
    hpg = H // G
    return {
        "x": out["x"], "dt_raw": out["dt_raw"],
        "B": out["B_h"].reshape(b, L, G, hpg, N).sum(axis=3),
        "C": out["C_h"].reshape(b, L, G, hpg, N).sum(axis=3),
        "A": out["A_h"].sum(axis=0), "dt_bias": out["dt_bias_h"].sum(axis=0), "D": out["D_h"].sum(axis=0),
        "init_state": out["init_state"],
    }


def conv1d_silu(xbc, weight, bias) -> np.ndarray:
    """Causal depthwise conv of width K over channels, plus bias, then SiLU,
    from zeros (the conv before the scan, read as in ssd_oracle.c).
    xbc [b, L, Cd], weight [Cd, K], bias [Cd] -> [b, L, Cd] float64."""
    xbc, weight, bias = _f32(xbc), _f32(weight), _f32(bias)
    b, L, Cd = xbc.shape
    if weight.ndim != 2 or weight.shape[0] != Cd or bias.shape != (Cd,):
        raise ValueError("oracle.conv1d_silu: weight must be [Cd, K] and bias [Cd]")
    out = np.empty((b, L, Cd), dtype=np.float64)
    rc = _load().ssd_oracle_conv1d_silu(_p32(xbc), _p32(weight), _p32(bias), _p64(out), b, L, Cd,
                                        weight.shape[1])
    if rc != 0:
        raise RuntimeError("ssd_oracle_conv1d_silu failed with code %d" % rc)
    return out


def gated_rmsnorm(y, z, weight, group: int, eps: float) -> np.ndarray:
    """v = y * silu(z); out = v / sqrt(mean over each group of `group`
    channels of v^2 + eps) * weight.  y, z [..., D], weight [D]."""
    y, z, weight = _f32(y), _f32(z), _f32(weight)
    D = y.shape[-1]
    if z.shape != y.shape or weight.shape != (D,):
        raise ValueError("oracle.gated_rmsnorm: z must match y and weight be [D]")
    T = y.size // D
    out = np.empty(y.shape, dtype=np.float64)
    rc = _load().ssd_oracle_gated_rmsnorm(_p32(y), _p32(z), _p32(weight), _p64(out), T, D, int(group), float(eps))
    if rc != 0:
        raise RuntimeError("ssd_oracle_gated_rmsnorm failed with code %d" % rc)
    return out


def step(x, dt_raw, dt_bias, A, B, C, D, state: np.ndarray,
         dt_limit: Tuple[float, float] = (0.0, float("inf")),
         nthreads: int = 0) -> np.ndarray:
    """One decode token.  ``state`` [b,H,N,P] float64 is updated in place;
    returns y [b,H,P] float64.  x [b,H,P], dt_raw [b,H], B/C [b,G,N]."""
    x, dt_raw, dt_bias, A, B, C, D = (_f32(v) for v in (x, dt_raw, dt_bias, A, B, C, D))
    b, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    if not (isinstance(state, np.ndarray) and state.dtype == np.float64
            and state.flags.c_contiguous and state.shape == (b, H, N, P)):
        raise ValueError("oracle.step: state must be a contiguous float64 [b,H,N,P] array")
    if dt_raw.shape != (b, H) or B.shape != (b, G, N) or C.shape != B.shape or H % G:
        raise ValueError("oracle.step: inconsistent shapes")
    y = np.empty((b, H, P), dtype=np.float64)
    rc = _load().ssd_oracle_step(
        _p32(x), _p32(dt_raw), _p32(dt_bias), _p32(A), _p32(B), _p32(C), _p32(D),
        _p64(state), _p64(y), b, H, P, N, G,
        float(dt_limit[0]), float(dt_limit[1]), int(nthreads))
    if rc != 0:
        raise RuntimeError("ssd_oracle_step failed with code %d" % rc)
    return y


def max_err_over_rms(got, ref) -> Tuple[float, float]:
    """(max |got - ref| / RMS(ref), relative L2 error), both in float64."""
    g = np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    if r.size == 0:
        return 0.0, 0.0
    rms = float(np.sqrt(np.mean(r * r)))
    err = np.abs(g - r)
    denom = rms if rms > 0 else 1.0
    l2 = float(np.linalg.norm((g - r).ravel()) / max(np.linalg.norm(r.ravel()), 1e-300))
    return float(err.max()) / denom, l2
