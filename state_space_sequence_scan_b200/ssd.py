"""Python binding of libssd.so (argument marshalling only).

Every step of the scan and of the decode update runs in the CUDA library; this
module checks tensor shapes/dtypes/devices, allocates outputs and workspace
through PyTorch (device memory is the only thing PyTorch provides here), and
passes raw pointers plus the current CUDA stream across the C ABI declared in
include/ssd.h.  There is no CPU fallback: without the built library, or
without a CUDA device, every compute call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libssd.so")

SSD_OK = 0
STATUS_NAMES = {
    0: "SSD_OK", 1: "SSD_ERR_INVALID_ARG", 2: "SSD_ERR_UNSUPPORTED", 3: "SSD_ERR_ALIGNMENT",
    4: "SSD_ERR_WORKSPACE", 5: "SSD_ERR_CUDA", 6: "SSD_ERR_DEVICE_TIMEOUT", 7: "SSD_ERR_PRECONDITION",
}
DTYPES = {torch.float32: 0, torch.bfloat16: 1}
PATHS = {"auto": 0, "simt": 1, "tensor": 2}

EXPORTED = ("ssd_chunk_scan_workspace_size", "ssd_chunk_scan_fwd", "ssd_chunk_scan_fwd_states", "ssd_step",
            "ssd_read_device_status", "ssd_status_string", "ssd_last_cuda_error", "ssd_version",
            "ssd_trace_enable", "ssd_trace_read", "ssd_trace_kernel_name", "ssd_trace_kernel_count",
            "ssd_conv1d_silu_split", "ssd_gated_rmsnorm", "ssd_chunk_scan_fwd_varlen",
            "ssd_chunk_scan_bwd_workspace_size", "ssd_chunk_scan_bwd", "ssd_chunk_scan_bwd_varlen",
            "ssd_set_test_fault", "ssd_conv_scan_fwd")

_lib = None


class SSDError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str = ""):
        self.status = status
        name = STATUS_NAMES.get(status, str(status))
        super().__init__("%s failed: %s%s" % (fn, name, (" (" + detail + ")") if detail else ""))


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libssd.so and declares the C signatures.  Raises if it is missing:
    there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError("libssd.so is not built (%s); run python -m state_space_sequence_scan_b200.build"
                           % path)
    lib = ctypes.CDLL(path)
    vp, i64, f32, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int, ctypes.c_size_t
    lib.ssd_chunk_scan_workspace_size.restype = i32
    lib.ssd_chunk_scan_workspace_size.argtypes = [i64] * 7 + [i32, i32, ctypes.POINTER(sz)]
    lib.ssd_chunk_scan_fwd.restype = i32
    lib.ssd_chunk_scan_fwd.argtypes = [vp] * 10 + [i64] * 7 + [f32, f32, i32, i32, vp, sz, vp]
    lib.ssd_chunk_scan_fwd_varlen.restype = i32
    lib.ssd_chunk_scan_fwd_varlen.argtypes = [vp] * 12 + [i64] * 7 + [f32, f32, i32, i32, vp, sz, vp]
    lib.ssd_chunk_scan_fwd_states.restype = i32
    lib.ssd_chunk_scan_fwd_states.argtypes = [vp] * 11 + [i64] * 7 + [f32, f32, i32, i32, vp, sz, vp]
    lib.ssd_chunk_scan_bwd_workspace_size.restype = i32
    lib.ssd_chunk_scan_bwd_workspace_size.argtypes = [i64] * 7 + [i32, ctypes.POINTER(sz)]
    lib.ssd_chunk_scan_bwd.restype = i32
    lib.ssd_chunk_scan_bwd.argtypes = [vp] * 18 + [i64] * 7 + [f32, f32, i32, vp, sz, vp]
    lib.ssd_chunk_scan_bwd_varlen.restype = i32
    lib.ssd_chunk_scan_bwd_varlen.argtypes = [vp] * 19 + [i64] * 7 + [f32, f32, i32, i32, vp, sz, vp]
    lib.ssd_step.restype = i32
    lib.ssd_step.argtypes = [vp] * 9 + [i64] * 5 + [f32, f32, i32, vp]
    lib.ssd_read_device_status.restype = i32
    lib.ssd_read_device_status.argtypes = [vp, vp]
    lib.ssd_status_string.restype = ctypes.c_char_p
    lib.ssd_status_string.argtypes = [i32]
    lib.ssd_last_cuda_error.restype = i32
    lib.ssd_last_cuda_error.argtypes = []
    lib.ssd_version.restype = i32
    lib.ssd_version.argtypes = []
    lib.ssd_trace_enable.restype = i32
    lib.ssd_trace_enable.argtypes = [i32]
    lib.ssd_trace_read.restype = i32
    lib.ssd_trace_read.argtypes = [i32, ctypes.POINTER(i32), ctypes.POINTER(ctypes.c_double)]
    lib.ssd_trace_kernel_name.restype = ctypes.c_char_p
    lib.ssd_trace_kernel_name.argtypes = [i32]
    lib.ssd_trace_kernel_count.restype = i32
    lib.ssd_trace_kernel_count.argtypes = []
    lib.ssd_set_test_fault.restype = i32
    lib.ssd_set_test_fault.argtypes = [i32]
    lib.ssd_conv1d_silu_split.restype = i32
    lib.ssd_conv1d_silu_split.argtypes = [vp] * 6 + [i64] * 7 + [i32, vp]
    lib.ssd_gated_rmsnorm.restype = i32
    lib.ssd_gated_rmsnorm.argtypes = [vp] * 4 + [i64] * 3 + [f32, i32, vp]
    lib.ssd_conv_scan_fwd.restype = i32
    lib.ssd_conv_scan_fwd.argtypes = [vp] * 3 + [i64] + [vp] * 7 + [i64] * 7 + [f32, f32, i32, vp, sz, vp]
    _lib = lib
    return lib


def set_test_fault(kind: int) -> None:
    """TEST ONLY (ssd_set_test_fault): kind 1 makes the tensor-path scan's
    waits run out (the first C and B tiles are never requested) so the device-side
    timeout path runs; kind 0 restores normal operation."""
    _check("ssd_set_test_fault", load_library().ssd_set_test_fault(int(kind)))


def _check(fn: str, st: int):
    if st != SSD_OK:
        detail = ""
        if st == 5:
            detail = "cudaError %d" % load_library().ssd_last_cuda_error()
        raise SSDError(fn, st, detail)


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(dev: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _need_cuda(name: str, t: torch.Tensor, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))


def workspace_size(batch: int, seqlen: int, nheads: int, head_dim: int, state_dim: int, ngroups: int,
                   chunk_size: int, dtype: torch.dtype = torch.bfloat16, path: str = "auto") -> int:
    lib = load_library()
    out = ctypes.c_size_t(0)
    _check("ssd_chunk_scan_workspace_size", lib.ssd_chunk_scan_workspace_size(
        batch, seqlen, nheads, head_dim, state_dim, ngroups, chunk_size, DTYPES[dtype], PATHS[path],
        ctypes.byref(out)))
    return int(out.value)


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    """Workspace as a uint8 CUDA tensor (PyTorch allocations are 256-byte aligned)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def chunk_scan_fwd(x: torch.Tensor, dt_raw: torch.Tensor, dt_bias: torch.Tensor, A: torch.Tensor,
                   B: torch.Tensor, C: torch.Tensor, D: torch.Tensor,
                   init_state: Optional[torch.Tensor] = None, chunk_size: int = 256,
                   dt_limit: Tuple[float, float] = (0.0, math.inf), path: str = "auto",
                   workspace: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                   final_state: Optional[torch.Tensor] = None,
                   want_final_state: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunked forward scan.  Shapes as in include/ssd.h:
    x [b,L,H,P], dt_raw [b,L,H] f32, dt_bias/A/D [H] f32, B/C [b,L,G,N] (same
    dtype as x, f32 or bf16), init_state [b,H,N,P] f32 or None.
    Returns (y [b,L,H,P] f32, final_state [b,H,N,P] f32 or None)."""
    lib = load_library()
    if x.dim() != 4 or B.dim() != 4:
        raise ValueError("x must be [b,L,H,P] and B, C [b,L,G,N]")
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dev = x.device
    _need_cuda("x", x)
    if x.dtype not in DTYPES:
        raise ValueError("x/B/C must be float32 or bfloat16")
    _need_cuda("B", B, x.dtype, (b, L, G, N))
    _need_cuda("C", C, x.dtype, (b, L, G, N))
    _need_cuda("dt_raw", dt_raw, torch.float32, (b, L, H))
    for nm, t in (("dt_bias", dt_bias), ("A", A), ("D", D)):
        _need_cuda(nm, t, torch.float32, (H,))
    if init_state is not None:
        _need_cuda("init_state", init_state, torch.float32, (b, H, N, P))
    if y is None:
        y = torch.empty((b, L, H, P), dtype=torch.float32, device=dev)
    else:
        _need_cuda("y", y, torch.float32, (b, L, H, P))
    if want_final_state and final_state is None:
        final_state = torch.empty((b, H, N, P), dtype=torch.float32, device=dev)
    elif final_state is not None:
        _need_cuda("final_state", final_state, torch.float32, (b, H, N, P))
    need = workspace_size(b, L, H, P, N, G, chunk_size, x.dtype, path)
    if workspace is None:
        workspace = alloc_workspace(need, dev)
    st = lib.ssd_chunk_scan_fwd(
        _ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(init_state),
        _ptr(y), _ptr(final_state), b, L, H, P, N, G, int(chunk_size),
        float(dt_limit[0]), float(dt_limit[1]), DTYPES[x.dtype], PATHS[path],
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(dev))
    _check("ssd_chunk_scan_fwd", st)
    return y, final_state


def chunk_scan_fwd_states(x: torch.Tensor, dt_raw: torch.Tensor, dt_bias: torch.Tensor, A: torch.Tensor,
                          B: torch.Tensor, C: torch.Tensor, D: torch.Tensor,
                          init_state: Optional[torch.Tensor] = None, chunk_size: int = 256,
                          dt_limit: Tuple[float, float] = (0.0, math.inf), path: str = "auto",
                          workspace: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                          final_state: Optional[torch.Tensor] = None,
                          chunk_states: Optional[torch.Tensor] = None
                          ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """chunk_scan_fwd that also returns the chunk-boundary states
    [b, ceil(L/chunk_size), H, N, P] f32 (ssd_chunk_scan_fwd_states): chunk c
    holds the state after token min((c+1) chunk_size, L) - 1.  Under
    path="auto" a chunk size that is not a multiple of 128 runs on the SIMT
    path, the one that has the state at any token."""
    lib = load_library()
    if x.dim() != 4 or B.dim() != 4:
        raise ValueError("x must be [b,L,H,P] and B, C [b,L,G,N]")
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dev = x.device
    _need_cuda("x", x)
    if x.dtype not in DTYPES:
        raise ValueError("x/B/C must be float32 or bfloat16")
    _need_cuda("B", B, x.dtype, (b, L, G, N))
    _need_cuda("C", C, x.dtype, (b, L, G, N))
    _need_cuda("dt_raw", dt_raw, torch.float32, (b, L, H))
    for nm, t in (("dt_bias", dt_bias), ("A", A), ("D", D)):
        _need_cuda(nm, t, torch.float32, (H,))
    if init_state is not None:
        _need_cuda("init_state", init_state, torch.float32, (b, H, N, P))
    if path == "auto" and int(chunk_size) % 128 != 0:
        path = "simt"
    nc = (L + int(chunk_size) - 1) // int(chunk_size)
    if y is None:
        y = torch.empty((b, L, H, P), dtype=torch.float32, device=dev)
    else:
        _need_cuda("y", y, torch.float32, (b, L, H, P))
    if final_state is None:
        final_state = torch.empty((b, H, N, P), dtype=torch.float32, device=dev)
    else:
        _need_cuda("final_state", final_state, torch.float32, (b, H, N, P))
    if chunk_states is None:
        chunk_states = torch.empty((b, nc, H, N, P), dtype=torch.float32, device=dev)
    else:
        _need_cuda("chunk_states", chunk_states, torch.float32, (b, nc, H, N, P))
    need = workspace_size(b, L, H, P, N, G, chunk_size, x.dtype, path)
    if workspace is None:
        workspace = alloc_workspace(need, dev)
    st = lib.ssd_chunk_scan_fwd_states(
        _ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(init_state),
        _ptr(y), _ptr(final_state), _ptr(chunk_states), b, L, H, P, N, G, int(chunk_size),
        float(dt_limit[0]), float(dt_limit[1]), DTYPES[x.dtype], PATHS[path],
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(dev))
    _check("ssd_chunk_scan_fwd_states", st)
    return y, final_state, chunk_states


def bwd_workspace_size(b: int, L: int, H: int, P: int, N: int, G: int, Q: int, in_dtype=torch.bfloat16) -> int:
    """Bytes of workspace ssd_chunk_scan_bwd needs for these sizes."""
    lib = load_library()
    out = ctypes.c_size_t(0)
    _check("ssd_chunk_scan_bwd_workspace_size",
           lib.ssd_chunk_scan_bwd_workspace_size(b, L, H, P, N, G, Q, DTYPES[in_dtype], ctypes.byref(out)))
    return int(out.value)


def chunk_scan_bwd(x: torch.Tensor, dt_raw: torch.Tensor, dt_bias: torch.Tensor, A: torch.Tensor,
                   B: torch.Tensor, C: torch.Tensor, D: torch.Tensor, dy: torch.Tensor,
                   dfinal_state: Optional[torch.Tensor] = None, init_state: Optional[torch.Tensor] = None,
                   chunk_size: int = 256, dt_limit: Tuple[float, float] = (0.0, math.inf),
                   workspace: Optional[torch.Tensor] = None, want_dinit: bool = True,
                   out: Optional[dict] = None, seq_idx: Optional[torch.Tensor] = None,
                   path: str = "simt") -> dict:
    """Deterministic backward of chunk_scan_fwd (ssd_chunk_scan_bwd), or of
    chunk_scan_fwd_varlen with the same seq_idx [b, L] int32 (packed rows,
    ssd_chunk_scan_bwd_varlen): the gradients of <dy, y> + <dfinal_state,
    final_state> with respect to every input, float32, keyed by input name
    ("x", "dt_raw", "dt_bias", "A", "B", "C", "D", "init_state"; the last None
    unless want_dinit).  `out` may hold preallocated outputs under the same
    keys.  path "simt" (fp32 CUDA cores), "tensor" (the block products on the
    tensor cores, bf16 inputs: the forward tensor path's precision) or
    "auto" (tensor where it applies)."""
    lib = load_library()
    if x.dim() != 4 or B.dim() != 4:
        raise ValueError("x must be [b,L,H,P] and B, C [b,L,G,N]")
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dev = x.device
    _need_cuda("x", x)
    if x.dtype not in DTYPES:
        raise ValueError("x/B/C must be float32 or bfloat16")
    _need_cuda("B", B, x.dtype, (b, L, G, N))
    _need_cuda("C", C, x.dtype, (b, L, G, N))
    _need_cuda("dt_raw", dt_raw, torch.float32, (b, L, H))
    _need_cuda("dy", dy, torch.float32, (b, L, H, P))
    for nm, t in (("dt_bias", dt_bias), ("A", A), ("D", D)):
        _need_cuda(nm, t, torch.float32, (H,))
    for nm, t in (("init_state", init_state), ("dfinal_state", dfinal_state)):
        if t is not None:
            _need_cuda(nm, t, torch.float32, (b, H, N, P))
    f = torch.float32
    shapes = {"x": (b, L, H, P), "dt_raw": (b, L, H), "dt_bias": (H,), "A": (H,), "B": (b, L, G, N),
              "C": (b, L, G, N), "D": (H,), "init_state": (b, H, N, P)}
    g = dict(out or {})
    for k, shp in shapes.items():
        if k == "init_state" and not want_dinit:
            g[k] = None
            continue
        if g.get(k) is None:
            g[k] = torch.empty(shp, dtype=f, device=dev)
        else:
            _need_cuda("out[%s]" % k, g[k], f, shp)
    Q = int(chunk_size)
    need = bwd_workspace_size(b, L, H, P, N, G, Q, x.dtype)
    if workspace is None:
        workspace = alloc_workspace(need, dev)
    if seq_idx is not None:
        _need_cuda("seq_idx", seq_idx, torch.int32, (b, L))
    st = lib.ssd_chunk_scan_bwd_varlen(
        _ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(init_state), _ptr(seq_idx),
        _ptr(dy),
        _ptr(dfinal_state), _ptr(g["x"]), _ptr(g["dt_raw"]), _ptr(g["dt_bias"]), _ptr(g["A"]), _ptr(g["B"]),
        _ptr(g["C"]), _ptr(g["D"]), _ptr(g["init_state"]), b, L, H, P, N, G, Q, float(dt_limit[0]),
        float(dt_limit[1]), DTYPES[x.dtype], PATHS[path], _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(dev))
    _check("ssd_chunk_scan_bwd_varlen", st)
    return g


def chunk_scan_fwd_varlen(x: torch.Tensor, dt_raw: torch.Tensor, dt_bias: torch.Tensor, A: torch.Tensor,
                          B: torch.Tensor, C: torch.Tensor, D: torch.Tensor, seq_idx: torch.Tensor,
                          init_state: Optional[torch.Tensor] = None, chunk_size: int = 256,
                          dt_limit: Tuple[float, float] = (0.0, math.inf), path: str = "auto",
                          workspace: Optional[torch.Tensor] = None, want_chunk_states: bool = False
                          ) -> Tuple[torch.Tensor, torch.Tensor, Optional[torch.Tensor]]:
    """Packed rows (ssd_chunk_scan_fwd_varlen): seq_idx [b, L] int32 document
    ids; the state restarts from zero at every document start (a row's first
    document from init_state).  Returns (y, final state, chunk-boundary
    states or None); with the states, path="auto" and a chunk size that is
    not a multiple of 128 runs on the SIMT path."""
    lib = load_library()
    if x.dim() != 4 or B.dim() != 4:
        raise ValueError("x must be [b,L,H,P] and B, C [b,L,G,N]")
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dev = x.device
    _need_cuda("x", x)
    if x.dtype not in DTYPES:
        raise ValueError("x/B/C must be float32 or bfloat16")
    _need_cuda("B", B, x.dtype, (b, L, G, N))
    _need_cuda("C", C, x.dtype, (b, L, G, N))
    _need_cuda("dt_raw", dt_raw, torch.float32, (b, L, H))
    _need_cuda("seq_idx", seq_idx, torch.int32, (b, L))
    for nm, t in (("dt_bias", dt_bias), ("A", A), ("D", D)):
        _need_cuda(nm, t, torch.float32, (H,))
    if init_state is not None:
        _need_cuda("init_state", init_state, torch.float32, (b, H, N, P))
    Q = int(chunk_size)
    y = torch.empty((b, L, H, P), dtype=torch.float32, device=dev)
    fs = torch.empty((b, H, N, P), dtype=torch.float32, device=dev)
    cs = torch.empty((b, (L + Q - 1) // Q, H, N, P), dtype=torch.float32, device=dev) if want_chunk_states else None
    if want_chunk_states and path == "auto" and Q % 128 != 0:
        path = "simt"
    need = workspace_size(b, L, H, P, N, G, Q, x.dtype, path)
    if workspace is None:
        workspace = alloc_workspace(need, dev)
    st = lib.ssd_chunk_scan_fwd_varlen(
        _ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(init_state), _ptr(seq_idx),
        _ptr(y), _ptr(fs), _ptr(cs), b, L, H, P, N, G, Q, float(dt_limit[0]), float(dt_limit[1]),
        DTYPES[x.dtype], PATHS[path], _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(dev))
    _check("ssd_chunk_scan_fwd_varlen", st)
    return y, fs, cs


def conv1d_silu_split(xbc: torch.Tensor, weight: torch.Tensor, bias: torch.Tensor, nheads: int, head_dim: int,
                      ngroups: int, state_dim: int) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Causal depthwise conv1d + SiLU over xbc [b, L, H*P + 2*G*N] (channels
    x | B | C), split into the scan's x [b,L,H,P], B and C [b,L,G,N] (same
    dtype as xbc).  weight [Cd, K] f32, bias [Cd] f32 (ssd_conv1d_silu_split)."""
    lib = load_library()
    if xbc.dim() != 3 or weight.dim() != 2:
        raise ValueError("xbc must be [b, L, Cd] and weight [Cd, K]")
    b, L, Cd = xbc.shape
    if Cd != nheads * head_dim + 2 * ngroups * state_dim:
        raise ValueError("xbc has %d channels, not H*P + 2*G*N" % Cd)
    _need_cuda("xbc", xbc)
    if xbc.dtype not in DTYPES:
        raise ValueError("xbc must be float32 or bfloat16")
    _need_cuda("weight", weight, torch.float32, (Cd, weight.shape[1]))
    _need_cuda("bias", bias, torch.float32, (Cd,))
    dev = xbc.device
    x = torch.empty((b, L, nheads, head_dim), dtype=xbc.dtype, device=dev)
    B = torch.empty((b, L, ngroups, state_dim), dtype=xbc.dtype, device=dev)
    C = torch.empty_like(B)
    st = lib.ssd_conv1d_silu_split(_ptr(xbc), _ptr(weight), _ptr(bias), _ptr(x), _ptr(B), _ptr(C), b, L, nheads,
                                   head_dim, ngroups, state_dim, weight.shape[1], DTYPES[xbc.dtype], _stream(dev))
    _check("ssd_conv1d_silu_split", st)
    return x, B, C


def conv_scan_fwd(xbc: torch.Tensor, conv_weight: torch.Tensor, conv_bias: torch.Tensor, dt_raw: torch.Tensor,
                  dt_bias: torch.Tensor, A: torch.Tensor, D: torch.Tensor, nheads: int, head_dim: int,
                  ngroups: int, state_dim: int, init_state: Optional[torch.Tensor] = None, chunk_size: int = 256,
                  dt_limit: Tuple[float, float] = (0.0, math.inf), workspace: Optional[torch.Tensor] = None,
                  y: Optional[torch.Tensor] = None, final_state: Optional[torch.Tensor] = None,
                  want_final_state: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """The conv1d and the scan in the combined arrangement (ssd_conv_scan_fwd):
    y and final_state of chunk_scan_fwd(*conv1d_silu_split(xbc, ...)) without
    writing x, B, C.  xbc [b, L, H*P + 2*G*N] bf16, conv_weight [Cd, 4] f32,
    conv_bias [Cd] f32; the rest as for chunk_scan_fwd (tensor-core shapes)."""
    lib = load_library()
    if xbc.dim() != 3:
        raise ValueError("xbc must be [b, L, Cd]")
    b, L, Cd = xbc.shape
    H, P, G, N = int(nheads), int(head_dim), int(ngroups), int(state_dim)
    if Cd != H * P + 2 * G * N:
        raise ValueError("xbc has %d channels, not H*P + 2*G*N" % Cd)
    dev = xbc.device
    _need_cuda("xbc", xbc, torch.bfloat16)
    _need_cuda("conv_weight", conv_weight, torch.float32, (Cd, conv_weight.shape[-1]))
    _need_cuda("conv_bias", conv_bias, torch.float32, (Cd,))
    _need_cuda("dt_raw", dt_raw, torch.float32, (b, L, H))
    for nm, t in (("dt_bias", dt_bias), ("A", A), ("D", D)):
        _need_cuda(nm, t, torch.float32, (H,))
    if init_state is not None:
        _need_cuda("init_state", init_state, torch.float32, (b, H, N, P))
    if y is None:
        y = torch.empty((b, L, H, P), dtype=torch.float32, device=dev)
    else:
        _need_cuda("y", y, torch.float32, (b, L, H, P))
    if want_final_state and final_state is None:
        final_state = torch.empty((b, H, N, P), dtype=torch.float32, device=dev)
    elif final_state is not None:
        _need_cuda("final_state", final_state, torch.float32, (b, H, N, P))
    need = workspace_size(b, L, H, P, N, G, chunk_size, torch.bfloat16, "tensor")
    if workspace is None:
        workspace = alloc_workspace(need, dev)
    st = lib.ssd_conv_scan_fwd(
        _ptr(xbc), _ptr(conv_weight), _ptr(conv_bias), conv_weight.shape[-1], _ptr(dt_raw), _ptr(dt_bias), _ptr(A),
        _ptr(D), _ptr(init_state), _ptr(y), _ptr(final_state), b, L, H, P, N, G, int(chunk_size),
        float(dt_limit[0]), float(dt_limit[1]), DTYPES[xbc.dtype], _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(dev))
    _check("ssd_conv_scan_fwd", st)
    return y, final_state


def gated_rmsnorm(y: torch.Tensor, z: torch.Tensor, weight: torch.Tensor, group_size: int,
                  eps: float = 1e-5) -> torch.Tensor:
    """out = rmsnorm_over_groups(y * silu(z)) * weight, f32 (ssd_gated_rmsnorm).
    y f32 [..., D], z [..., D] f32 or bf16, weight [D] f32."""
    lib = load_library()
    D = y.shape[-1]
    _need_cuda("y", y, torch.float32)
    _need_cuda("z", z, None, tuple(y.shape))
    if z.dtype not in DTYPES:
        raise ValueError("z must be float32 or bfloat16")
    _need_cuda("weight", weight, torch.float32, (D,))
    out = torch.empty(y.shape, dtype=torch.float32, device=y.device)
    st = lib.ssd_gated_rmsnorm(_ptr(y), _ptr(z), _ptr(weight), _ptr(out), y.numel() // D, D, int(group_size),
                               float(eps), DTYPES[z.dtype], _stream(y.device))
    _check("ssd_gated_rmsnorm", st)
    return out


def read_device_status(workspace: Optional[torch.Tensor]) -> int:
    """Synchronises the current stream and returns the device status code of
    the calls on `workspace`; with None, reads and clears the current
    device's status of the calls that take no workspace (conv1d)."""
    lib = load_library()
    if workspace is None:
        dev = torch.device("cuda", torch.cuda.current_device())
        return int(lib.ssd_read_device_status(None, _stream(dev)))
    return int(lib.ssd_read_device_status(_ptr(workspace), _stream(workspace.device)))


def step(x: torch.Tensor, dt_raw: torch.Tensor, dt_bias: torch.Tensor, A: torch.Tensor,
         B: torch.Tensor, C: torch.Tensor, D: torch.Tensor, state: torch.Tensor,
         dt_limit: Tuple[float, float] = (0.0, math.inf),
         y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One decode token: x [b,H,P], dt_raw [b,H] f32, B/C [b,G,N], state
    [b,H,N,P] f32 updated in place.  Returns y [b,H,P] f32."""
    lib = load_library()
    if x.dim() != 3 or B.dim() != 3:
        raise ValueError("x must be [b,H,P] and B, C [b,G,N]")
    b, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    _need_cuda("x", x)
    if x.dtype not in DTYPES:
        raise ValueError("x/B/C must be float32 or bfloat16")
    _need_cuda("B", B, x.dtype, (b, G, N))
    _need_cuda("C", C, x.dtype, (b, G, N))
    _need_cuda("dt_raw", dt_raw, torch.float32, (b, H))
    for nm, t in (("dt_bias", dt_bias), ("A", A), ("D", D)):
        _need_cuda(nm, t, torch.float32, (H,))
    _need_cuda("state", state, torch.float32, (b, H, N, P))
    if y is None:
        y = torch.empty((b, H, P), dtype=torch.float32, device=x.device)
    else:
        _need_cuda("y", y, torch.float32, (b, H, P))
    st = lib.ssd_step(_ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                      _ptr(state), _ptr(y), b, H, P, N, G, float(dt_limit[0]), float(dt_limit[1]),
                      DTYPES[x.dtype], _stream(x.device))
    _check("ssd_step", st)
    return y


def trace_enable(max_launches: int) -> None:
    """Start (max_launches > 0) or stop (0) per-kernel event tracing."""
    _check("ssd_trace_enable", load_library().ssd_trace_enable(int(max_launches)))


def trace_read() -> dict:
    """{kernel name: (launches, total device ms)} for every traced kernel."""
    lib = load_library()
    out = {}
    for k in range(lib.ssd_trace_kernel_count()):
        n = ctypes.c_int(0)
        ms = ctypes.c_double(0.0)
        _check("ssd_trace_read", lib.ssd_trace_read(k, ctypes.byref(n), ctypes.byref(ms)))
        if n.value:
            out[lib.ssd_trace_kernel_name(k).decode()] = (int(n.value), float(ms.value))
    return out
