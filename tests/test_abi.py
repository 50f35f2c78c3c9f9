"""Host-side checks of the C ABI: the library loads, exports every entry
point include/ssd.h declares, and rejects bad arguments before touching the
GPU (no compute call is made here)."""
import ctypes
import math
import os
import re

import pytest

from state_space_sequence_scan_b200 import ssd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"SSD_API\s+[\w\s\*]*?\b(ssd_\w+)\s*\(", txt)
    return names


@pytest.fixture(scope="module")
def lib():
    from state_space_sequence_scan_b200 import build
    build.build_library()
    return ssd.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 7
    for n in names:
        assert hasattr(lib, n), n
    assert set(ssd.EXPORTED) <= set(names)


def test_test_fault_hook_validates_its_argument(lib):
    """The timeout-path test hook takes 0 (off) or 1 only; host-side, no GPU."""
    assert lib.ssd_set_test_fault(7) == 1
    assert lib.ssd_set_test_fault(-1) == 1
    assert lib.ssd_set_test_fault(0) == 0


def test_version_and_status_strings(lib):
    assert lib.ssd_version() >> 16 == 1
    for code in range(8):
        s = lib.ssd_status_string(code)
        assert s and s != b"unknown status"
    assert lib.ssd_status_string(99) == b"unknown status"


def _ws(lib, *dims, dtype=1, path=0):
    out = ctypes.c_size_t(0)
    st = lib.ssd_chunk_scan_workspace_size(*dims, dtype, path, ctypes.byref(out))
    return st, out.value


def test_workspace_size_validation(lib):
    assert _ws(lib, 1, 64, 4, 16, 16, 1, 16, dtype=0)[0] == 0
    assert _ws(lib, 1, 64, 4, 16, 16, 1, 16, dtype=0)[1] >= 256
    assert _ws(lib, 1, 64, 4, 16, 16, 3, 16)[0] == 1          # H % G != 0
    assert _ws(lib, 1, 64, 0, 16, 16, 1, 16)[0] == 1          # no heads
    assert _ws(lib, 1, 64, 4, 16, 16, 1, 0)[0] == 1           # chunk 0
    assert _ws(lib, -1, 64, 4, 16, 16, 1, 16)[0] == 1
    assert _ws(lib, 1, 64, 4, 16, 16, 1, 16, dtype=7)[0] == 2  # unknown dtype
    assert _ws(lib, 1, 64, 4, 16, 16, 1, 16, path=9)[0] == 1   # unknown path
    assert _ws(lib, 1, 64, 4, 24, 16, 1, 16)[0] == 2          # head_dim must divide 256 (SIMT)
    st = lib.ssd_chunk_scan_workspace_size(1, 64, 4, 16, 16, 1, 16, 0, 0, None)
    assert st == 1


def test_workspace_grows_with_chunks(lib):
    _, small = _ws(lib, 2, 1024, 4, 64, 128, 1, 256, path=1)
    _, big = _ws(lib, 2, 1024, 4, 64, 128, 1, 16, path=1)
    assert big > small > 0


def _fwd(lib, **kw):
    a = dict(x=None, dt_raw=None, dt_bias=None, A=None, B=None, C=None, D=None, init=None, y=None, fs=None,
             b=1, L=8, H=2, P=16, N=16, G=1, Q=4, lo=0.0, hi=math.inf, dtype=0, path=0, ws=None, wsb=0,
             stream=None)
    a.update(kw)
    return lib.ssd_chunk_scan_fwd(a["x"], a["dt_raw"], a["dt_bias"], a["A"], a["B"], a["C"], a["D"], a["init"],
                                  a["y"], a["fs"], a["b"], a["L"], a["H"], a["P"], a["N"], a["G"], a["Q"],
                                  a["lo"], a["hi"], a["dtype"], a["path"], a["ws"], a["wsb"], a["stream"])


def test_forward_rejects_bad_arguments_on_host(lib):
    fake = 0x10000          # aligned non-null stand-in; never dereferenced (calls fail validation first)
    ok = dict(x=fake, dt_raw=fake, dt_bias=fake, A=fake, B=fake, C=fake, D=fake, y=fake, fs=fake)
    assert _fwd(lib) == 1                                     # null pointers
    assert _fwd(lib, **ok, H=3, G=2) == 1                     # H % G
    assert _fwd(lib, **ok, lo=0.5, hi=0.1) == 1               # dt limits reversed
    assert _fwd(lib, **ok, lo=-1.0) == 1                      # negative lower limit
    assert _fwd(lib, **ok, lo=float("nan")) == 1
    assert _fwd(lib, **dict(ok, x=fake + 4)) == 3             # misaligned
    assert _fwd(lib, **ok) == 4                               # no workspace
    assert _fwd(lib, **ok, ws=fake, wsb=16) == 4              # workspace too small
    assert _fwd(lib, **ok, ws=fake + 16, wsb=1 << 30) == 3    # workspace not 256-aligned
    assert _fwd(lib, **ok, dtype=5) == 2
    assert _fwd(lib, **ok, path=2, dtype=0) == 2              # tensor path needs bf16


def _fwd_states(lib, **kw):
    a = dict(x=None, dt_raw=None, dt_bias=None, A=None, B=None, C=None, D=None, init=None, y=None, fs=None,
             cs=None, b=1, L=8, H=2, P=16, N=16, G=1, Q=4, lo=0.0, hi=math.inf, dtype=0, path=0, ws=None, wsb=0,
             stream=None)
    a.update(kw)
    return lib.ssd_chunk_scan_fwd_states(a["x"], a["dt_raw"], a["dt_bias"], a["A"], a["B"], a["C"], a["D"],
                                         a["init"], a["y"], a["fs"], a["cs"], a["b"], a["L"], a["H"], a["P"],
                                         a["N"], a["G"], a["Q"], a["lo"], a["hi"], a["dtype"], a["path"], a["ws"],
                                         a["wsb"], a["stream"])


def test_forward_states_rejects_bad_arguments_on_host(lib):
    """The chunk-states entry point checks as the plain one does, plus: the
    states pointer's alignment, and that a call resolving to the tensor path
    has a chunk size that is a multiple of its 128-token blocks."""
    fake = 0x10000
    ok = dict(x=fake, dt_raw=fake, dt_bias=fake, A=fake, B=fake, C=fake, D=fake, y=fake, fs=fake, cs=fake)
    assert _fwd_states(lib) == 1
    assert _fwd_states(lib, **dict(ok, cs=fake + 4)) == 3                  # misaligned states
    assert _fwd_states(lib, **ok) == 4                                     # no workspace (SIMT, any Q)
    tc = dict(ok, dtype=1, H=2, P=64, N=128, G=1, L=512)
    for path in (0, 2):                                                    # auto resolves to the tensor path
        assert _fwd_states(lib, **tc, Q=64, path=path) == 2                # no 64-token boundary there
        assert _fwd_states(lib, **tc, Q=128, path=path) == 4               # fine, then no workspace
        assert _fwd_states(lib, **dict(tc, cs=None), Q=64, path=path) == 4  # no states: as the plain call
    assert _fwd_states(lib, **tc, Q=64, path=1) == 4                       # SIMT takes it


def test_forward_varlen_rejects_bad_arguments_on_host(lib):
    """Packed rows: seq_idx 4-byte aligned; both paths take them (then no
    workspace here)."""
    fake = 0x10000
    f = lambda **kw: lib.ssd_chunk_scan_fwd_varlen(
        *([fake] * 8), kw.get("si", fake), fake, fake, None, 1, 512, 2, 64, 128, 1, kw.get("Q", 128), 0.0, math.inf,
        1, kw.get("path", 0), None, 0, None)
    assert f(si=fake + 2) == 3                         # misaligned ids
    for path in (0, 1, 2):
        assert f(path=path) == 4 and f(Q=64, path=path) == 4


def _bwd(lib, **kw):
    fake = 0x10000
    a = dict(ptrs=[fake] * 18, b=1, L=64, H=2, P=16, N=16, G=1, Q=16, lo=0.0, hi=math.inf, dtype=0, ws=None, wsb=0)
    a.update(kw)
    return lib.ssd_chunk_scan_bwd(*a["ptrs"], a["b"], a["L"], a["H"], a["P"], a["N"], a["G"], a["Q"], a["lo"],
                                  a["hi"], a["dtype"], a["ws"], a["wsb"], None)


def test_backward_rejects_bad_arguments_on_host(lib):
    """The backward checks its sizes, pointers and workspace before anything
    is enqueued: head_dim 8/16/32/64, state_dim a multiple of 8 up to 128."""
    fake = 0x10000
    sz = ctypes.c_size_t(0)
    assert lib.ssd_chunk_scan_bwd_workspace_size(1, 64, 2, 16, 16, 1, 16, 0, ctypes.byref(sz)) == 0 and sz.value > 0
    for P, N, want in ((48, 16, 2), (16, 136, 2), (16, 12, 2), (128, 16, 2), (64, 128, 0), (8, 8, 0)):
        assert lib.ssd_chunk_scan_bwd_workspace_size(1, 64, 2, P, N, 1, 16, 0, ctypes.byref(sz)) == want, (P, N)
    assert lib.ssd_chunk_scan_bwd_workspace_size(1, 64, 3, 16, 16, 2, 16, 0, ctypes.byref(sz)) == 1   # H % G
    assert _bwd(lib) == 4                                                  # no workspace
    assert _bwd(lib, ptrs=[fake] * 8 + [None] + [fake] * 9) == 1          # dy missing
    assert _bwd(lib, ptrs=[fake] * 10 + [fake + 4] + [fake] * 7) == 3     # dx misaligned
    assert _bwd(lib, ptrs=[fake] * 11 + [fake + 2] + [fake] * 6) == 3     # ddt_raw misaligned
    assert _bwd(lib, P=48) == 2
    assert _bwd(lib, lo=0.5, hi=0.1) == 1
    assert _bwd(lib, ws=fake, wsb=16) == 4
    assert _bwd(lib, ws=fake + 16, wsb=1 << 30) == 3


def test_front_back_reject_bad_arguments_on_host(lib):
    """The conv1d and gated-norm entry points check sizes, dtypes and
    alignment before anything is queued."""
    fake = 0x10000
    conv = lambda **kw: lib.ssd_conv1d_silu_split(*([kw.get("p", fake)] * 3), *([kw.get("o", fake)] * 3),
                                                  kw.get("b", 2), kw.get("L", 40), kw.get("H", 4), kw.get("P", 16),
                                                  kw.get("G", 2), kw.get("N", 16), kw.get("K", 4),
                                                  kw.get("dtype", 1), None)
    assert conv(b=0) == 0 and conv(L=0) == 0          # nothing to do
    assert conv(H=0) == 1
    assert conv(K=5) == 2 and conv(K=0) == 2           # widths 1..4
    assert conv(P=5) == 2                              # H*P = 20, not a multiple of 8
    assert conv(dtype=7) == 2
    assert conv(p=None) == 1
    assert conv(o=fake + 8) == 3                       # misaligned outputs
    norm = lambda **kw: lib.ssd_gated_rmsnorm(kw.get("y", fake), kw.get("z", fake), fake, kw.get("out", fake),
                                              kw.get("T", 10), kw.get("D", 64), kw.get("g", 16), kw.get("eps", 1e-5),
                                              kw.get("dtype", 1), None)
    assert norm(T=0) == 0
    assert norm(g=24) == 1                             # 64 % 24
    assert norm(g=6, D=60) == 2                        # group not a multiple of 4
    assert norm(eps=-1.0) == 1 and norm(eps=float("nan")) == 1
    assert norm(y=None) == 1
    assert norm(out=fake + 4) == 3 and norm(z=fake + 2) == 3


def test_step_rejects_bad_arguments_on_host(lib):
    fake = 0x10000
    f = lambda **kw: lib.ssd_step(*([kw.get("p", fake)] * 9), kw.get("b", 2), kw.get("H", 4), kw.get("P", 16),
                                 kw.get("N", 16), kw.get("G", 2), kw.get("lo", 0.0), kw.get("hi", math.inf),
                                 kw.get("dtype", 1), None)
    assert f(p=None) == 1
    assert f(H=3) == 1
    assert f(P=6) == 2
    assert f(P=12) == 2                                       # 12/4 = 3 does not divide 256
    assert f(dtype=3) == 2
    assert f(lo=2.0, hi=1.0) == 1
    assert f(b=0) == 0                                        # empty batch: nothing to do
    assert lib.ssd_step(*([fake + 8] * 9), 2, 4, 16, 16, 2, 0.0, math.inf, 1, None) == 3


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 4, 2, 16)
    with pytest.raises(ValueError):
        ssd.chunk_scan_fwd(x, torch.zeros(1, 4, 2), torch.zeros(2), torch.zeros(2), torch.zeros(1, 4, 1, 16),
                           torch.zeros(1, 4, 1, 16), torch.zeros(2), chunk_size=4)


def test_backward_workspace_holds_per_head_buffers_only_when_groups_are_shared(lib):
    """With G < H the pair kernels write per-head dB, dC ([b, L, H, N] f32
    each) that a last launch sums per group; with G = H they write dB, dC
    directly and the workspace has no room for them."""
    sz = ctypes.c_size_t(0)

    def ws(G):
        assert lib.ssd_chunk_scan_bwd_workspace_size(2, 300, 4, 64, 128, G, 64, 1, ctypes.byref(sz)) == 0
        return sz.value

    per_head = 2 * 2 * 300 * 4 * 128 * 4
    assert ws(2) - ws(4) >= per_head
    assert ws(1) == ws(2)
