"""The C ABI library on the host: it loads, exports what include/la_seg.h declares, sizes its
workspace, and rejects bad arguments before touching a GPU (CPU only, no compute calls)."""
import ctypes
import os
import re

import pytest

from sequence_linear_attention_chunked_b200 import build as la_build
from sequence_linear_attention_chunked_b200 import la_seg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "la_seg.h")


@pytest.fixture(scope="module")
def lib():
    la_build.build()
    return la_seg.lib()


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"LA_API\s+[\w\s\*]+?\b(la_\w+)\s*\(", src)))


def test_header_declares_binding_symbols():
    assert declared_symbols() == sorted(la_seg.EXPORTED)


def test_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {la_seg.LIB_PATH}").read()
    exported = set(re.findall(r" T (la_\w+)", out))
    assert set(declared_symbols()) <= exported


def test_workspace_sizes(lib):
    w = la_seg.la_seg_workspace_bytes
    assert w(1, 16, 16384, 128, 128, 1, 64) > 0
    assert w(1, 16, 4194304, 128, 128, 256, 64) > 0
    assert w(1, 2, 256, 32, 32, 4, 16, la_seg.LA_F32) > 0
    assert w(1, 1, 0, 32, 32, 1, 16) > 0  # empty sequence is legal
    # rejected sizes report 0
    assert w(1, 1, 100, 32, 32, 3, 16) == 0     # L % P
    assert w(1, 1, 96, 32, 32, 1, 64) == 0      # segment not a multiple of chunk
    assert w(1, 1, 64, 48, 48, 1, 16) == 0      # d not supported
    assert w(1, 1, 64, 32, 64, 1, 16) == 0      # dk != dv
    assert w(1, 1, 64, 32, 32, 1, 8) == 0       # chunk not supported
    assert w(1, 1, 64, 32, 32, 1, 16, 7) == 0   # dtype


def _fwd(lib, **kw):
    """Calls la_seg_forward with fake (but aligned) pointers: only argument checks may run."""
    args = dict(q=0x1000, k=0x2000, v=0x3000, g=0x4000, S0=None, B=1, H=1, L=64, dk=32, dv=32,
                P=1, chunk=16, dt=0, o=0x5000, Sf=None, Sr=None, sched=0, ws=0x10000,
                ws_bytes=1 << 30, stream=None)
    args.update(kw)
    V = ctypes.c_void_p
    return lib.la_seg_forward(V(args["q"]), V(args["k"]), V(args["v"]), V(args["g"]),
                              V(args["S0"]), args["B"], args["H"], args["L"], args["dk"],
                              args["dv"], args["P"], args["chunk"], args["dt"], V(args["o"]),
                              V(args["Sf"]), V(args["Sr"]), args["sched"], V(args["ws"]),
                              args["ws_bytes"], V(args["stream"]))


@pytest.mark.parametrize("kw,status", [
    (dict(L=100, P=3), -2),
    (dict(L=96, chunk=64), -2),
    (dict(dk=48, dv=48), -2),
    (dict(dk=32, dv=64), -2),
    (dict(chunk=8), -2),
    (dict(B=0), -2),
    (dict(P=0), -2),
    (dict(L=-64), -2),
    (dict(dt=5), -4),
    (dict(q=None), -1),
    (dict(o=None), -1),
    (dict(sched=9), -1),
    (dict(q=0x1008), -3),
    (dict(S0=0x7004), -3),
    (dict(ws=None), -5),
    (dict(ws_bytes=16), -5),
    (dict(ws=0x10010), -3),
])
def test_forward_rejects_bad_arguments(lib, kw, status):
    assert _fwd(lib, **kw) == status
    assert len(la_seg.la_last_error_detail()) > 0


def _scan(lib, S_in=0x1000, lg=0x2000, d=32, dv=None, out=0x3000, S_next=None, S_last=None,
          carry=None):
    """la_seg_scan with fake (but aligned) pointers: only argument checks may run."""
    V = ctypes.c_void_p
    return lib.la_seg_scan(V(S_in), V(lg), None, 1, 2, d, d if dv is None else dv, 0, V(out),
                           None, V(S_next), V(S_last), V(carry), None, None)


def test_scan_rejects_bad_arguments(lib):
    assert _scan(lib, dv=30) == -2
    assert _scan(lib, S_in=None) == -1
    assert _scan(lib, S_in=0x1004) == -3
    assert _scan(lib, out=0x1000) == -1                        # out aliases S_in
    assert _scan(lib, carry=0x5000) == -1                      # carry needs S_next
    assert _scan(lib, dv=24, S_next=0x4000, carry=0x5000) == -2  # dv / 4 must divide 32
    assert _scan(lib, S_next=0x4008, carry=0x5000) == -3
    assert _scan(lib, S_next=0x4000, S_last=0x6004, carry=0x5000) == -3


def test_error_detail_handles_small_buffers(lib):
    assert _fwd(lib, chunk=8) == -2
    buf = ctypes.create_string_buffer(8)
    assert lib.la_last_error_detail(buf, 8) == 0
    assert len(buf.value) == 7
    assert lib.la_last_error_detail(None, 8) == -1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(la_seg, "_lib", None)
    monkeypatch.setattr(la_seg, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        la_seg.lib()


def _bwd(lib, **kw):
    """Calls la_seg_backward with fake (but aligned) pointers: only argument checks may run."""
    a = dict(q=0x1000, k=0x2000, v=0x3000, g=0x4000, S0=None, Sr=None, dO=0x5000, dSf=None, B=1,
             H=1, L=64, d=32, P=1, chunk=16, dt=0, dq=0x6000, dk=0x7000, dv=0x8000, dg=0x9000,
             dS0=None, ws=0x10000, ws_bytes=1 << 30)
    a.update(kw)
    V = ctypes.c_void_p
    return lib.la_seg_backward(V(a["q"]), V(a["k"]), V(a["v"]), V(a["g"]), V(a["S0"]), V(a["Sr"]),
                               V(a["dO"]), V(a["dSf"]), a["B"], a["H"], a["L"], a["d"], a["d"],
                               a["P"], a["chunk"], a["dt"], V(a["dq"]), V(a["dk"]), V(a["dv"]),
                               V(a["dg"]), V(a["dS0"]), V(a["ws"]), a["ws_bytes"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(L=100, P=3), -2), (dict(d=48), -2), (dict(chunk=128), -2), (dict(dt=2), -4),
    (dict(dO=None), -1), (dict(dg=None), -1), (dict(dq=0x6004), -3), (dict(Sr=0x1234), -3),
    (dict(ws=None), -5), (dict(ws_bytes=1024), -5),
])
def test_backward_rejects_bad_arguments(lib, kw, status):
    assert _bwd(lib, **kw) == status


def test_backward_workspace_covers_both_splits(lib):
    w = la_seg.la_seg_workspace_bytes
    # C4: the fwd+bwd workload; the backward needs the fp32 dq staging buffer
    need = w(2, 16, 131072, 128, 128, 8, 64, la_seg.LA_BF16, True)
    assert need >= 2 * 16 * 131072 * 128 * 4
    assert w(2, 16, 131072, 128, 128, 8, 64, la_seg.LA_BF16, False) < need


def _chain(lib, **kw):
    """Calls la_seg_chain_pass with fake (but aligned) pointers: only argument checks may run."""
    a = dict(q=0x1000, k=0x2000, v=0x3000, g=0x4000, B=1, H=2, L=1024, d=128, NP=4, chunk=64,
             dt=la_seg.LA_BF16, states=0x8000, ready=0x9000, o=0x5000, Sf=None, Ss=None, every=1,
             status=None)
    a.update(kw)
    V = ctypes.c_void_p
    return lib.la_seg_chain_pass(V(a["q"]), V(a["k"]), V(a["v"]), V(a["g"]), a["B"], a["H"],
                                 a["L"], a["d"], a["d"], a["NP"], a["chunk"], a["dt"],
                                 V(a["states"]), V(a["ready"]), V(a["o"]), V(a["Sf"]), V(a["Ss"]),
                                 a["every"], V(a["status"]), None)


@pytest.mark.parametrize("kw,status", [
    (dict(dt=la_seg.LA_F32), -2),      # the single pass exists for bf16, d = 128, chunk 64 only
    (dict(d=64), -2),
    (dict(chunk=32), -2),
    (dict(NP=3), -2),                  # L % NP
    (dict(states=None), -1),
    (dict(ready=None), -1),
    (dict(o=None), -1),
    (dict(every=0), -1),
    (dict(every=3), -1),               # save_every must divide NP
    (dict(states=0x8004), -3),
    (dict(Sf=0x7008), -3),
    (dict(dt=9), -4),
])
def test_chain_pass_rejects_bad_arguments(lib, kw, status):
    assert _chain(lib, **kw) == status
    assert len(la_seg.la_last_error_detail()) > 0


def test_chain_reset_rejects_bad_arguments(lib):
    V = ctypes.c_void_p
    reset = lib.la_seg_chain_reset
    assert reset(None, 0, 2, 128, 128, V(0x8000), V(0x9000), None) == -2
    assert reset(None, 1, 2, 48, 48, V(0x8000), V(0x9000), None) == -2
    assert reset(None, 1, 2, 128, 128, None, V(0x9000), None) == -1
    assert reset(None, 1, 2, 128, 128, V(0x8000), None, None) == -1
    assert reset(V(0x7004), 1, 2, 128, 128, V(0x8000), V(0x9000), None) == -3


def test_single_pass_and_overlap_schedules_are_accepted(lib):
    # an unknown schedule is rejected, the single pass and the overlap schedule are not (the
    # call then stops at the workspace check, before any launch)
    assert _fwd(lib, sched=5) == -1
    assert _fwd(lib, sched=-1) == -1
    assert _fwd(lib, sched=la_seg.SCHED_SINGLE_PASS, ws=None) == -5
    assert _fwd(lib, sched=la_seg.SCHED_OVERLAP, ws=None) == -5


def test_local_pass_states_go_together(lib):
    # S_loc without log_gamma (or the reverse) is an argument error, found before any launch
    V, L_ = ctypes.c_void_p, ctypes.c_longlong
    f = lib.la_seg_local_pass
    for sl, lgm in ((0x6000, None), (None, 0x7000)):
        st = f(V(0x1000), V(0x2000), V(0x3000), V(0x4000), 1, 1, L_(64), 32, 32, 1, 16, 0,
               V(0x5000), V(sl) if sl else None, V(lgm) if lgm else None, None, None)
        assert st == -1
