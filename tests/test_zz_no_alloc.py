"""la_seg_forward_noalloc: the forward for callers that cannot allocate device memory.

Such callers (plug-ins inside an engine that owns all device memory, runtimes that forbid
allocation after start-up, hosts that reach the C ABI but not the CUDA allocator) get the
forward pass with its scratch in a static device array.  These tests call it through the
C ABI and check it against la_seg_forward, which takes a caller-provided workspace: both run
the same kernels in the same order, so the results must agree bit for bit.  The file is
named to be collected last.
"""
import ctypes

import pytest
import torch

from sequence_linear_attention_chunked_b200 import la_seg
from sequence_linear_attention_chunked_b200.inputs import WORKLOADS, Workload, make_inputs
from tests.parity import TOL, rel_err

NOALLOC_BYTES = 32 << 20
SCHEDULES = {"auto": la_seg.SCHED_AUTO, "two_pass": la_seg.SCHED_TWO_PASS,
             "three_phase": la_seg.SCHED_THREE_PHASE, "single_pass": la_seg.SCHED_SINGLE_PASS,
             "overlap": la_seg.SCHED_OVERLAP}


def _noalloc(x, w, o, Sf, Sr, schedule):
    dt = la_seg.LA_F32 if w.dtype == "f32" else la_seg.LA_BF16
    st = la_seg.lib().la_seg_forward_noalloc(
        la_seg._ptr(x["q"]), la_seg._ptr(x["k"]), la_seg._ptr(x["v"]), la_seg._ptr(x["log_g"]),
        la_seg._ptr(x.get("S0")), w.B, w.H, w.L, w.dk, w.dv, w.P, w.chunk, dt, la_seg._ptr(o),
        la_seg._ptr(Sf), la_seg._ptr(Sr), schedule, la_seg._stream(None))
    la_seg._check(st, "la_seg_forward_noalloc")


CASES = [WORKLOADS["C0"], WORKLOADS["C1"].with_(H=4, L=8192, P=2),
         Workload("mixed", 2, 3, 1536, 64, 64, 3, 32, "bf16", "gla")]


@pytest.mark.gpu
@pytest.mark.parametrize("sched", list(SCHEDULES), ids=str)
@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_matches_workspace_forward(cuda_device, w, sched):
    B, H, L, d, P = w.B, w.H, w.L, w.dk, w.P
    assert la_seg.la_seg_workspace_bytes(B, H, L, d, d, P, w.chunk,
                                         la_seg._dt(torch.empty(0, dtype=w.torch_dtype))) <= NOALLOC_BYTES
    # two calls in a row, on different inputs, each against the workspace entry point with the
    # same schedule: the shared array keeps the previous call's contents (the single pass's
    # chain counters among them), which must not leak into the next result
    for seed in (0, 1):
        x = make_inputs(w.with_(seed=seed), cuda_device, with_s0=(seed == 1))
        o_ref, Sf_ref, Sr_ref = la_seg.la_seg_forward(x["q"], x["k"], x["v"], x["log_g"],
                                                      x.get("S0"), P, w.chunk, SCHEDULES[sched],
                                                      want_S_recv=True)
        o = torch.full_like(o_ref, float("nan"))
        Sf = torch.full_like(Sf_ref, float("nan"))
        Sr = torch.full_like(Sr_ref, float("nan"))
        _noalloc(x, w, o, Sf, Sr, SCHEDULES[sched])
        # the status word of the static scratch: a clean run reports LA_OK
        la_seg._check(la_seg.lib().la_seg_noalloc_check_status(la_seg._stream(None)),
                      "la_seg_noalloc_check_status")
        tol = TOL[w.torch_dtype]
        for got, ref in ((o, o_ref), (Sf, Sf_ref), (Sr, Sr_ref)):
            assert torch.equal(got, ref)
            assert rel_err(got, ref.double().cpu().numpy()) <= tol


def test_noalloc_rejects_oversized_work():
    """Sizes whose scratch exceeds the static array are refused before any device work."""
    V = ctypes.c_void_p
    w = WORKLOADS["C2"]
    need = la_seg.la_seg_workspace_bytes(w.B, w.H, w.L, w.dk, w.dv, w.P, w.chunk)
    assert need > NOALLOC_BYTES
    st = la_seg.lib().la_seg_forward_noalloc(V(0x1000), V(0x2000), V(0x3000), V(0x4000), None,
                                             w.B, w.H, w.L, w.dk, w.dv, w.P, w.chunk, 1,
                                             V(0x5000), None, None, 0, None)
    assert st == -5
    assert "static scratch" in la_seg.la_last_error_detail()
    # rejected shapes report the same error as la_seg_forward
    st = la_seg.lib().la_seg_forward_noalloc(V(0x1000), V(0x2000), V(0x3000), V(0x4000), None,
                                             1, 1, 100, 32, 32, 3, 16, 0, V(0x5000), None, None,
                                             0, None)
    assert st == -2
