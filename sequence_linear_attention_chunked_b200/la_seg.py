"""ctypes binding of libla_seg.so -- argument marshalling only.

Every step of the computation runs in the library's CUDA kernels; this module checks tensor
placement and dtypes, allocates outputs and the workspace through PyTorch (plumbing), passes
raw device pointers and the current CUDA stream, and raises ``LaSegError`` on any non-OK
status.  There is no CPU or PyTorch fallback: if the library is missing, importing the
functions fails loudly.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libla_seg.so")

LA_OK = 0
STATUS_NAMES = {0: "LA_OK", -1: "LA_ERR_ARG", -2: "LA_ERR_SHAPE", -3: "LA_ERR_ALIGN",
                -4: "LA_ERR_DTYPE", -5: "LA_ERR_WORKSPACE", -6: "LA_ERR_GATE_RANGE",
                -7: "LA_ERR_TIMEOUT", -8: "LA_ERR_CUDA"}
LA_F32, LA_BF16 = 0, 1
SCHED_AUTO, SCHED_TWO_PASS, SCHED_THREE_PHASE, SCHED_SINGLE_PASS, SCHED_OVERLAP = 0, 1, 2, 3, 4
EXPORTED = ("la_seg_workspace_bytes", "la_seg_forward", "la_seg_backward", "la_seg_scan",
            "la_seg_state_pass", "la_seg_local_pass", "la_seg_output_pass", "la_seg_correct_pass",
            "la_seg_subsegments", "la_seg_check_status", "la_last_error_detail",
            "la_seg_forward_noalloc", "la_seg_dstate_pass", "la_seg_dq_pass", "la_seg_dkv_pass",
            "la_seg_backward_parts", "la_seg_chain_pass", "la_seg_chain_reset",
            "la_seg_noalloc_check_status", "la_seg_gather_states", "la_seg_log_gamma_total",
            "la_seg_rank_scan", "la_seg_combine", "la_seg_train_saved_states",
            "la_seg_train_workspace_bytes", "la_seg_train_forward", "la_seg_train_backward")

_lib = None


class LaSegError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {detail}")


def lib():
    """The loaded library (ctypes.CDLL) with argument types declared."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m sequence_linear_attention_chunked_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t
        L.la_seg_workspace_bytes.argtypes = [i32, i32, i64, i32, i32, i32, i32, i32, i32]
        L.la_seg_workspace_bytes.restype = sz
        L.la_seg_forward.argtypes = [P, P, P, P, P, i32, i32, i64, i32, i32, i32, i32, i32,
                                     P, P, P, i32, P, sz, P]
        L.la_seg_forward.restype = i32
        L.la_seg_backward.argtypes = [P, P, P, P, P, P, P, P, i32, i32, i64, i32, i32, i32, i32,
                                      i32, P, P, P, P, P, P, sz, P]
        L.la_seg_backward.restype = i32
        L.la_seg_scan.argtypes = [P, P, P, i32, i32, i32, i32, i32, P, P, P, P, P, P, P]
        L.la_seg_scan.restype = i32
        L.la_seg_state_pass.argtypes = [P, P, P, i32, i32, i64, i32, i32, i32, i32, i32, P, P, P, P]
        L.la_seg_state_pass.restype = i32
        L.la_seg_local_pass.argtypes = [P, P, P, P, i32, i32, i64, i32, i32, i32, i32, i32, P, P, P,
                                        P, P]
        L.la_seg_local_pass.restype = i32
        L.la_seg_output_pass.argtypes = [P, P, P, P, P, i32, i32, i64, i32, i32, i32, i32, i32, P,
                                         P, P]
        L.la_seg_output_pass.restype = i32
        L.la_seg_correct_pass.argtypes = [P, P, P, i32, i32, i64, i32, i32, i32, i32, i32, P, P, P]
        L.la_seg_correct_pass.restype = i32
        L.la_seg_subsegments.argtypes = [i32, i32, i64, i32, i32, i32, i32, i32]
        L.la_seg_subsegments.restype = i32
        L.la_seg_forward_noalloc.argtypes = [P, P, P, P, P, i32, i32, i64, i32, i32, i32, i32,
                                             i32, P, P, P, i32, P]
        L.la_seg_forward_noalloc.restype = i32
        L.la_seg_train_saved_states.argtypes = [i32, i32, i64, i32, i32, i32, i32, i32]
        L.la_seg_train_saved_states.restype = i32
        L.la_seg_train_workspace_bytes.argtypes = [i32, i32, i64, i32, i32, i32, i32, i32, i32]
        L.la_seg_train_workspace_bytes.restype = sz
        L.la_seg_train_forward.argtypes = L.la_seg_forward.argtypes
        L.la_seg_train_forward.restype = i32
        L.la_seg_train_backward.argtypes = L.la_seg_backward.argtypes
        L.la_seg_train_backward.restype = i32
        L.la_seg_log_gamma_total.argtypes = [P, i32, i32, i32, P, P]
        L.la_seg_log_gamma_total.restype = i32
        L.la_seg_rank_scan.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, P, P, P]
        L.la_seg_rank_scan.restype = i32
        L.la_seg_combine.argtypes = [P, P, P, P, i32, i32, i32, P, P, P]
        L.la_seg_combine.restype = i32
        L.la_seg_gather_states.argtypes = [P, i32, i32, i32, i32, i32, P, P]
        L.la_seg_gather_states.restype = i32
        L.la_seg_noalloc_check_status.argtypes = [P]
        L.la_seg_noalloc_check_status.restype = i32
        L.la_seg_dstate_pass.argtypes = [P, P, P, i32, i32, i64, i32, i32, i32, i32, i32, P, P,
                                         P, P]
        L.la_seg_dstate_pass.restype = i32
        L.la_seg_dq_pass.argtypes = [P, P, P, P, P, P, i32, i32, i64, i32, i32, i32, i32, i32,
                                     i32, P, P, P, P, P, P, P]
        L.la_seg_dq_pass.restype = i32
        L.la_seg_dkv_pass.argtypes = [P, P, P, P, P, P, P, P, P, P, i32, i32, i64, i32, i32, i32,
                                      i32, i32, P, P, P, P, P]
        L.la_seg_dkv_pass.restype = i32
        L.la_seg_backward_parts.argtypes = [i32, i32, i64, i32, i32, i32, i32, i32, i32]
        L.la_seg_backward_parts.restype = i32
        L.la_seg_chain_pass.argtypes = [P, P, P, P, i32, i32, i64, i32, i32, i32, i32, i32, P, P,
                                        P, P, P, i32, P, P]
        L.la_seg_chain_pass.restype = i32
        L.la_seg_chain_reset.argtypes = [P, i32, i32, i32, i32, P, P, P]
        L.la_seg_chain_reset.restype = i32
        L.la_seg_check_status.argtypes = [P, P]
        L.la_seg_check_status.restype = i32
        L.la_last_error_detail.argtypes = [ctypes.c_char_p, sz]
        L.la_last_error_detail.restype = i32
        _lib = L
    return _lib


def la_last_error_detail() -> str:
    buf = ctypes.create_string_buffer(512)
    lib().la_last_error_detail(buf, 512)
    return buf.value.decode(errors="replace")


def _check(status: int, where: str):
    if status != LA_OK:
        raise LaSegError(status, where, la_last_error_detail())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return LA_F32
    if t.dtype == torch.bfloat16:
        return LA_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype=None, shape=None, device=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def la_seg_workspace_bytes(B, H, L, dk, dv, P, chunk, dt=LA_BF16, backward=False) -> int:
    return int(lib().la_seg_workspace_bytes(B, H, L, dk, dv, P, chunk, dt, int(bool(backward))))


def workspace(B, H, L, dk, dv, P, chunk, dt, backward=False, device="cuda"):
    """A caller-owned workspace of the size the library asks for (256-byte aligned)."""
    n = la_seg_workspace_bytes(B, H, L, dk, dv, P, chunk, dt, backward)
    if n == 0:
        raise LaSegError(-2, "la_seg_workspace_bytes", "sizes rejected by the library")
    return torch.empty(n, dtype=torch.uint8, device=device)


def la_seg_forward(q, k, v, log_g, S0=None, P=1, chunk=64, schedule=SCHED_AUTO, *, o=None,
                   want_S_final=True, want_S_recv=False, ws=None, stream=None):
    """o, S_final, S_recv = la_seg_forward(q, k, v, log_g, S0, P, chunk).

    q, k, log_g [B,H,L,dk], v [B,H,L,dv]: float32 or bfloat16 CUDA tensors of one dtype.
    S0: fp32 [B,H,dk,dv] or None.  S_final / S_recv (fp32 [B,H,dk,dv] / [B,H,P,dk,dv]) are
    None unless asked for.
    """
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    for t, n, shp in ((q, "q", (B, H, L, dk)), (k, "k", (B, H, L, dk)), (v, "v", (B, H, L, dv)),
                      (log_g, "log_g", (B, H, L, dk))):
        _need(t, n, q.dtype, shp, dev)
    _need(S0, "S0", torch.float32, (B, H, dk, dv), dev)
    dt = _dt(q)
    if o is None:
        o = torch.empty((B, H, L, dv), dtype=q.dtype, device=dev)
    _need(o, "o", q.dtype, (B, H, L, dv), dev)
    S_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev) if want_S_final else None
    S_recv = torch.empty((B, H, P, dk, dv), dtype=torch.float32, device=dev) if want_S_recv else None
    if ws is None:
        ws = workspace(B, H, L, dk, dv, P, chunk, dt, False, dev)
    st = lib().la_seg_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(log_g), _ptr(S0), B, H, L, dk, dv,
                              P, chunk, dt, _ptr(o), _ptr(S_final), _ptr(S_recv), int(schedule),
                              _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "la_seg_forward")
    return o, S_final, S_recv


def la_seg_backward(q, k, v, log_g, dO, S0=None, S_recv_saved=None, dS_final=None, P=1,
                    chunk=64, *, want_dS0=False, ws=None, stream=None):
    """dq, dk, dv, dlog_g, dS0 for loss = <o, dO> + <S_final, dS_final>."""
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    for t, n, shp in ((q, "q", (B, H, L, dk)), (k, "k", (B, H, L, dk)), (v, "v", (B, H, L, dv)),
                      (log_g, "log_g", (B, H, L, dk)), (dO, "dO", (B, H, L, dv))):
        _need(t, n, q.dtype, shp, dev)
    _need(S0, "S0", torch.float32, (B, H, dk, dv), dev)
    _need(S_recv_saved, "S_recv_saved", torch.float32, (B, H, P, dk, dv), dev)
    _need(dS_final, "dS_final", torch.float32, (B, H, dk, dv), dev)
    dt = _dt(q)
    dq = torch.empty_like(q)
    dk_ = torch.empty_like(k)
    dv_ = torch.empty_like(v)
    dg = torch.empty_like(log_g)
    dS0 = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev) if want_dS0 else None
    if ws is None:
        ws = workspace(B, H, L, dk, dv, P, chunk, dt, True, dev)
    st = lib().la_seg_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(log_g), _ptr(S0),
                               _ptr(S_recv_saved), _ptr(dO), _ptr(dS_final), B, H, L, dk, dv, P,
                               chunk, dt, _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(dg), _ptr(dS0),
                               _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "la_seg_backward")
    return dq, dk_, dv_, dg, dS0


def train_workspace(B, H, L, dk, dv, P, chunk, dt, backward=False, device="cuda"):
    n = int(lib().la_seg_train_workspace_bytes(B, H, L, dk, dv, P, chunk, dt, int(bool(backward))))
    if n == 0:
        raise LaSegError(-2, "la_seg_train_workspace_bytes", "sizes rejected by the library")
    return torch.empty(n, dtype=torch.uint8, device=device)


def la_seg_train_forward(q, k, v, log_g, S0=None, P=1, chunk=64, schedule=SCHED_AUTO, *, o=None,
                         ws=None, stream=None):
    """o, S_final, saved: the forward of a P-segment caller that will run the backward, with the
    received states saved at the library's own split (saved: fp32 [B, H, NS, dk, dv])."""
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    for t, n, shp in ((q, "q", (B, H, L, dk)), (k, "k", (B, H, L, dk)), (v, "v", (B, H, L, dv)),
                      (log_g, "log_g", (B, H, L, dk))):
        _need(t, n, q.dtype, shp, dev)
    _need(S0, "S0", torch.float32, (B, H, dk, dv), dev)
    dt = _dt(q)
    NS = int(lib().la_seg_train_saved_states(B, H, L, dk, dv, P, chunk, dt))
    if NS == 0:
        raise LaSegError(-2, "la_seg_train_saved_states", "sizes rejected by the library")
    o = torch.empty((B, H, L, dv), dtype=q.dtype, device=dev) if o is None else o
    S_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    saved = torch.empty((B, H, NS, dk, dv), dtype=torch.float32, device=dev)
    ws = train_workspace(B, H, L, dk, dv, P, chunk, dt, False, dev) if ws is None else ws
    _check(lib().la_seg_train_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(log_g), _ptr(S0), B, H, L,
                                      dk, dv, P, chunk, dt, _ptr(o), _ptr(S_final), _ptr(saved),
                                      int(schedule), _ptr(ws), ws.numel(), _stream(stream)),
           "la_seg_train_forward")
    return o, S_final, saved


def la_seg_train_backward(q, k, v, log_g, dO, saved, S0=None, dS_final=None, P=1, chunk=64, *,
                          want_dS0=False, ws=None, stream=None):
    """dq, dk, dv, dlog_g, dS0 reusing la_seg_train_forward's saved states."""
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    dt = _dt(q)
    NS = int(lib().la_seg_train_saved_states(B, H, L, dk, dv, P, chunk, dt))
    _need(saved, "saved", torch.float32, (B, H, NS, dk, dv), dev)
    _need(S0, "S0", torch.float32, (B, H, dk, dv), dev)
    _need(dS_final, "dS_final", torch.float32, (B, H, dk, dv), dev)
    dq, dk_, dv_, dg = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                        torch.empty_like(log_g))
    dS0 = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev) if want_dS0 else None
    ws = train_workspace(B, H, L, dk, dv, P, chunk, dt, True, dev) if ws is None else ws
    _check(lib().la_seg_train_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(log_g), _ptr(S0),
                                       _ptr(saved), _ptr(dO), _ptr(dS_final), B, H, L, dk, dv, P,
                                       chunk, dt, _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(dg),
                                       _ptr(dS0), _ptr(ws), ws.numel(), _stream(stream)),
           "la_seg_train_backward")
    return dq, dk_, dv_, dg, dS0


def la_seg_scan(S_in, log_gamma, init=None, reverse=False, *, want_final=True, S_next=None,
                S_last=None, out=None, final=None, carry=None, status=None, stream=None):
    """out, final = exclusive decayed scan over dim 1 of S_in [BH, NP, dk, dv] (fp32).

    With S_next (and optionally S_last) a carry tensor fp32 [BH, NP, dk] is filled too (given,
    or allocated and returned as a third value): the dlog_g carries of la_seg_dkv_pass."""
    BH, NP, dk, dv = S_in.shape
    dev = S_in.device
    _need(S_in, "S_in", torch.float32, None, dev)
    _need(log_gamma, "log_gamma", torch.float32, (BH, NP, dk), dev)
    _need(init, "init", torch.float32, (BH, dk, dv), dev)
    _need(S_next, "S_next", torch.float32, (BH, NP, dk, dv), dev)
    _need(S_last, "S_last", torch.float32, (BH, dk, dv), dev)
    out = torch.empty_like(S_in) if out is None else out
    if final is None and want_final:
        final = torch.empty((BH, dk, dv), dtype=torch.float32, device=dev)
    want_carry = S_next is not None
    if want_carry and carry is None:
        carry = torch.empty((BH, NP, dk), dtype=torch.float32, device=dev)
    st = lib().la_seg_scan(_ptr(S_in), _ptr(log_gamma), _ptr(init), BH, NP, dk, dv,
                           int(bool(reverse)), _ptr(out), _ptr(final), _ptr(S_next),
                           _ptr(S_last), _ptr(carry if want_carry else None), _ptr(status),
                           _stream(stream))
    _check(st, "la_seg_scan")
    return (out, final, carry) if want_carry else (out, final)


def la_seg_check_status(ws, stream=None):
    """Synchronise and raise LaSegError if a kernel flagged a device-side condition."""
    _check(lib().la_seg_check_status(_ptr(ws), _stream(stream)), "la_seg_check_status")


# ---- the steps of the path (see la_seg.h) ----------------------------------------------
def la_seg_subsegments(B, H, L, dk, dv, P, chunk, dt=LA_BF16) -> int:
    """Segments per (b, h) that la_seg_forward runs its passes over (P times the split)."""
    return int(lib().la_seg_subsegments(B, H, L, dk, dv, P, chunk, dt))


def _seq_shapes(q_or_k, v=None):
    B, H, L, dk = q_or_k.shape
    dv = v.shape[-1] if v is not None else dk
    return B, H, L, dk, dv


def la_seg_state_pass(k, v, log_g, NP, chunk, *, S_loc=None, log_gamma=None, status=None,
                      stream=None):
    B, H, L, dk, dv = _seq_shapes(k, v)
    dev = k.device
    S_loc = torch.empty((B, H, NP, dk, dv), dtype=torch.float32, device=dev) if S_loc is None else S_loc
    log_gamma = (torch.empty((B, H, NP, dk), dtype=torch.float32, device=dev)
                 if log_gamma is None else log_gamma)
    _check(lib().la_seg_state_pass(_ptr(k), _ptr(v), _ptr(log_g), B, H, L, dk, dv, NP, chunk,
                                   _dt(k), _ptr(S_loc), _ptr(log_gamma), _ptr(status),
                                   _stream(stream)), "la_seg_state_pass")
    return S_loc, log_gamma


def la_seg_local_pass(q, k, v, log_g, NP, chunk, *, o=None, S_loc=None, log_gamma=None,
                      want_states=True, status=None, stream=None):
    """Segment-local outputs; with want_states=False the local states are not written (and
    S_loc, log_gamma come back as None)."""
    B, H, L, dk, dv = _seq_shapes(q, v)
    dev = q.device
    o = torch.empty((B, H, L, dv), dtype=q.dtype, device=dev) if o is None else o
    if want_states:
        S_loc = (torch.empty((B, H, NP, dk, dv), dtype=torch.float32, device=dev)
                 if S_loc is None else S_loc)
        log_gamma = (torch.empty((B, H, NP, dk), dtype=torch.float32, device=dev)
                     if log_gamma is None else log_gamma)
    else:
        S_loc = log_gamma = None
    _check(lib().la_seg_local_pass(_ptr(q), _ptr(k), _ptr(v), _ptr(log_g), B, H, L, dk, dv, NP,
                                   chunk, _dt(q), _ptr(o), _ptr(S_loc), _ptr(log_gamma),
                                   _ptr(status), _stream(stream)), "la_seg_local_pass")
    return o, S_loc, log_gamma


def la_seg_output_pass(q, k, v, log_g, S_recv, NP, chunk, *, o=None, status=None, stream=None):
    B, H, L, dk, dv = _seq_shapes(q, v)
    o = torch.empty((B, H, L, dv), dtype=q.dtype, device=q.device) if o is None else o
    _check(lib().la_seg_output_pass(_ptr(q), _ptr(k), _ptr(v), _ptr(log_g), _ptr(S_recv), B, H, L,
                                    dk, dv, NP, chunk, _dt(q), _ptr(o), _ptr(status),
                                    _stream(stream)), "la_seg_output_pass")
    return o


def la_seg_correct_pass(q, log_g, S_recv, NP, chunk, o, *, status=None, stream=None):
    B, H, L, dk, dv = _seq_shapes(q, o)
    _check(lib().la_seg_correct_pass(_ptr(q), _ptr(log_g), _ptr(S_recv), B, H, L, dk, dv, NP,
                                     chunk, _dt(q), _ptr(o), _ptr(status), _stream(stream)),
           "la_seg_correct_pass")
    return o


def la_seg_dstate_pass(q, dO, log_g, NP, chunk, *, dSloc=None, log_gamma=None, status=None,
                       stream=None):
    B, H, L, dk, dv = _seq_shapes(q, dO)
    dev = q.device
    dSloc = torch.empty((B, H, NP, dk, dv), dtype=torch.float32, device=dev) if dSloc is None else dSloc
    log_gamma = (torch.empty((B, H, NP, dk), dtype=torch.float32, device=dev)
                 if log_gamma is None else log_gamma)
    _check(lib().la_seg_dstate_pass(_ptr(q), _ptr(dO), _ptr(log_g), B, H, L, dk, dv, NP, chunk,
                                    _dt(q), _ptr(dSloc), _ptr(log_gamma), _ptr(status),
                                    _stream(stream)), "la_seg_dstate_pass")
    return dSloc, log_gamma


def la_seg_backward_parts(B, H, L, dk, dv, P, chunk, dt=LA_BF16, reuse=True) -> int:
    return int(lib().la_seg_backward_parts(B, H, L, dk, dv, P, chunk, dt, int(bool(reuse))))


def la_seg_dq_pass(q, k, v, log_g, dO, S_recv, NP, fine, chunk, *, dq=None, qdq=None, S_fine=None,
                   dSloc=None, log_gamma=None, status=None, stream=None):
    """dq and q . dq; optionally (dSloc and log_gamma given, both or neither) the fine parts'
    gradient states and log-decay sums, as la_seg_dstate_pass over NP * fine parts.  q . dq is
    a buffer of B*H*L*dk floats for la_seg_dkv_pass in the library's internal arrangement (see
    la_seg.h), not a [B, H, L, dk] tensor in general."""
    B, H, L, dk, dv = _seq_shapes(q, v)
    dq = torch.empty_like(q) if dq is None else dq
    qdq = torch.empty((B, H, L, dk), dtype=torch.float32, device=q.device) if qdq is None else qdq
    _check(lib().la_seg_dq_pass(_ptr(q), _ptr(k), _ptr(v), _ptr(log_g), _ptr(dO), _ptr(S_recv), B,
                                H, L, dk, dv, NP, fine, chunk, _dt(q), _ptr(dq), _ptr(qdq),
                                _ptr(S_fine), _ptr(dSloc), _ptr(log_gamma), _ptr(status),
                                _stream(stream)), "la_seg_dq_pass")
    return dq, qdq


def la_seg_dkv_pass(q, k, v, log_g, dO, S_recv, S_final, dX, qdq, NP, chunk, *, carry=None,
                    out=None, status=None, stream=None):
    B, H, L, dk, dv = _seq_shapes(q, v)
    if out is None:
        out = (torch.empty_like(k), torch.empty_like(v), torch.empty_like(log_g))
    dk_, dv_, dg = out
    _check(lib().la_seg_dkv_pass(_ptr(q), _ptr(k), _ptr(v), _ptr(log_g), _ptr(dO), _ptr(S_recv),
                                 _ptr(S_final), _ptr(dX), _ptr(qdq), _ptr(carry), B, H, L, dk, dv,
                                 NP, chunk,
                                 _dt(q), _ptr(dk_), _ptr(dv_), _ptr(dg), _ptr(status),
                                 _stream(stream)), "la_seg_dkv_pass")
    return out


def la_seg_gather_states(src, m, *, dst=None, stream=None):
    """dst[:, :, p] = src[:, :, p * m]: the states at API-segment boundaries (src fp32
    [B, H, NP, dk, dv], dst [B, H, NP / m, dk, dv])."""
    B, H, NP, dk, dv = src.shape
    _need(src, "src", torch.float32, None, src.device)
    dst = torch.empty((B, H, NP // m, dk, dv), dtype=torch.float32, device=src.device) if dst is None else dst
    _need(dst, "dst", torch.float32, (B, H, NP // m, dk, dv), src.device)
    _check(lib().la_seg_gather_states(_ptr(src), B * H, NP, m, dk, dv, _ptr(dst), _stream(stream)),
           "la_seg_gather_states")
    return dst


def la_seg_log_gamma_total(log_gamma, *, out=None, stream=None):
    """Sum over the segment axis: fp32 [..., NP, dk] -> [..., dk]."""
    *lead, NP, dk = log_gamma.shape
    BH = 1
    for x in lead:
        BH *= x
    _need(log_gamma, "log_gamma", torch.float32, None, log_gamma.device)
    out = torch.empty((*lead, dk), dtype=torch.float32, device=log_gamma.device) if out is None else out
    _check(lib().la_seg_log_gamma_total(_ptr(log_gamma), BH, NP, dk, _ptr(out), _stream(stream)),
           "la_seg_log_gamma_total")
    return out


def la_seg_rank_scan(S_ranks, log_gamma_ranks, rank, init=None, reverse=False, *, S_in=None,
                     total=None, want_total=True, stream=None):
    """S_in (and the total) of the exclusive scan across ranks: S_ranks fp32 [N, *lead, dk, dv],
    log_gamma_ranks fp32 [N, *lead, dk] in rank order."""
    N = S_ranks.shape[0]
    dk, dv = S_ranks.shape[-2:]
    lead = S_ranks.shape[1:-2]
    BH = 1
    for x in lead:
        BH *= x
    dev = S_ranks.device
    _need(S_ranks, "S_ranks", torch.float32, None, dev)
    _need(log_gamma_ranks, "log_gamma_ranks", torch.float32, (N, *lead, dk), dev)
    _need(init, "init", torch.float32, (*lead, dk, dv), dev)
    S_in = torch.empty((*lead, dk, dv), dtype=torch.float32, device=dev) if S_in is None else S_in
    if want_total and total is None:
        total = torch.empty((*lead, dk, dv), dtype=torch.float32, device=dev)
    _check(lib().la_seg_rank_scan(_ptr(S_ranks), _ptr(log_gamma_ranks), _ptr(init), N, BH, dk, dv,
                                  int(rank), int(bool(reverse)), _ptr(S_in),
                                  _ptr(total if want_total else None), _stream(stream)),
           "la_seg_rank_scan")
    return S_in, (total if want_total else None)


def la_seg_combine(lg_a, S_a, lg_b, S_b, *, lg_out=None, S_out=None, stream=None):
    """(lg_a, S_a) followed by (lg_b, S_b): (lg_a + lg_b, exp(lg_b) S_a + S_b)."""
    dk, dv = S_a.shape[-2:]
    BH = S_a.numel() // (dk * dv)
    dev = S_a.device
    for t, n in ((lg_a, "lg_a"), (S_a, "S_a"), (lg_b, "lg_b"), (S_b, "S_b")):
        _need(t, n, torch.float32, None, dev)
    lg_out = torch.empty_like(lg_a) if lg_out is None else lg_out
    S_out = torch.empty_like(S_a) if S_out is None else S_out
    _check(lib().la_seg_combine(_ptr(lg_a), _ptr(S_a), _ptr(lg_b), _ptr(S_b), BH, dk, dv,
                                _ptr(lg_out), _ptr(S_out), _stream(stream)), "la_seg_combine")
    return lg_out, S_out


def chain_buffers(B, H, dk, dv, device="cuda"):
    """Caller-owned chain buffers of la_seg_chain_pass: fp32 [B*H, 2, dk, dv] state slots and
    int32 [B*H + 1] ready words (the last one the ticket counter)."""
    states = torch.empty((B * H, 2, dk, dv), dtype=torch.float32, device=device)
    ready = torch.empty((B * H + 1,), dtype=torch.int32, device=device)
    return states, ready


def la_seg_chain_reset(S0, B, H, dk, dv, states, ready, *, stream=None):
    """Slot 0 of every sequence's chain = S0 (None: zeros); ready words and ticket = 0."""
    _need(S0, "S0", torch.float32, (B, H, dk, dv), states.device)
    _check(lib().la_seg_chain_reset(_ptr(S0), B, H, dk, dv, _ptr(states), _ptr(ready),
                                    _stream(stream)), "la_seg_chain_reset")


def la_seg_chain_pass(q, k, v, log_g, NP, chunk, states, ready, *, o=None, S_final=None,
                      S_recv_save=None, save_every=1, status=None, stream=None):
    """One-kernel forward over NP sub-segments per (b, h) with the scan chained between them
    (la_seg.h); states / ready as la_seg_chain_reset left them.  Returns o."""
    B, H, L, dk, dv = _seq_shapes(q, v)
    dev = q.device
    for t, n, shp in ((q, "q", (B, H, L, dk)), (k, "k", (B, H, L, dk)), (v, "v", (B, H, L, dv)),
                      (log_g, "log_g", (B, H, L, dk))):
        _need(t, n, q.dtype, shp, dev)
    _need(states, "states", torch.float32, (B * H, 2, dk, dv), dev)
    _need(ready, "ready", torch.int32, (B * H + 1,), dev)
    o = torch.empty((B, H, L, dv), dtype=q.dtype, device=dev) if o is None else o
    _check(lib().la_seg_chain_pass(_ptr(q), _ptr(k), _ptr(v), _ptr(log_g), B, H, L, dk, dv, NP,
                                   chunk, _dt(q), _ptr(states), _ptr(ready), _ptr(o),
                                   _ptr(S_final), _ptr(S_recv_save), int(save_every),
                                   _ptr(status), _stream(stream)), "la_seg_chain_pass")
    return o
