"""ctypes front end of ``la_oracle.c`` (CPU, fp64, token-by-token) -- test infrastructure.

The C file holds the arithmetic; this module only compiles it with gcc, converts numpy /
torch inputs to contiguous float64 arrays and returns float64 arrays.  See the header of
``la_oracle.c`` for the recurrence and the passages of the ZeCO pages it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC_PATH = os.path.join(_HERE, "la_oracle.c")
LIB_PATH = os.path.join(_HERE, "liboracle.so")


def compile_lib(src: str, out: str) -> str:
    """gcc -O2 with OpenMP; no fast-math, so every double operation is IEEE."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                           src, "-o", tmp, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile la_oracle.c into oracle/liboracle.so if it is missing or stale."""
    if force or not os.path.exists(LIB_PATH) or os.path.getmtime(LIB_PATH) < os.path.getmtime(SRC_PATH):
        compile_lib(SRC_PATH, LIB_PATH)
    return LIB_PATH


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor -> exact float64 copy of the (already rounded) values
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """Bound copy of the oracle library at ``path`` (tests also bind deliberately broken
    copies of the source to show that the pins catch them)."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        lng = ctypes.c_long
        lib.la_oracle_forward.argtypes = [P, P, P, P, P, lng, lng, lng, lng, lng, lng, P, P, P]
        lib.la_oracle_forward.restype = None
        lib.la_oracle_backward.argtypes = [P, P, P, P, P, P, P, lng, lng, lng, lng, lng,
                                           P, P, P, P, P]
        lib.la_oracle_backward.restype = None
        lib.la_oracle_num_threads.argtypes = []
        lib.la_oracle_num_threads.restype = ctypes.c_int
        self.lib = lib

    def num_threads(self) -> int:
        return int(self.lib.la_oracle_num_threads())

    def forward(self, q, k, v, log_g, S0=None, seg_len: int | None = None):
        """Token-by-token GLA forward in fp64.

        q, k, log_g: [B, H, L, dk]; v: [B, H, L, dv]; S0: [B, H, dk, dv] or None (zeros).
        Returns (o [B,H,L,dv], S_final [B,H,dk,dv], S_seg [B,H,L/seg_len,dk,dv] or None),
        S_seg[..., p, :, :] being the state entering token p*seg_len (what segment p receives).
        """
        q, k, v, g, S0 = (_f64(t) for t in (q, k, v, log_g, S0))
        B, H, L, dk = q.shape
        dv = v.shape[-1]
        assert k.shape == q.shape == g.shape and v.shape == (B, H, L, dv)
        if S0 is not None:
            assert S0.shape == (B, H, dk, dv)
        o = np.zeros((B, H, L, dv))
        S_final = np.zeros((B, H, dk, dv))
        S_seg = None
        if seg_len:
            assert L % seg_len == 0
            S_seg = np.zeros((B, H, L // seg_len, dk, dv))
        self.lib.la_oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(S0), B, H, L, dk, dv,
                                   int(seg_len or 0), _ptr(o), _ptr(S_final), _ptr(S_seg))
        return o, S_final, S_seg

    def backward(self, q, k, v, log_g, dO, S0=None, dS_final=None):
        """Exact reverse-mode gradients of the fp64 forward (loss = <o, dO> + <S_final, dS_final>).

        Returns (dq, dk, dv, dlog_g, dS0) as float64 arrays of the input shapes.
        """
        q, k, v, g, dO, S0, dSf = (_f64(t) for t in (q, k, v, log_g, dO, S0, dS_final))
        B, H, L, dk = q.shape
        dv = v.shape[-1]
        assert dO.shape == (B, H, L, dv)
        dq, dk_, dv_, dg = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v), np.zeros_like(g)
        dS0 = np.zeros((B, H, dk, dv))
        self.lib.la_oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(S0), _ptr(dO),
                                    _ptr(dSf), B, H, L, dk, dv, _ptr(dq), _ptr(dk_), _ptr(dv_),
                                    _ptr(dg), _ptr(dS0))
        return dq, dk_, dv_, dg, dS0


_default: Oracle | None = None


def _oracle() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def num_threads() -> int:
    """OpenMP threads the oracle runs with (set OMP_NUM_THREADS before the first call)."""
    return _oracle().num_threads()


def forward(q, k, v, log_g, S0=None, seg_len=None):
    return _oracle().forward(q, k, v, log_g, S0, seg_len)


def backward(q, k, v, log_g, dO, S0=None, dS_final=None):
    return _oracle().backward(q, k, v, log_g, dO, S0, dS_final)


forward.__doc__ = Oracle.forward.__doc__
backward.__doc__ = Oracle.backward.__doc__
