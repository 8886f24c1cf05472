"""fp64 CPU oracle of the Gated Delta Rule-2 operator -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (``libgdn2.so`` and its
Python binding) never imports, links or runs anything here, and the two share
no code.

Contents
  * ``gdn2_oracle.c`` -- the token-by-token recurrence (forward, reverse-mode
    backward, decode step) in plain fp64 C with OpenMP, built into
    ``libgdn2_oracle.so`` by :func:`build`. Source: "Gated DeltaNet-2:
    Decoupling Erase and Write in Linear Attention", GitHub README method
    bullets (erase gate on the key side of the decayed state, write gate on the
    value side, channel-wise decay) and the arXiv abstract (subtract the current
    read before writing; fixed-size state).
  * :mod:`oracle.chunkwise` -- an fp64 numpy restatement of the chunkwise WY
    form (forward and backward). It is not the oracle of record; tests pin it
    to the token oracle so that the chunk algebra used by the CUDA kernels is
    checked independently of them.

All functions take and return float64 numpy arrays. Token tensors are
``[B, T, H, D]``, decode tensors ``[B, H, D]``, states ``[B, H, Dk, Dv]``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn2_oracle.c")
_LIB = os.path.join(_HERE, "libgdn2_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``gdn2_oracle.c`` into ``libgdn2_oracle.so`` (gcc, -fopenmp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.gdn2_oracle_fwd.argtypes = [P] * 9 + [I] * 5
        lib.gdn2_oracle_fwd.restype = I
        lib.gdn2_oracle_bwd.argtypes = [P] * 16 + [I] * 5
        lib.gdn2_oracle_bwd.restype = I
        lib.gdn2_oracle_decode.argtypes = [P] * 8 + [I] * 4
        lib.gdn2_oracle_decode.restype = I
        lib.gdn2_oracle_threads.argtypes = []
        lib.gdn2_oracle_threads.restype = I
        _lib = lib
    return _lib


def _f64(x):
    if x is None:
        return None
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(x):
    return None if x is None else x.ctypes.data_as(ctypes.c_void_p)


def threads() -> int:
    """Number of OpenMP threads the oracle runs on."""
    return int(_load().gdn2_oracle_threads())


def fwd(q, k, v, log_alpha, b, w, S0=None):
    """Token recurrence forward. Returns ``(o [B,T,H,Dv], ST [B,H,Dk,Dv])``."""
    q, k, v, log_alpha, b, w, S0 = map(_f64, (q, k, v, log_alpha, b, w, S0))
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    o = np.zeros((B, T, H, Dv))
    ST = np.zeros((B, H, Dk, Dv))
    rc = _load().gdn2_oracle_fwd(*map(_ptr, (q, k, v, log_alpha, b, w, S0, o, ST)), B, T, H, Dk, Dv)
    if rc:
        raise RuntimeError("gdn2_oracle_fwd failed (%d)" % rc)
    return o, ST


def bwd(q, k, v, log_alpha, b, w, dout, S0=None, dST=None):
    """Adjoint of :func:`fwd` for ``L = <dout, o> + <dST, ST>``.

    Returns a dict with ``dq, dk, dv, dlog_alpha, db, dw, dS0``.
    """
    q, k, v, log_alpha, b, w, S0, dout, dST = map(_f64, (q, k, v, log_alpha, b, w, S0, dout, dST))
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    g = {n: np.zeros((B, T, H, Dk)) for n in ("dq", "dk", "dlog_alpha", "db")}
    g.update({n: np.zeros((B, T, H, Dv)) for n in ("dv", "dw")})
    g["dS0"] = np.zeros((B, H, Dk, Dv))
    rc = _load().gdn2_oracle_bwd(
        *map(_ptr, (q, k, v, log_alpha, b, w, S0, dout, dST, g["dq"], g["dk"], g["dv"],
                    g["dlog_alpha"], g["db"], g["dw"], g["dS0"])), B, T, H, Dk, Dv)
    if rc:
        raise RuntimeError("gdn2_oracle_bwd failed (%d)" % rc)
    return g


def decode(q, k, v, log_alpha, b, w, S):
    """One decode step. ``S`` is updated in a copy; returns ``(o [B,H,Dv], S_new)``."""
    q, k, v, log_alpha, b, w = map(_f64, (q, k, v, log_alpha, b, w))
    S = np.array(S, dtype=np.float64, copy=True, order="C")
    B, H, Dk = q.shape
    Dv = v.shape[-1]
    o = np.zeros((B, H, Dv))
    rc = _load().gdn2_oracle_decode(*map(_ptr, (q, k, v, log_alpha, b, w, S, o)), B, H, Dk, Dv)
    if rc:
        raise RuntimeError("gdn2_oracle_decode failed (%d)" % rc)
    return o, S
