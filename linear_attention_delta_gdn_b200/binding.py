"""ctypes binding of libgdn2.so (the C ABI declared in include/gdn2.h).

Argument marshalling only: every step of the operator runs in the library's
CUDA kernels. torch supplies device memory (outputs and the workspace are
allocated as torch tensors) and the current CUDA stream. There is no CPU or
library fallback: if ``libgdn2.so`` is missing or a tensor is not on a CUDA
device, these functions raise.

Names mirror the C entry points: :func:`gdn2_fwd`, :func:`gdn2_bwd`,
:func:`gdn2_decode_step`, :func:`gdn2_workspace_size`.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_DEBUG_BUILD = os.environ.get("GDN2_DEBUG", "") not in ("", "0")
#: the library this process loads: the debug build (index checks, see build.py) when GDN2_DEBUG is set
_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                         "libgdn2_debug.so" if _DEBUG_BUILD else "libgdn2.so")
_lib = None

GDN2_F32, GDN2_BF16 = 0, 1
GDN2_OP_FWD, GDN2_OP_FWD_SAVE, GDN2_OP_BWD, GDN2_OP_MAP = 0, 1, 2, 3
GDN2_OK, GDN2_ERR_INVALID, GDN2_ERR_TIMEOUT = 0, 1, 5
GDN2_ERR_UNSUPPORTED = 2
STATUS = {0: "GDN2_OK", 1: "GDN2_ERR_INVALID", 2: "GDN2_ERR_UNSUPPORTED", 3: "GDN2_ERR_WORKSPACE",
          4: "GDN2_ERR_CUDA", 5: "GDN2_ERR_TIMEOUT"}

#: exported symbols, as declared in include/gdn2.h
EXPORTS = ("gdn2_workspace_size", "gdn2_fwd", "gdn2_bwd", "gdn2_decode_step", "gdn2_status_string",
           "gdn2_last_error", "gdn2_version", "gdn2_bwd_no_alloc", "gdn2_no_alloc_scratch_bytes",
           "gdn2_trace_enable", "gdn2_trace_read", "gdn2_device_status", "gdn2_beta_workspace_size",
           "gdn2_beta_fwd", "gdn2_beta_bwd", "gdn2_varlen_workspace_size", "gdn2_varlen_fwd", "gdn2_varlen_bwd",
           "gdn2_fwd_map", "gdn2_bwd_map", "gdn2_state_affine", "gdn2_layer_gates_fwd", "gdn2_layer_gates_bwd")
GDN2_GATE_KDA, GDN2_GATE_GDN = 1, 2


class Gdn2Error(RuntimeError):
    def __init__(self, fn, status, detail):
        super().__init__("%s -> %s: %s" % (fn, STATUS.get(status, status), detail))
        self.status = status


def lib(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libgdn2.so (built by ``python -m linear_attention_delta_gdn_b200.build``)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or _LIB_PATH
    if not os.path.exists(p):
        raise FileNotFoundError("%s is missing: build it with `python -m linear_attention_delta_gdn_b200.build`" % p)
    L = ctypes.CDLL(p)
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.gdn2_workspace_size.argtypes = [I] * 8
    L.gdn2_workspace_size.restype = Z
    L.gdn2_fwd.argtypes = [P] * 9 + [I] * 8 + [P, Z, P]
    L.gdn2_fwd.restype = I
    L.gdn2_bwd.argtypes = [P] * 16 + [I] * 8 + [P, Z, P]
    L.gdn2_bwd.restype = I
    L.gdn2_decode_step.argtypes = [P] * 8 + [I] * 5 + [P]
    L.gdn2_decode_step.restype = I
    L.gdn2_status_string.argtypes = [I]
    L.gdn2_status_string.restype = ctypes.c_char_p
    L.gdn2_last_error.argtypes = []
    L.gdn2_last_error.restype = ctypes.c_char_p
    L.gdn2_version.argtypes = []
    L.gdn2_version.restype = I
    L.gdn2_bwd_no_alloc.argtypes = [P] * 16 + [I] * 7 + [P]
    L.gdn2_bwd_no_alloc.restype = I
    L.gdn2_no_alloc_scratch_bytes.argtypes = []
    L.gdn2_no_alloc_scratch_bytes.restype = Z
    L.gdn2_beta_workspace_size.argtypes = [I] * 9
    L.gdn2_beta_workspace_size.restype = Z
    L.gdn2_beta_fwd.argtypes = [I] + [P] * 8 + [I] * 8 + [P, Z, P]
    L.gdn2_beta_fwd.restype = I
    L.gdn2_beta_bwd.argtypes = [I] + [P] * 14 + [I] * 8 + [P, Z, P]
    L.gdn2_beta_bwd.restype = I
    LL = ctypes.c_longlong
    L.gdn2_varlen_workspace_size.argtypes = [I] * 8
    L.gdn2_varlen_workspace_size.restype = Z
    L.gdn2_varlen_fwd.argtypes = [P] * 7 + [I, I, LL] + [P] * 3 + [I] * 6 + [P, Z, P]
    L.gdn2_varlen_fwd.restype = I
    L.gdn2_varlen_bwd.argtypes = [P] * 7 + [I, I, LL] + [P] * 10 + [I] * 6 + [P, Z, P]
    L.gdn2_varlen_bwd.restype = I
    L.gdn2_fwd_map.argtypes = [P] * 8 + [I] * 7 + [P, Z, P]
    L.gdn2_fwd_map.restype = I
    L.gdn2_bwd_map.argtypes = [P] * 9 + [I] * 7 + [P, Z, P]
    L.gdn2_bwd_map.restype = I
    L.gdn2_state_affine.argtypes = [P] * 4 + [I] * 4 + [P]
    L.gdn2_state_affine.restype = I
    L.gdn2_layer_gates_fwd.argtypes = [P] * 8 + [I] * 6 + [P]
    L.gdn2_layer_gates_fwd.restype = I
    L.gdn2_layer_gates_bwd.argtypes = [P] * 9 + [I] * 6 + [P]
    L.gdn2_layer_gates_bwd.restype = I
    L.gdn2_device_status.argtypes = [P]
    L.gdn2_device_status.restype = I
    L.gdn2_trace_enable.argtypes = [I]
    L.gdn2_trace_enable.restype = None
    L.gdn2_trace_read.argtypes = [ctypes.c_char_p, Z, P, P, I]
    L.gdn2_trace_read.restype = I
    if path is None:
        _lib = L
    return L


def _check(fn, rc):
    if rc != 0:
        raise Gdn2Error(fn, rc, lib().gdn2_last_error().decode(errors="replace"))


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN2_BF16
    if t.dtype == torch.float32:
        return GDN2_F32
    raise TypeError("dtype %s is not supported (float32 or bfloat16)" % t.dtype)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _state(t, like, B, H, Dk, Dv):
    if t is None:
        return None
    if t.dtype != torch.float32 or tuple(t.shape) != (B, H, Dk, Dv):
        raise ValueError("states must be float32 [B, H, Dk, Dv] = %s" % ((B, H, Dk, Dv),))
    return t


def gdn2_workspace_size(op: int, B: int, T: int, H: int, Dk: int, Dv: int, chunk: int, dt: int) -> int:
    return int(lib().gdn2_workspace_size(op, B, T, H, Dk, Dv, chunk, dt))


def gdn2_fwd(q, k, v, log_alpha, b, w, S0=None, chunk: int = 64, want_state: bool = True,
             save_states: bool = False, ws: Optional[torch.Tensor] = None, o=None, ST=None):
    """Forward. Tensors [B, T, H, D] (bf16 or fp32), S0 [B, H, Dk, Dv] fp32 or None.

    Returns ``(o, ST)`` (``ST`` is None unless ``want_state``). ``ws`` is a uint8
    CUDA tensor of at least ``gdn2_workspace_size(GDN2_OP_FWD[_SAVE], ...)`` bytes,
    allocated if not given. With ``save_states`` the chunk-start states are kept in
    it for a later :func:`gdn2_bwd` with ``states_saved=True``.
    """
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = _dt(q)
    for name, t, D in (("k", k, Dk), ("v", v, Dv), ("log_alpha", log_alpha, Dk), ("b", b, Dk), ("w", w, Dv)):
        if t.dtype != q.dtype or tuple(t.shape) != (B, T, H, D):
            raise ValueError("%s must be %s [%d, %d, %d, %d]" % (name, q.dtype, B, T, H, D))
    _state(S0, q, B, H, Dk, Dv)
    if o is None:
        o = torch.empty((B, T, H, Dv), dtype=q.dtype, device=q.device)
    if ST is None and want_state:
        ST = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=q.device)
    ws_bytes = 0
    need = gdn2_workspace_size(GDN2_OP_FWD_SAVE if save_states else GDN2_OP_FWD, B, T, H, Dk, Dv, chunk, dt)
    if need and ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    if ws is not None:
        ws_bytes = ws.numel()
    rc = lib().gdn2_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(S0), _ptr(o),
                        _ptr(ST), B, T, H, Dk, Dv, chunk, dt, int(save_states), _ptr(ws), ws_bytes,
                        _stream(q.device))
    _check("gdn2_fwd", rc)
    return o, ST


def gdn2_bwd(q, k, v, log_alpha, b, w, dout, S0=None, dST=None, chunk: int = 64, want_dS0: bool = True,
             states_saved: bool = False, ws: Optional[torch.Tensor] = None, grads=None):
    """Gate-aware backward for L = <dout, o> + <dST, S_T>.

    Returns a dict with dq, dk, dv, dlog_alpha, db, dw (input dtype) and dS0 (fp32 or None).
    """
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = _dt(q)
    _state(S0, q, B, H, Dk, Dv)
    _state(dST, q, B, H, Dk, Dv)
    if tuple(dout.shape) != (B, T, H, Dv) or dout.dtype != q.dtype:
        raise ValueError("dout must be %s [%d, %d, %d, %d]" % (q.dtype, B, T, H, Dv))
    if grads is None:
        grads = {n: torch.empty_like(q) for n in ("dq", "dk", "dlog_alpha", "db")}
        grads.update({n: torch.empty_like(v) for n in ("dv", "dw")})
        grads["dS0"] = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=q.device) if want_dS0 else None
    need = gdn2_workspace_size(GDN2_OP_BWD, B, T, H, Dk, Dv, chunk, dt)
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    g = grads
    rc = lib().gdn2_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(S0), _ptr(dout),
                        _ptr(dST), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dlog_alpha"]),
                        _ptr(g["db"]), _ptr(g["dw"]), _ptr(g.get("dS0")), B, T, H, Dk, Dv, chunk, dt,
                        int(states_saved), _ptr(ws), ws.numel(), _stream(q.device))
    _check("gdn2_bwd", rc)
    return grads


def _map_ws(q, v, chunk, ws):
    B, T, H, Dk = q.shape
    need = gdn2_workspace_size(GDN2_OP_MAP, B, T, H, Dk, v.shape[-1], chunk, _dt(q))
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    return ws


def gdn2_fwd_map(q, k, v, log_alpha, b, w, chunk: int = 64, ws: Optional[torch.Tensor] = None):
    """Affine map of a sequence piece, ``S_end = M S_start + N``: returns ``(M, N)``, fp32
    ``[B, H, Dk, Dk]`` and ``[B, H, Dk, Dv]``."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    M = torch.empty((B, H, Dk, Dk), dtype=torch.float32, device=q.device)
    N = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=q.device)
    ws = _map_ws(q, v, chunk, ws)
    rc = lib().gdn2_fwd_map(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(M), _ptr(N),
                            B, T, H, Dk, Dv, chunk, _dt(q), _ptr(ws), ws.numel(), _stream(q.device))
    _check("gdn2_fwd_map", rc)
    return M, N


def gdn2_bwd_map(q, k, v, log_alpha, b, w, dout, chunk: int = 64, ws: Optional[torch.Tensor] = None):
    """Reverse affine map of a sequence piece, ``dS_start = A dS_end + B``: returns ``(A, B)``."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    A = torch.empty((B, H, Dk, Dk), dtype=torch.float32, device=q.device)
    Bm = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=q.device)
    ws = _map_ws(q, v, chunk, ws)
    rc = lib().gdn2_bwd_map(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(dout), _ptr(A),
                            _ptr(Bm), B, T, H, Dk, Dv, chunk, _dt(q), _ptr(ws), ws.numel(), _stream(q.device))
    _check("gdn2_bwd_map", rc)
    return A, Bm


def gdn2_state_affine(M, N, S_in, out=None):
    """``M S_in + N`` per (batch, head) in fp32 (``N`` or ``S_in`` may be None: zero)."""
    B, H, Dk, _ = M.shape
    ref = N if N is not None else S_in
    Dv = ref.shape[-1] if ref is not None else Dk
    if out is None:
        out = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=M.device)
    rc = lib().gdn2_state_affine(_ptr(M), _ptr(N), _ptr(S_in), _ptr(out), B, H, Dk, Dv, _stream(M.device))
    _check("gdn2_state_affine", rc)
    return out


def gdn2_layer_gates_fwd(z, Dk: int, Dv: int, a_bias=None):
    """Operator inputs from the layer's pre-activations ``z [B, T, H, 4 Dk + 2 Dv]``: returns
    ``(q, k, v, b, w, log_alpha)`` in z's dtype (``a_bias``: fp32 [H, Dk] decay bias or None)."""
    B, T, H, W = z.shape
    if W != 4 * Dk + 2 * Dv:
        raise ValueError("z must be [B, T, H, 4 Dk + 2 Dv]")
    if a_bias is not None and (a_bias.dtype != torch.float32 or tuple(a_bias.shape) != (H, Dk)):
        raise ValueError("a_bias must be float32 [H, Dk]")
    mk = lambda D: torch.empty((B, T, H, D), dtype=z.dtype, device=z.device)
    q, k, v, b, w, la = mk(Dk), mk(Dk), mk(Dv), mk(Dk), mk(Dv), mk(Dk)
    rc = lib().gdn2_layer_gates_fwd(_ptr(z), _ptr(a_bias), _ptr(q), _ptr(k), _ptr(v), _ptr(b), _ptr(w), _ptr(la),
                                    B, T, H, Dk, Dv, _dt(z), _stream(z.device))
    _check("gdn2_layer_gates_fwd", rc)
    return q, k, v, b, w, la


def gdn2_layer_gates_bwd(z, dq, dk, dv, db, dw, dlog_alpha, Dk: int, Dv: int, a_bias=None):
    """dz (z's layout) from z and the gradients of the six operator inputs."""
    B, T, H, _ = z.shape
    dz = torch.empty_like(z)
    rc = lib().gdn2_layer_gates_bwd(_ptr(z), _ptr(a_bias), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(db), _ptr(dw),
                                    _ptr(dlog_alpha), _ptr(dz), B, T, H, Dk, Dv, _dt(z), _stream(z.device))
    _check("gdn2_layer_gates_bwd", rc)
    return dz


def gdn2_beta_workspace_size(gate: int, op: int, B: int, T: int, H: int, Dk: int, Dv: int, chunk: int,
                             dt: int) -> int:
    return int(lib().gdn2_beta_workspace_size(gate, op, B, T, H, Dk, Dv, chunk, dt))


def gdn2_beta_fwd(gate, q, k, v, log_alpha, beta, S0=None, chunk: int = 64, want_state: bool = True,
                  save_states: bool = False, ws: Optional[torch.Tensor] = None, o=None, ST=None):
    """KDA (gate=GDN2_GATE_KDA, log_alpha [B,T,H,Dk]) or Gated DeltaNet (GDN2_GATE_GDN, log_alpha [B,T,H])
    forward through the Gated Delta Rule-2 kernels; beta [B,T,H]. Returns ``(o, ST)``."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = _dt(q)
    la_shape = (B, T, H, Dk) if gate == GDN2_GATE_KDA else (B, T, H)
    for name, t, shp in (("k", k, (B, T, H, Dk)), ("v", v, (B, T, H, Dv)), ("log_alpha", log_alpha, la_shape),
                         ("beta", beta, (B, T, H))):
        if t.dtype != q.dtype or tuple(t.shape) != shp:
            raise ValueError("%s must be %s %s" % (name, q.dtype, shp))
    _state(S0, q, B, H, Dk, Dv)
    if o is None:
        o = torch.empty((B, T, H, Dv), dtype=q.dtype, device=q.device)
    if ST is None and want_state:
        ST = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=q.device)
    op = GDN2_OP_FWD_SAVE if save_states else GDN2_OP_FWD
    need = gdn2_beta_workspace_size(gate, op, B, T, H, Dk, Dv, chunk, dt)
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    rc = lib().gdn2_beta_fwd(gate, _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(o),
                             _ptr(ST), B, T, H, Dk, Dv, chunk, dt, int(save_states), _ptr(ws), ws.numel(),
                             _stream(q.device))
    _check("gdn2_beta_fwd", rc)
    return o, ST


def gdn2_beta_bwd(gate, q, k, v, log_alpha, beta, dout, S0=None, dST=None, chunk: int = 64, want_dS0: bool = True,
                  states_saved: bool = False, ws: Optional[torch.Tensor] = None, grads=None):
    """Backward of :func:`gdn2_beta_fwd`: dict with dq, dk, dv, dlog_alpha (shape of log_alpha), dbeta
    [B,T,H] and dS0."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = _dt(q)
    _state(S0, q, B, H, Dk, Dv)
    _state(dST, q, B, H, Dk, Dv)
    if grads is None:
        grads = {"dq": torch.empty_like(q), "dk": torch.empty_like(q), "dv": torch.empty_like(v),
                 "dlog_alpha": torch.empty_like(log_alpha), "dbeta": torch.empty_like(beta),
                 "dS0": torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=q.device) if want_dS0 else None}
    need = gdn2_beta_workspace_size(gate, GDN2_OP_BWD, B, T, H, Dk, Dv, chunk, dt)
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    g = grads
    rc = lib().gdn2_beta_bwd(gate, _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(dout),
                             _ptr(dST), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dlog_alpha"]),
                             _ptr(g["dbeta"]), _ptr(g.get("dS0")), B, T, H, Dk, Dv, chunk, dt, int(states_saved),
                             _ptr(ws), ws.numel(), _stream(q.device))
    _check("gdn2_beta_bwd", rc)
    return grads


def gdn2_varlen_workspace_size(op: int, N: int, Tmax: int, H: int, Dk: int, Dv: int, chunk: int, dt: int) -> int:
    return int(lib().gdn2_varlen_workspace_size(op, N, Tmax, H, Dk, Dv, chunk, dt))


def gdn2_varlen_fwd(q, k, v, log_alpha, b, w, cu_seqlens, Tmax: int, S0=None, chunk: int = 64,
                    want_state: bool = True, save_states: bool = False, ws: Optional[torch.Tensor] = None):
    """Packed sequences: tensors [Ttot, H, D], cu_seqlens int32 [N + 1] on the device, Tmax >= every length.
    Returns ``(o [Ttot, H, Dv], ST [N, H, Dk, Dv] or None)``."""
    Ttot, H, Dk = q.shape
    Dv = v.shape[-1]
    N = cu_seqlens.numel() - 1
    dt = _dt(q)
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda:
        raise ValueError("cu_seqlens must be an int32 CUDA tensor")
    _state(S0, q, N, H, Dk, Dv)
    o = torch.empty((Ttot, H, Dv), dtype=q.dtype, device=q.device)
    ST = torch.empty((N, H, Dk, Dv), dtype=torch.float32, device=q.device) if want_state else None
    need = gdn2_varlen_workspace_size(GDN2_OP_FWD_SAVE if save_states else GDN2_OP_FWD, N, Tmax, H, Dk, Dv, chunk, dt)
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    rc = lib().gdn2_varlen_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(cu_seqlens), N,
                               Tmax, Ttot, _ptr(S0), _ptr(o), _ptr(ST), H, Dk, Dv, chunk, dt, int(save_states),
                               _ptr(ws), ws.numel(), _stream(q.device))
    _check("gdn2_varlen_fwd", rc)
    return o, ST


def gdn2_varlen_bwd(q, k, v, log_alpha, b, w, dout, cu_seqlens, Tmax: int, S0=None, dST=None, chunk: int = 64,
                    want_dS0: bool = True, states_saved: bool = False, ws: Optional[torch.Tensor] = None):
    """Backward of :func:`gdn2_varlen_fwd`: dict of packed dq, dk, dv, dlog_alpha, db, dw and dS0 [N, ...]."""
    Ttot, H, Dk = q.shape
    Dv = v.shape[-1]
    N = cu_seqlens.numel() - 1
    dt = _dt(q)
    _state(S0, q, N, H, Dk, Dv)
    _state(dST, q, N, H, Dk, Dv)
    g = {n: torch.empty_like(q) for n in ("dq", "dk", "dlog_alpha", "db")}
    g.update({n: torch.empty_like(v) for n in ("dv", "dw")})
    g["dS0"] = torch.empty((N, H, Dk, Dv), dtype=torch.float32, device=q.device) if want_dS0 else None
    need = gdn2_varlen_workspace_size(GDN2_OP_BWD, N, Tmax, H, Dk, Dv, chunk, dt)
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    rc = lib().gdn2_varlen_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(cu_seqlens), N,
                               Tmax, Ttot, _ptr(S0), _ptr(dout), _ptr(dST), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]),
                               _ptr(g["dlog_alpha"]), _ptr(g["db"]), _ptr(g["dw"]), _ptr(g["dS0"]), H, Dk, Dv, chunk,
                               dt, int(states_saved), _ptr(ws), ws.numel(), _stream(q.device))
    _check("gdn2_varlen_bwd", rc)
    return g


def gdn2_decode_step(q, k, v, log_alpha, b, w, S, o=None):
    """One decode step: inputs [B, H, D]; S [B, H, Dk, Dv] fp32 is updated in place. Returns o."""
    B, H, Dk = q.shape
    Dv = v.shape[-1]
    _state(S, q, B, H, Dk, Dv)
    if o is None:
        o = torch.empty((B, H, Dv), dtype=q.dtype, device=q.device)
    rc = lib().gdn2_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(S), _ptr(o),
                                B, H, Dk, Dv, _dt(q), _stream(q.device))
    _check("gdn2_decode_step", rc)
    return o


def gdn2_device_status(device=None) -> int:
    """Synchronise the current stream and return the device-side status of the tensor-core kernels
    (0, or GDN2_ERR_TIMEOUT if a bounded wait inside them gave up since the previous call; the record is
    cleared). The detail is in :func:`last_error`."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return int(lib().gdn2_device_status(_stream(dev)))


def last_error() -> str:
    return lib().gdn2_last_error().decode()


def trace_enable(on: bool = True) -> None:
    """Start (or stop) per-kernel event timing of the library's launches."""
    lib().gdn2_trace_enable(1 if on else 0)


def trace_read() -> dict:
    """{kernel name: (launches, summed device ms)} since the last read (waits for the events)."""
    n_max = 16
    names = ctypes.create_string_buffer(1024)
    launches = (ctypes.c_int * n_max)()
    ms = (ctypes.c_double * n_max)()
    n = lib().gdn2_trace_read(names, 1024, ctypes.cast(launches, ctypes.c_void_p), ctypes.cast(ms, ctypes.c_void_p), n_max)
    keys = names.value.decode().split(",") if n else []
    return {k: (int(launches[i]), float(ms[i])) for i, k in enumerate(keys)}


class GatedDeltaRule2(torch.autograd.Function):
    """autograd wrapper: forward keeps the chunk-start states for the backward."""

    @staticmethod
    def forward(ctx, q, k, v, log_alpha, b, w, S0, chunk):
        B, T, H, Dk = q.shape
        Dv = v.shape[-1]
        need = gdn2_workspace_size(GDN2_OP_BWD, B, T, H, Dk, Dv, chunk, _dt(q))
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
        o, ST = gdn2_fwd(q, k, v, log_alpha, b, w, S0, chunk=chunk, save_states=True, ws=ws)
        ctx.save_for_backward(q, k, v, log_alpha, b, w, S0, ws)
        ctx.chunk = chunk
        return o, ST

    @staticmethod
    def backward(ctx, do, dST):
        q, k, v, log_alpha, b, w, S0, ws = ctx.saved_tensors
        g = gdn2_bwd(q, k, v, log_alpha, b, w, do.contiguous(), S0,
                     None if dST is None else dST.contiguous(), chunk=ctx.chunk,
                     want_dS0=S0 is not None, states_saved=True, ws=ws)
        return g["dq"], g["dk"], g["dv"], g["dlog_alpha"], g["db"], g["dw"], g["dS0"], None


def gated_delta_rule2(q, k, v, log_alpha, b, w, S0=None, chunk: int = 64):
    """Differentiable Gated Delta Rule-2 operator. Returns ``(o, S_T)``."""
    return GatedDeltaRule2.apply(q, k, v, log_alpha, b, w, S0, chunk)
