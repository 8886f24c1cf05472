"""fp64 chunkwise (WY) restatement of the Gated Delta Rule-2 operator -- TEST INFRASTRUCTURE.

"Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention" names, in its
arXiv abstract and GitHub README ("Hardware-efficient Training" bullet), a
chunkwise WY algorithm in which the channel-wise decay is absorbed into
asymmetric erase factors, and a gate-aware backward. The pages print neither.
This module writes that chunk algebra out, as derived below, in plain numpy
fp64, so that tests can pin it to the token oracle (``oracle.fwd``/``bwd``) at
several chunk sizes. It is a model of the algebra the CUDA kernels implement,
not the oracle of record, and it shares no code with them.

Derivation, per head and per chunk of L <= C tokens starting from state S:
  G_t = sum_{tau<=t in chunk} log_alpha_tau (inclusive),  g_t = exp(G_t),  gC = g_{L-1}
  E = b*k,  U = w*v
  Et = g*E (erase factor scaled forward),  Kt = k/g (key scaled backward),
  Qt = g*q,  Kh = (gC/g)*k
  Writing S_t = D_t S_{t-1} + k_t delta_t^T with delta_t = u_t - (D_t S_{t-1})^T e_t
  and unrolling inside the chunk gives (I + A) Delta = U - Et S with
  A = strictly_lower(Et Kt^T). With T = (I + A)^{-1}:
    Delta = T U - (T Et) S = Ut - Wm S
    O     = Qt S + tril(Qt Kt^T) Delta          (read-out after the update: inclusive mask)
    S'    = Diag(gC) S + Kh^T Delta
"""
from __future__ import annotations

import numpy as np


def _heads(x):
    """[B, T, H, D] -> [B, H, T, D] float64 copy."""
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64).transpose(0, 2, 1, 3))


def _mT(x):
    return np.swapaxes(x, -1, -2)


def _chunk_factors(q, k, v, la, b, w):
    """Per-chunk factors for [B, H, L, D] slices."""
    L = q.shape[-2]
    G = np.cumsum(la, axis=-2)
    g = np.exp(G)
    gC = g[..., L - 1, :]
    E = b * k
    U = w * v
    Et = g * E
    Kt = k / g
    Qt = g * q
    Kh = (gC[..., None, :] / g) * k
    strict = np.tril(np.ones((L, L)), -1)
    incl = np.tril(np.ones((L, L)), 0)
    A = (Et @ _mT(Kt)) * strict
    Tm = np.linalg.inv(np.eye(L) + A)
    P = (Qt @ _mT(Kt)) * incl
    return dict(G=G, g=g, gC=gC, E=E, U=U, Et=Et, Kt=Kt, Qt=Qt, Kh=Kh, A=A, Tm=Tm, P=P,
                Wm=Tm @ Et, Ut=Tm @ U, strict=strict, incl=incl)


def fwd(q, k, v, log_alpha, b, w, S0=None, chunk=64, return_states=False):
    """Chunkwise forward. Returns ``(o [B,T,H,Dv], ST)`` (and the list of chunk-start states)."""
    q, k, v, la, b, w = map(_heads, (q, k, v, log_alpha, b, w))
    Bn, H, T, Dk = q.shape
    Dv = v.shape[-1]
    S = np.zeros((Bn, H, Dk, Dv)) if S0 is None else np.array(S0, dtype=np.float64)
    o = np.zeros((Bn, H, T, Dv))
    states = []
    for t0 in range(0, T, chunk):
        t1 = min(t0 + chunk, T)
        f = _chunk_factors(q[..., t0:t1, :], k[..., t0:t1, :], v[..., t0:t1, :],
                           la[..., t0:t1, :], b[..., t0:t1, :], w[..., t0:t1, :])
        Delta = f["Ut"] - f["Wm"] @ S
        o[..., t0:t1, :] = f["Qt"] @ S + f["P"] @ Delta
        states.append(S.copy())
        S = f["gC"][..., :, None] * S + _mT(f["Kh"]) @ Delta
    o = np.ascontiguousarray(o.transpose(0, 2, 1, 3))
    if return_states:
        return o, S, states
    return o, S


def bwd(q, k, v, log_alpha, b, w, dout, S0=None, dST=None, chunk=64):
    """Chunkwise gate-aware backward of :func:`fwd` for ``L = <dout, o> + <dST, ST>``.

    Per chunk, going backwards with dS' = dL/dS_{next}:
      dDelta = Kh dS' + P^T dO
      dS     = Diag(gC) dS' + Qt^T dO - Wm^T dDelta
      dQt    = dO S^T + dP Kt,  dP = (dO Delta^T) * incl
      dKh    = Delta dS'^T,     dgC = rowsum(dS' * S)
      dUt    = dDelta,          dWm = -dDelta S^T
      dTm    = dUt U^T + dWm Et^T ;  dU = Tm^T dUt ;  dEt = Tm^T dWm + dA Kt
      dA     = -(Tm^T dTm Tm^T) * strict ;  dKt = dP^T Qt + dA^T Et
    then the gate chain through g = exp(cumsum(log_alpha)):
      dG = Qt*dQt + Et*dEt - Kt*dKt - Kh*dKh ;  dG[last] += sum_t Kh*dKh + gC*dgC
      dlog_alpha = reverse in-chunk cumsum of dG
      dq = g*dQt ; dE = g*dEt ; db = dE*k ; dk = dKt/g + (gC/g)*dKh + dE*b
      dw = dU*v ; dv = dU*w
    """
    q_, k_, v_, la_, b_, w_, do_ = map(_heads, (q, k, v, log_alpha, b, w, dout))
    Bn, H, T, Dk = q_.shape
    Dv = v_.shape[-1]
    _, _, states = fwd(q, k, v, log_alpha, b, w, S0=S0, chunk=chunk, return_states=True)
    dS = np.zeros((Bn, H, Dk, Dv)) if dST is None else np.array(dST, dtype=np.float64)
    out = {n: np.zeros((Bn, H, T, Dk)) for n in ("dq", "dk", "dlog_alpha", "db")}
    out.update({n: np.zeros((Bn, H, T, Dv)) for n in ("dv", "dw")})
    starts = list(range(0, T, chunk))
    for ci in reversed(range(len(starts))):
        t0 = starts[ci]
        t1 = min(t0 + chunk, T)
        sl = slice(t0, t1)
        qc, kc, vc, lac, bc, wc, dO = (x[..., sl, :] for x in (q_, k_, v_, la_, b_, w_, do_))
        f = _chunk_factors(qc, kc, vc, lac, bc, wc)
        S = states[ci]
        dSn = dS
        Delta = f["Ut"] - f["Wm"] @ S
        dDelta = f["Kh"] @ dSn + _mT(f["P"]) @ dO
        dS = f["gC"][..., :, None] * dSn + _mT(f["Qt"]) @ dO - _mT(f["Wm"]) @ dDelta
        dP = (dO @ _mT(Delta)) * f["incl"]
        dQt = dO @ _mT(S) + dP @ f["Kt"]
        dKt = _mT(dP) @ f["Qt"]
        dKh = Delta @ _mT(dSn)
        dgC = np.sum(dSn * S, axis=-1)
        dUt = dDelta
        dWm = -dDelta @ _mT(S)
        dTm = dUt @ _mT(f["U"]) + dWm @ _mT(f["Et"])
        dU = _mT(f["Tm"]) @ dUt
        dA = -(_mT(f["Tm"]) @ dTm @ _mT(f["Tm"])) * f["strict"]
        dEt = _mT(f["Tm"]) @ dWm + dA @ f["Kt"]
        dKt = dKt + _mT(dA) @ f["Et"]
        g, gC = f["g"], f["gC"]
        dG = f["Qt"] * dQt + f["Et"] * dEt - f["Kt"] * dKt - f["Kh"] * dKh
        dG[..., -1, :] += np.sum(f["Kh"] * dKh, axis=-2) + gC * dgC
        out["dlog_alpha"][..., sl, :] = np.flip(np.cumsum(np.flip(dG, -2), axis=-2), -2)
        dE = g * dEt
        out["dq"][..., sl, :] = g * dQt
        out["db"][..., sl, :] = dE * kc
        out["dk"][..., sl, :] = dKt / g + (gC[..., None, :] / g) * dKh + dE * bc
        out["dw"][..., sl, :] = dU * vc
        out["dv"][..., sl, :] = dU * wc
    res = {n: np.ascontiguousarray(x.transpose(0, 2, 1, 3)) for n, x in out.items()}
    res["dS0"] = dS
    return res
