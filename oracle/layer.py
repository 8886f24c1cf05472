"""Gated DeltaNet-2 layer around the operator, in fp64 numpy (test infrastructure only).

The pages name the layer's two per-channel gate computations (erase gate b_t in [0,1]^{d_k}, write gate
w_t in [0,1]^{d_v}: GitHub README method bullets; the aiexpert.news article puts the overhead over KDA on
them) and KDA's channel-wise decay, but print no parameterisation. This file writes out the plainest
reading, the same one the CUDA gate kernels take:

    z = x W_in                       (per token; per head the columns [z_q | z_k | z_v | z_b | z_w | z_a])
    q = z_q / sqrt(|z_q|^2 + eps),  k = z_k / sqrt(|z_k|^2 + eps),  v = z_v
    b = sigmoid(z_b),  w = sigmoid(z_w),  log_alpha = -softplus(z_a + a_bias)
    o, S_T = the Gated Delta Rule-2 operator (oracle.fwd)
    y = o W_out                      (o flattened over heads)

Parity of the layer is pinned to this reading, not to the pages (which do not fix it): finite differences
pin the backward, closed forms pin the activations (tests/test_oracle_layer.py).
"""
from __future__ import annotations

import numpy as np

from . import bwd as op_bwd
from . import fwd as op_fwd

EPS = 1e-6


def _split(z, Dk, Dv):
    widths = (Dk, Dk, Dv, Dk, Dv, Dk)
    out, o = [], 0
    for wd in widths:
        out.append(z[..., o:o + wd])
        o += wd
    return out


def _sigmoid(x):
    return 0.5 * (1.0 + np.tanh(0.5 * x))


def _softplus(x):
    return np.logaddexp(0.0, x)


def gates(z, Dk, Dv, a_bias=None):
    """Operator inputs from the pre-activations z [B, T, H, 4 Dk + 2 Dv]."""
    z = np.asarray(z, dtype=np.float64)
    zq, zk, zv, zb, zw, za = _split(z, Dk, Dv)
    if a_bias is not None:
        za = za + np.asarray(a_bias, dtype=np.float64)
    return {
        "q": zq / np.sqrt((zq * zq).sum(-1, keepdims=True) + EPS),
        "k": zk / np.sqrt((zk * zk).sum(-1, keepdims=True) + EPS),
        "v": zv.copy(),
        "b": _sigmoid(zb),
        "w": _sigmoid(zw),
        "log_alpha": -_softplus(za),
    }


def gates_bwd(z, g, Dk, Dv, a_bias=None):
    """dz from the gradients g of the six operator inputs (keys q, k, v, b, w, log_alpha or dq, ...)."""
    z = np.asarray(z, dtype=np.float64)
    get = lambda n: np.asarray(g[n] if n in g else g["d" + n], dtype=np.float64)
    zq, zk, zv, zb, zw, za = _split(z, Dk, Dv)
    if a_bias is not None:
        za = za + np.asarray(a_bias, dtype=np.float64)
    parts = []
    for zz, gg in ((zq, get("q")), (zk, get("k"))):
        n = np.sqrt((zz * zz).sum(-1, keepdims=True) + EPS)
        u = zz / n
        parts.append((gg - u * (u * gg).sum(-1, keepdims=True)) / n)
    parts.append(get("v"))
    for zz, gg in ((zb, get("b")), (zw, get("w"))):
        s = _sigmoid(zz)
        parts.append(gg * s * (1.0 - s))
    parts.append(-get("log_alpha") * _sigmoid(za))
    return np.concatenate(parts, -1)


def layer_fwd(x, W_in, W_out, H, Dk, Dv, a_bias=None, S0=None):
    """y [B, T, Dm] and S_T [B, H, Dk, Dv] of the layer on x [B, T, Dm]."""
    x = np.asarray(x, dtype=np.float64)
    B, T, _ = x.shape
    z = (x @ np.asarray(W_in, dtype=np.float64)).reshape(B, T, H, 4 * Dk + 2 * Dv)
    gt = gates(z, Dk, Dv, a_bias)
    o, ST = op_fwd(gt["q"], gt["k"], gt["v"], gt["log_alpha"], gt["b"], gt["w"], S0=S0)
    y = o.reshape(B, T, H * Dv) @ np.asarray(W_out, dtype=np.float64)
    return y, ST


def layer_bwd(x, W_in, W_out, H, Dk, Dv, dy, a_bias=None, S0=None, dST=None):
    """Gradients of L = <dy, y> + <dST, S_T>: dict with dx, dW_in, dW_out, da_bias, dS0."""
    x = np.asarray(x, dtype=np.float64)
    W_in = np.asarray(W_in, dtype=np.float64)
    W_out = np.asarray(W_out, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    B, T, Dm = x.shape
    z = (x @ W_in).reshape(B, T, H, 4 * Dk + 2 * Dv)
    gt = gates(z, Dk, Dv, a_bias)
    o, _ = op_fwd(gt["q"], gt["k"], gt["v"], gt["log_alpha"], gt["b"], gt["w"], S0=S0)
    dW_out = o.reshape(B * T, H * Dv).T @ dy.reshape(B * T, Dm)
    do = (dy @ W_out.T).reshape(B, T, H, Dv)
    g = op_bwd(gt["q"], gt["k"], gt["v"], gt["log_alpha"], gt["b"], gt["w"], do, S0=S0, dST=dST)
    dz = gates_bwd(z, g, Dk, Dv, a_bias)
    dzf = dz.reshape(B * T, H * (4 * Dk + 2 * Dv))
    da = dz[..., 3 * Dk + 2 * Dv:].sum((0, 1))   # [H, Dk]
    return {"dx": (dzf @ W_in.T).reshape(B, T, Dm), "dW_in": x.reshape(B * T, Dm).T @ dzf, "dW_out": dW_out,
            "da_bias": da, "dS0": g["dS0"]}
