"""Pins of the layer oracle (oracle/layer.py), CPU only: the activations' closed forms and segment layout,
the unit norm of q and k, and fp64 central finite differences of the gate backward and of the whole layer's
backward (every parameter, the input and S0). A swapped segment, a dropped bias, a sign slip in a
derivative or a transposed weight fails one of these."""
import numpy as np
import pytest

import oracle
from oracle import layer as L


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def test_gates_closed_forms_and_layout():
    Dk, Dv = 4, 6
    W = 4 * Dk + 2 * Dv
    z = np.zeros((1, 1, 2, W))
    g0 = L.gates(z, Dk, Dv)
    assert np.all(g0["q"] == 0) and np.all(g0["k"] == 0) and np.all(g0["v"] == 0)
    assert np.allclose(g0["b"], 0.5) and np.allclose(g0["w"], 0.5)
    assert np.allclose(g0["log_alpha"], -np.log(2.0))
    # each segment holds its own constant: the layout is [q | k | v | b | w | a]
    vals = [3.0, -2.0, 0.25, 1.0, 2.0, -1.5]
    widths = [Dk, Dk, Dv, Dk, Dv, Dk]
    z = np.concatenate([np.full((1, 1, 2, wd), c) for c, wd in zip(vals, widths)], -1)
    bias = np.array([[0.5] * Dk, [-0.5] * Dk])
    g = L.gates(z, Dk, Dv, bias)
    assert np.allclose(g["q"], 1 / np.sqrt(Dk + L.EPS / 9.0))          # 3 / sqrt(9 Dk + eps)
    assert np.allclose(g["k"], -1 / np.sqrt(Dk + L.EPS / 4.0))
    assert np.allclose(g["v"], 0.25)
    assert np.allclose(g["b"], 1 / (1 + np.exp(-1.0))) and np.allclose(g["w"], 1 / (1 + np.exp(-2.0)))
    assert np.allclose(g["log_alpha"][0, 0, 0], -np.log1p(np.exp(-1.0)))   # -softplus(-1.5 + 0.5)
    assert np.allclose(g["log_alpha"][0, 0, 1], -np.log1p(np.exp(-2.0)))   # -softplus(-1.5 - 0.5)


def test_q_k_have_unit_norm():
    z = _rng(1).standard_normal((2, 5, 3, 4 * 8 + 2 * 8))
    g = L.gates(z, 8, 8)
    for n in ("q", "k"):
        assert np.allclose(np.linalg.norm(g[n], axis=-1), 1.0, atol=1e-6)


def _fd(f, x, d, h=1e-6):
    return (f(x + h * d) - f(x - h * d)) / (2 * h)


def test_gates_backward_matches_finite_differences():
    rng = _rng(2)
    Dk, Dv = 8, 4
    z = rng.standard_normal((2, 3, 2, 4 * Dk + 2 * Dv))
    bias = rng.standard_normal((2, Dk))
    G = {n: rng.standard_normal(t.shape) for n, t in L.gates(z, Dk, Dv, bias).items()}
    loss = lambda zz: sum(float((L.gates(zz, Dk, Dv, bias)[n] * G[n]).sum()) for n in G)
    dz = L.gates_bwd(z, G, Dk, Dv, bias)
    for _ in range(4):
        d = rng.standard_normal(z.shape)
        assert _fd(loss, z, d) == pytest.approx(float((dz * d).sum()), rel=1e-7, abs=1e-9)


def test_layer_backward_matches_finite_differences():
    rng = _rng(3)
    B, T, H, Dk, Dv, Dm = 1, 7, 2, 4, 3, 5
    x = rng.standard_normal((B, T, Dm))
    W_in = rng.standard_normal((Dm, H * (4 * Dk + 2 * Dv))) * 0.5
    W_out = rng.standard_normal((H * Dv, Dm)) * 0.5
    bias = rng.standard_normal((H, Dk))
    S0 = rng.standard_normal((B, H, Dk, Dv)) * 0.3
    dy = rng.standard_normal((B, T, Dm))
    dST = rng.standard_normal((B, H, Dk, Dv))
    args = {"x": x, "W_in": W_in, "W_out": W_out, "a_bias": bias, "S0": S0}

    def loss(**kw):
        a = dict(args, **kw)
        y, ST = L.layer_fwd(a["x"], a["W_in"], a["W_out"], H, Dk, Dv, a["a_bias"], a["S0"])
        return float((y * dy).sum() + (ST * dST).sum())

    g = L.layer_bwd(x, W_in, W_out, H, Dk, Dv, dy, bias, S0, dST)
    names = {"x": "dx", "W_in": "dW_in", "W_out": "dW_out", "a_bias": "da_bias", "S0": "dS0"}
    for n, gn in names.items():
        for _ in range(2):
            d = rng.standard_normal(args[n].shape)
            fd = _fd(lambda v: loss(**{n: v}), args[n], d)
            assert fd == pytest.approx(float((g[gn] * d).sum()), rel=1e-6, abs=1e-8), n


def test_layer_with_identity_projection_is_the_operator():
    """With W_in that routes x straight into the pre-activations and W_out = I, the layer is the operator on
    the activated x (the composition adds nothing else)."""
    rng = _rng(4)
    B, T, H, Dk, Dv = 1, 9, 1, 4, 4
    Wd = 4 * Dk + 2 * Dv
    x = rng.standard_normal((B, T, Wd))
    W_out = np.eye(H * Dv)
    y, ST = L.layer_fwd(x, np.eye(Wd), W_out, H, Dk, Dv)
    g = L.gates(x.reshape(B, T, H, Wd), Dk, Dv)
    o, ST_ref = oracle.fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["b"], g["w"])
    assert np.allclose(y, o.reshape(B, T, H * Dv)) and np.allclose(ST, ST_ref)
