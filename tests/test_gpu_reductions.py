"""KDA and Gated DeltaNet through the Gated Delta Rule-2 kernels (gdn2_beta_fwd / gdn2_beta_bwd), against the
fp64 oracle run with the broadcast gates b = w = beta * 1 (and, for Gated DeltaNet, log_alpha = log_a * 1).

The oracle's agreement with the two published recurrences is pinned on the CPU
(tests/test_oracle_pins.py::test_reduces_to_kda, ::test_reduces_to_gated_deltanet). Gradients of the reduced
gates follow from the chain rule through the broadcast: dbeta_t = sum_i db_ti + sum_j dw_tj and
dlog_a_t = sum_i dlog_alpha_ti. Tolerances as for the operator (relative L2, whole tensor and worst head):
fp32 1e-4; bf16 o, S_T 2e-2 and gradients 3e-2.
"""
import numpy as np
import pytest
import torch

from conftest import rel_l2, worst_head_rel_l2
from linear_attention_delta_gdn_b200 import binding
from linear_attention_delta_gdn_b200.inputs import make_inputs, make_reduced_gates, to_f64

pytestmark = pytest.mark.gpu

TOL_OUT = {"f32": 1e-4, "bf16": 2e-2}
TOL_GRAD = {"f32": 1e-4, "bf16": 3e-2}
GATES = {"kda": binding.GDN2_GATE_KDA, "gdn": binding.GDN2_GATE_GDN}


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_attention_delta_gdn_b200 import build
    build.build()


def _case(gate, B, T, H, Dk, Dv, dtype, seed):
    x = make_inputs(B, T, H, Dk, Dv, seed=seed, dtype=dtype, with_do=True, with_S0=True)
    r = make_reduced_gates(B, T, H, seed + 1, dtype)
    la = x["log_alpha"] if gate == "kda" else r["log_a"]
    return x, r["beta"], la


def _check(got, ref, tol, name, state=False):
    got = np.asarray(got)
    assert np.all(np.isfinite(got)), name
    e = rel_l2(got, ref)
    wh = worst_head_rel_l2(got, ref, state=state) if got.ndim == 4 else e
    assert e <= tol and wh <= tol, "%s: rel err %.3g (worst head %.3g) > %g" % (name, e, wh, tol)


def _worst_rows(got, ref):
    """[B, T, H] tensors: worst per-(b, h) relative error."""
    worst = 0.0
    for b in range(ref.shape[0]):
        for h in range(ref.shape[2]):
            worst = max(worst, rel_l2(got[b, :, h], ref[b, :, h]))
    return worst


@pytest.mark.parametrize("gate", ["kda", "gdn"])
@pytest.mark.parametrize("dtype,T,Dk,Dv,chunk,saved", [("bf16", 150, 128, 128, 64, True),
                                                       ("bf16", 300, 128, 128, 64, True),
                                                       ("bf16", 300, 128, 128, 64, False),
                                                       ("f32", 70, 64, 64, 32, True), ("f32", 70, 64, 64, 32, False),
                                                       ("bf16", 97, 64, 128, 64, True)])
def test_reduced_gates_against_oracle(oracle_mod, gate, dtype, T, Dk, Dv, chunk, saved):
    """saved: the backward runs on the forward's workspace (its saved states and broadcast gates); else on a
    workspace of its own, filled with 0xFF bytes first, so it must broadcast the gates itself."""
    B, H = 2, 3
    x, beta, la = _case(gate, B, T, H, Dk, Dv, dtype, seed=1200 + T + Dk)
    d = {n: t.cuda() for n, t in x.items()}
    dST = torch.randn((B, H, Dk, Dv), generator=torch.Generator().manual_seed(9))
    g_beta, g_la = beta.cuda(), la.cuda()
    ws = torch.empty(binding.gdn2_beta_workspace_size(GATES[gate], binding.GDN2_OP_BWD, B, T, H, Dk, Dv, chunk,
                                                      binding._dt(d["q"])), dtype=torch.uint8, device="cuda")
    o, ST = binding.gdn2_beta_fwd(GATES[gate], d["q"], d["k"], d["v"], g_la, g_beta, d["S0"], chunk=chunk,
                                  save_states=True, ws=ws)
    if not saved:
        ws = torch.full_like(ws, 255)
    g = binding.gdn2_beta_bwd(GATES[gate], d["q"], d["k"], d["v"], g_la, g_beta, d["dout"], d["S0"], dST.cuda(),
                              chunk=chunk, states_saved=saved, ws=ws)
    torch.cuda.synchronize()

    f = {n: to_f64(t) for n, t in x.items()}
    be, lae = to_f64(beta), to_f64(la)
    b_full = np.repeat(be[..., None], Dk, axis=-1)
    w_full = np.repeat(be[..., None], Dv, axis=-1)
    la_full = lae if gate == "kda" else np.repeat(lae[..., None], Dk, axis=-1)
    o_ref, ST_ref = oracle_mod.fwd(f["q"], f["k"], f["v"], la_full, b_full, w_full, S0=f["S0"])
    ref = oracle_mod.bwd(f["q"], f["k"], f["v"], la_full, b_full, w_full, dout=f["dout"], S0=f["S0"],
                         dST=dST.double().numpy())
    _check(to_f64(o), o_ref, TOL_OUT[dtype], "o")
    _check(to_f64(ST), ST_ref, TOL_OUT[dtype], "S_T", state=True)
    for n in ("dq", "dk", "dv"):
        _check(to_f64(g[n]), ref[n], TOL_GRAD[dtype], n)
    _check(to_f64(g["dS0"]), ref["dS0"], TOL_GRAD[dtype], "dS0", state=True)
    dbeta_ref = ref["db"].sum(-1) + ref["dw"].sum(-1)
    got = to_f64(g["dbeta"])
    assert rel_l2(got, dbeta_ref) <= TOL_GRAD[dtype] and _worst_rows(got, dbeta_ref) <= TOL_GRAD[dtype], \
        "dbeta %.3g" % rel_l2(got, dbeta_ref)
    if gate == "kda":
        _check(to_f64(g["dlog_alpha"]), ref["dlog_alpha"], TOL_GRAD[dtype], "dlog_alpha")
    else:
        dla_ref = ref["dlog_alpha"].sum(-1)
        got = to_f64(g["dlog_alpha"])
        assert rel_l2(got, dla_ref) <= TOL_GRAD[dtype] and _worst_rows(got, dla_ref) <= TOL_GRAD[dtype], \
            "dlog_a %.3g" % rel_l2(got, dla_ref)


@pytest.mark.parametrize("gate,B,T,H,strong", [("kda", 1, 4200, 2, False), ("gdn", 1, 4200, 2, False),
                                                ("kda", 2, 300, 2, True), ("gdn", 2, 300, 2, True)])
def test_reduced_gates_tensor_core_paths(oracle_mod, gate, B, T, H, strong):
    """The scalar-gate kernel instances on the tensor-core path where it branches: a long sequence with few heads
    (cut into segments) and strong decay: for KDA a few channels decaying by e^-20 per token, for Gated DeltaNet
    one head decaying by e^-20 per token over its second half (every channel of its chunks there takes the exact
    pair terms, which read b and the decay from the per-token gates); against the oracle, dbeta on every (b, h)."""
    D = 128
    x, beta, la = _case(gate, B, T, H, D, D, "bf16", seed=1300 + T)
    if strong:
        la = la.float()
        if gate == "kda":
            la[..., [5, 70, 127]] = -20.0
        else:
            la[:, T // 2:, 1] = -20.0
        la = la.to(torch.bfloat16)
    d = {n: t.cuda() for n, t in x.items()}
    g_beta, g_la = beta.cuda(), la.cuda()
    ws = torch.empty(binding.gdn2_beta_workspace_size(GATES[gate], binding.GDN2_OP_BWD, B, T, H, D, D, 64,
                                                      binding.GDN2_BF16), dtype=torch.uint8, device="cuda")
    o, ST = binding.gdn2_beta_fwd(GATES[gate], d["q"], d["k"], d["v"], g_la, g_beta, d["S0"], save_states=True, ws=ws)
    g = binding.gdn2_beta_bwd(GATES[gate], d["q"], d["k"], d["v"], g_la, g_beta, d["dout"], d["S0"], None,
                              states_saved=True, ws=ws)
    torch.cuda.synchronize()
    assert binding.gdn2_device_status() == binding.GDN2_OK, binding.last_error()
    f = {n: to_f64(t) for n, t in x.items()}
    be, lae = to_f64(beta), to_f64(la)
    b_full = np.repeat(be[..., None], D, axis=-1)
    la_full = lae if gate == "kda" else np.repeat(lae[..., None], D, axis=-1)
    o_ref, ST_ref = oracle_mod.fwd(f["q"], f["k"], f["v"], la_full, b_full, b_full, S0=f["S0"])
    ref = oracle_mod.bwd(f["q"], f["k"], f["v"], la_full, b_full, b_full, dout=f["dout"], S0=f["S0"])
    _check(to_f64(o), o_ref, TOL_OUT["bf16"], "o")
    _check(to_f64(ST), ST_ref, TOL_OUT["bf16"], "S_T", state=True)
    for n in ("dq", "dk", "dv"):
        _check(to_f64(g[n]), ref[n], TOL_GRAD["bf16"], n)
    dbeta_ref = ref["db"].sum(-1) + ref["dw"].sum(-1)
    got = to_f64(g["dbeta"])
    assert np.all(np.isfinite(got))
    assert rel_l2(got, dbeta_ref) <= TOL_GRAD["bf16"] and _worst_rows(got, dbeta_ref) <= TOL_GRAD["bf16"], \
        "dbeta %.3g (worst row %.3g)" % (rel_l2(got, dbeta_ref), _worst_rows(got, dbeta_ref))
    dla_ref = ref["dlog_alpha"] if gate == "kda" else ref["dlog_alpha"].sum(-1)
    got = to_f64(g["dlog_alpha"])
    if gate == "kda":
        _check(got, dla_ref, TOL_GRAD["bf16"], "dlog_alpha")
    else:
        assert rel_l2(got, dla_ref) <= TOL_GRAD["bf16"] and _worst_rows(got, dla_ref) <= TOL_GRAD["bf16"]


@pytest.mark.parametrize("gate", ["kda", "gdn"])
def test_unaligned_beta_takes_the_broadcast_path(gate):
    """The scalar-gate kernel instances read beta as 4-byte words; a beta that is only 2-byte aligned goes through
    the broadcast path instead, with the same results (to rounding: the gate sums run in another order)."""
    B, T, H, D = 2, 200, 2, 128
    x, beta, la = _case(gate, B, T, H, D, D, "bf16", seed=1400)
    d = {n: t.cuda() for n, t in x.items()}
    g_la = la.cuda()
    store = torch.empty(beta.numel() + 1, dtype=torch.bfloat16, device="cuda")
    shifted = store[1:].view(beta.shape)          # 2 bytes past a 256-byte boundary
    shifted.copy_(beta.cuda())
    aligned = beta.cuda()
    assert shifted.data_ptr() % 4 == 2 and aligned.data_ptr() % 4 == 0
    out = {}
    for name, bt in (("aligned", aligned), ("shifted", shifted)):
        ws = torch.empty(binding.gdn2_beta_workspace_size(GATES[gate], binding.GDN2_OP_BWD, B, T, H, D, D, 64,
                                                          binding.GDN2_BF16), dtype=torch.uint8, device="cuda")
        o, ST = binding.gdn2_beta_fwd(GATES[gate], d["q"], d["k"], d["v"], g_la, bt, d["S0"], save_states=True,
                                      ws=ws)
        g = binding.gdn2_beta_bwd(GATES[gate], d["q"], d["k"], d["v"], g_la, bt, d["dout"], d["S0"], None,
                                  states_saved=True, ws=ws)
        out[name] = {"o": o, "ST": ST, **g}
    torch.cuda.synchronize()
    assert binding.gdn2_device_status() == binding.GDN2_OK, binding.last_error()
    for n in ("o", "ST", "dq", "dk", "dv", "dbeta", "dlog_alpha", "dS0"):
        a_, b_ = to_f64(out["aligned"][n]), to_f64(out["shifted"][n])
        assert np.all(np.isfinite(b_)), n
        assert rel_l2(b_, a_) <= 1e-2, (n, rel_l2(b_, a_))


def test_reduced_gates_empty_sequence():
    B, T, H, D = 1, 0, 2, 128
    x = make_inputs(B, T, H, D, D, seed=5, dtype="bf16", with_do=True, with_S0=True)
    r = make_reduced_gates(B, T, H, 6, "bf16")
    d = {n: t.cuda() for n, t in x.items()}
    o, ST = binding.gdn2_beta_fwd(binding.GDN2_GATE_GDN, d["q"], d["k"], d["v"], r["log_a"].cuda(),
                                  r["beta"].cuda(), d["S0"])
    torch.cuda.synchronize()
    assert torch.equal(ST, d["S0"])
