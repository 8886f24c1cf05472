"""Maps of sequence pieces (gdn2_fwd_map, gdn2_bwd_map, gdn2_state_affine) and a sequence cut into pieces
(context parallelism emulated in one process: the pieces run one after another on this GPU, the exchange is a
Python list) against the fp64 oracle. The oracle's maps are its own recurrence run from the identity without
input (M, A) and from a zero start (N, B). Tolerances as for the operator (relative L2): bf16 o, S_T and the
maps 2e-2, gradients 3e-2.
"""
import numpy as np
import pytest
import torch

from conftest import rel_l2, worst_head_rel_l2
from linear_attention_delta_gdn_b200 import binding
from linear_attention_delta_gdn_b200 import context_parallel as cp
from linear_attention_delta_gdn_b200.inputs import make_inputs, to_f64

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "log_alpha", "b", "w")
GRADS = ("dq", "dk", "dv", "dlog_alpha", "db", "dw")
TOL_OUT, TOL_GRAD = 2e-2, 3e-2


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_attention_delta_gdn_b200 import build
    build.build()


def _oracle_maps(oracle_mod, f):
    B, T, H, Dk = f["q"].shape
    z = np.zeros((B, T, H, Dk))
    eye = np.broadcast_to(np.eye(Dk), (B, H, Dk, Dk)).copy()
    _, M = oracle_mod.fwd(f["q"], f["k"], z, f["log_alpha"], f["b"], z, S0=eye)
    _, N = oracle_mod.fwd(*(f[n] for n in NAMES))
    A = oracle_mod.bwd(f["q"], f["k"], z, f["log_alpha"], f["b"], z, z, dST=eye)["dS0"]
    Bm = oracle_mod.bwd(*(f[n] for n in NAMES), f["dout"])["dS0"]
    return M, N, A, Bm


@pytest.mark.parametrize("B,T,H,decay", [(2, 700, 2, "recipe"), (2, 64, 2, "recipe"), (2, 1, 2, "recipe"),
                                         (2, 300, 2, "strong"), (1, 4100, 3, "slow")])
def test_maps_against_oracle(oracle_mod, B, T, H, decay):
    """The maps against the oracle's. The "slow" case is a 65-chunk piece with 3 heads, whose maps are computed
    over segments and composed; its decay is the recipe's / 100 so that M (a product of 4100 transitions) stays
    far from fp32 underflow."""
    x = make_inputs(B, T, H, 128, 128, seed=2100 + T, dtype="bf16", with_do=True)
    if decay == "strong":   # a few channels decay by e^-20 per token (exact pair terms on the tensor-core path)
        la = x["log_alpha"].float()
        la[..., [3, 64, 101]] = -20.0
        x["log_alpha"] = la.to(torch.bfloat16)
    elif decay == "slow":
        x["log_alpha"] = (x["log_alpha"].float() / 100.0).to(torch.bfloat16)
    d = {n: t.cuda() for n, t in x.items()}
    M, N = binding.gdn2_fwd_map(*(d[n] for n in NAMES))
    A, Bm = binding.gdn2_bwd_map(*(d[n] for n in NAMES), d["dout"])
    assert binding.gdn2_device_status() == binding.GDN2_OK, binding.last_error()
    f = {n: to_f64(t) for n, t in x.items()}
    ref = _oracle_maps(oracle_mod, f)
    for name, got, r in zip(("M", "N", "A", "B"), (M, N, A, Bm), ref):
        got = to_f64(got)
        assert np.all(np.isfinite(got)), name
        assert worst_head_rel_l2(got, r, state=True) <= TOL_OUT, (name, worst_head_rel_l2(got, r, state=True))
    # the reverse map is the forward map's transpose
    assert rel_l2(to_f64(A), to_f64(M.transpose(-1, -2))) <= TOL_OUT


def test_maps_of_an_empty_piece():
    q = torch.empty((1, 0, 3, 128), dtype=torch.bfloat16, device="cuda")
    v = torch.empty((1, 0, 3, 128), dtype=torch.bfloat16, device="cuda")
    M, N = binding.gdn2_fwd_map(q, q, v, q, q, v)
    A, Bm = binding.gdn2_bwd_map(q, q, v, q, q, v, v)
    eye = torch.eye(128, device="cuda").expand(1, 3, 128, 128)
    assert torch.equal(M, eye) and torch.equal(A, eye)
    assert not N.any() and not Bm.any()


def test_state_affine_in_place():
    g = torch.Generator(device="cuda").manual_seed(4)
    M = torch.randn((2, 3, 128, 128), generator=g, device="cuda")
    N = torch.randn((2, 3, 128, 128), generator=g, device="cuda")
    S = torch.randn((2, 3, 128, 128), generator=g, device="cuda")
    ref = (M.double() @ S.double() + N.double())
    out = binding.gdn2_state_affine(M, N, S, out=S)   # in place over S_in
    assert out.data_ptr() == S.data_ptr()
    assert rel_l2(to_f64(out), ref.cpu().numpy()) <= 1e-6
    out2 = binding.gdn2_state_affine(M, None, None)
    assert not out2.any()


@pytest.mark.parametrize("P,T,with_S0", [(4, 3000, True), (3, 1000, False), (2, 8192, True)])
def test_pieces_equal_the_whole_sequence(oracle_mod, P, T, with_S0):
    """The sequence cut into P pieces (ragged cuts inside chunks) gives the whole sequence's outputs, final
    state and gradients."""
    B, H = 1, 3
    x = make_inputs(B, T, H, 128, 128, seed=2200 + P, dtype="bf16", with_do=True, with_S0=with_S0)
    dST = torch.randn((B, H, 128, 128), generator=torch.Generator().manual_seed(9))
    d = {n: t.cuda() for n, t in x.items()}
    cuts = [0] + [(r * T) // P + 5 * r for r in range(1, P)] + [T]
    pieces = [tuple(d[n][:, cuts[r]:cuts[r + 1]].contiguous() for n in NAMES) for r in range(P)]
    douts = [d["dout"][:, cuts[r]:cuts[r + 1]].contiguous() for r in range(P)]
    S0 = d.get("S0")
    outs, starts, ST = cp.pieces_forward(pieces, S0)
    grads, dS0 = cp.pieces_backward(pieces, douts, starts, dST.cuda())
    assert binding.gdn2_device_status() == binding.GDN2_OK, binding.last_error()
    f = {n: to_f64(t) for n, t in x.items()}
    o_ref, ST_ref = oracle_mod.fwd(*(f[n] for n in NAMES), S0=f.get("S0"))
    gr = oracle_mod.bwd(*(f[n] for n in NAMES), f["dout"], S0=f.get("S0"), dST=dST.double().numpy())
    o = to_f64(torch.cat(outs, 1))
    assert worst_head_rel_l2(o, o_ref) <= TOL_OUT
    assert worst_head_rel_l2(to_f64(ST), ST_ref, state=True) <= TOL_OUT
    for n in GRADS:
        got = to_f64(torch.cat([g[n] for g in grads], 1))
        assert np.all(np.isfinite(got)), n
        assert worst_head_rel_l2(got, gr[n]) <= TOL_GRAD, (n, worst_head_rel_l2(got, gr[n]))
    assert worst_head_rel_l2(to_f64(dS0), gr["dS0"], state=True) <= TOL_GRAD
    # and the same as the uncut sequence through gdn2_fwd
    o_whole, _ = binding.gdn2_fwd(*(d[n] for n in NAMES), S0)
    assert rel_l2(o, to_f64(o_whole)) <= TOL_OUT
