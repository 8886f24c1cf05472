"""The layer around the operator on the GPU: the gate-activation kernels (gdn2_layer_gates_fwd / _bwd) against
the fp64 layer oracle's activations, and the whole layer (cuBLAS projections, the library's gate kernels and
operator, autograd) against the oracle layer, forward and backward.

Tolerances (relative L2). Gate kernels: fp32 arithmetic, outputs rounded once to the dtype, so bf16 <= 4e-3
(2^-9 per value) and fp32 <= 1e-5. Layer (bf16): the operator's 2e-2 (outputs) / 3e-2 (gradients) plus one
bf16 rounding of each projection's output: y, S_T <= 3e-2, gradients <= 4e-2.
"""
import numpy as np
import pytest
import torch

from conftest import rel_l2
from linear_attention_delta_gdn_b200 import binding
from linear_attention_delta_gdn_b200.inputs import to_f64

pytestmark = pytest.mark.gpu

OUTS = ("q", "k", "v", "b", "w", "log_alpha")


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_attention_delta_gdn_b200 import build
    build.build()


@pytest.mark.parametrize("dtype,Dk,Dv,bias", [(torch.bfloat16, 128, 128, True), (torch.bfloat16, 64, 128, False),
                                              (torch.bfloat16, 16, 16, True), (torch.float32, 32, 32, True)])
def test_gate_kernels_against_oracle(dtype, Dk, Dv, bias):
    from oracle import layer as L
    g = torch.Generator().manual_seed(Dk + Dv)
    B, T, H = 2, 77, 3
    z = (torch.randn((B, T, H, 4 * Dk + 2 * Dv), generator=g) * 2).to(dtype)
    a_bias = (torch.randn((H, Dk), generator=g) - 3) if bias else None
    grads = {n: torch.randn((B, T, H, Dv if n in ("v", "w") else Dk), generator=g).to(dtype) for n in OUTS}
    zd = z.cuda()
    bd = a_bias.cuda() if bias else None
    outs = binding.gdn2_layer_gates_fwd(zd, Dk, Dv, bd)
    dz = binding.gdn2_layer_gates_bwd(zd, *(grads[n].cuda() for n in OUTS), Dk, Dv, bd)
    torch.cuda.synchronize()
    tol = 4e-3 if dtype == torch.bfloat16 else 1e-5
    ref = L.gates(to_f64(z), Dk, Dv, None if a_bias is None else a_bias.double().numpy())
    for n, t in zip(OUTS, outs):
        assert rel_l2(to_f64(t), ref[n]) <= tol, (n, rel_l2(to_f64(t), ref[n]))
    dz_ref = L.gates_bwd(to_f64(z), {n: to_f64(t) for n, t in grads.items()}, Dk, Dv,
                         None if a_bias is None else a_bias.double().numpy())
    assert rel_l2(to_f64(dz), dz_ref) <= tol, rel_l2(to_f64(dz), dz_ref)


@pytest.mark.parametrize("T,with_S0", [(300, True), (64, False)])
def test_layer_against_oracle(T, with_S0):
    from oracle import layer as L
    from linear_attention_delta_gdn_b200.layer import Gdn2Layer
    torch.manual_seed(7)
    B, H, Dm = 2, 2, 256
    layer = Gdn2Layer(Dm, H, device="cuda")
    with torch.no_grad():   # a spread of resting decays
        layer.a_bias.copy_(torch.linspace(-6, 0, H * 128, device="cuda").view(H, 128))
    g = torch.Generator().manual_seed(T)
    x = torch.randn((B, T, Dm), generator=g).to(torch.bfloat16).cuda().requires_grad_(True)
    S0 = (torch.randn((B, H, 128, 128), generator=g) * 0.02).cuda().requires_grad_(True) if with_S0 else None
    dy = torch.randn((B, T, Dm), generator=g).to(torch.bfloat16).cuda()
    dST = torch.randn((B, H, 128, 128), generator=g).cuda()
    y, ST = layer(x, S0)
    ((y.float() * dy.float()).sum() + (ST * dST).sum()).backward()
    assert binding.gdn2_device_status() == binding.GDN2_OK, binding.last_error()
    args = (to_f64(x), to_f64(layer.W_in), to_f64(layer.W_out), H, 128, 128)
    bias = to_f64(layer.a_bias)
    S0n = to_f64(S0) if with_S0 else None
    y_ref, ST_ref = L.layer_fwd(*args, bias, S0n)
    gr = L.layer_bwd(*args, to_f64(dy), bias, S0n, to_f64(dST))
    assert rel_l2(to_f64(y), y_ref) <= 3e-2, rel_l2(to_f64(y), y_ref)
    assert rel_l2(to_f64(ST), ST_ref) <= 3e-2
    got = {"dx": x.grad, "dW_in": layer.W_in.grad, "dW_out": layer.W_out.grad, "da_bias": layer.a_bias.grad}
    if with_S0:
        got["dS0"] = S0.grad
    for n, t in got.items():
        v = to_f64(t)
        assert np.all(np.isfinite(v)), n
        assert rel_l2(v, gr[n]) <= 4e-2, (n, rel_l2(v, gr[n]))
