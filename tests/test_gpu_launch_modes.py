"""The two launch forms of the tensor-core path give the same results.

The forward and the backward each run as one cooperative launch (per-head chain and per-chunk work
share the SMs and hand chunks over through ready flags) or, when the device cannot hold every CTA at
once or GDN2_NO_COOPERATIVE is set, as two ordinary launches. Every unit of work is computed the same
way in both forms, so the results must agree bit for bit; a problem with more heads than SMs must
agree with the same heads run in a small problem.
"""
import os

import pytest
import torch

from linear_attention_delta_gdn_b200 import binding
from linear_attention_delta_gdn_b200.inputs import make_inputs

NAMES = ("q", "k", "v", "log_alpha", "b", "w")
GRADS = ("dq", "dk", "dv", "dlog_alpha", "db", "dw", "dS0")


def _run(d, dST):
    B, T, H, _ = d["q"].shape
    need = binding.gdn2_workspace_size(binding.GDN2_OP_BWD, B, T, H, 128, 128, 64, binding.GDN2_BF16)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    o, ST = binding.gdn2_fwd(*(d[n] for n in NAMES), d["S0"], save_states=True, ws=ws)
    g = binding.gdn2_bwd(*(d[n] for n in NAMES), d["dout"], d["S0"], dST, states_saved=True, ws=ws)
    torch.cuda.synchronize()
    out = {"o": o, "ST": ST}
    out.update({n: g[n] for n in GRADS})
    return out


def _inputs(B, T, H, seed):
    x = make_inputs(B, T, H, 128, 128, seed=seed, dtype="bf16", with_do=True, with_S0=True)
    d = {n: t.cuda() for n, t in x.items()}
    dST = torch.randn((B, H, 128, 128), generator=torch.Generator().manual_seed(seed)).cuda()
    return d, dST


@pytest.fixture
def no_cooperative():
    os.environ["GDN2_NO_COOPERATIVE"] = "1"
    try:
        yield
    finally:
        del os.environ["GDN2_NO_COOPERATIVE"]


@pytest.mark.gpu
def test_two_launch_form_matches_cooperative_launch(request):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    d, dST = _inputs(2, 333, 3, seed=4242)
    coop = _run(d, dST)
    request.getfixturevalue("no_cooperative")
    two = _run(d, dST)
    for n in coop:
        assert torch.equal(coop[n], two[n]), n


@pytest.mark.gpu
def test_more_heads_than_sms_match_the_same_heads_alone():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    H = 16
    B = sms // H + 1                      # B*H > number of SMs: both passes take the two-launch form
    d, dST = _inputs(B, 70, H, seed=777)
    big = _run(d, dST)
    for bsel in (0, B - 1):
        sl = {n: t[bsel:bsel + 1].contiguous() for n, t in d.items()}
        small = _run(sl, dST[bsel:bsel + 1].contiguous())
        for n in big:
            assert torch.equal(big[n][bsel:bsel + 1], small[n]), (bsel, n)


@pytest.mark.gpu
@pytest.mark.parametrize("gate", ["kda", "gdn"])
def test_two_launch_form_matches_for_scalar_gates(request, gate):
    """The same for the kernels' scalar-gate (KDA) and scalar-decay (Gated DeltaNet) instances."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    B, T, H = 2, 333, 3
    d, dST = _inputs(B, T, H, seed=4343)
    g = torch.Generator().manual_seed(17)
    beta = torch.sigmoid(torch.randn((B, T, H), generator=g)).to(torch.bfloat16).cuda()
    code = binding.GDN2_GATE_KDA if gate == "kda" else binding.GDN2_GATE_GDN
    la = d["log_alpha"] if gate == "kda" else \
        (-torch.nn.functional.softplus(torch.randn((B, T, H), generator=g)) / 16.0).to(torch.bfloat16).cuda()

    def run():
        need = binding.gdn2_beta_workspace_size(code, binding.GDN2_OP_BWD, B, T, H, 128, 128, 64, binding.GDN2_BF16)
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        o, ST = binding.gdn2_beta_fwd(code, d["q"], d["k"], d["v"], la, beta, d["S0"], save_states=True, ws=ws)
        gr = binding.gdn2_beta_bwd(code, d["q"], d["k"], d["v"], la, beta, d["dout"], d["S0"], dST,
                                   states_saved=True, ws=ws)
        torch.cuda.synchronize()
        return {"o": o, "ST": ST, **gr}

    coop = run()
    request.getfixturevalue("no_cooperative")
    two = run()
    for n in coop:
        assert torch.equal(coop[n], two[n]), n
