"""GPU parity on the method's degenerate cases and on an empty sequence (tensor-core path: bf16, d = 128,
chunk 64), against the fp64 oracle with the bf16 tolerances (o, S_T <= 2e-2; gradients <= 3e-2).

The degenerate cases are the ones the oracle is pinned on (closed forms and the exact-retrieval invariant):
  no decay         log_alpha = 0 (alpha = 1)
  no erase         b = 0 (gated linear attention)
  no write         w = 0 and S0 = 0: o and S_T are exactly zero
  exact retrieval  b = 1 and q = k (unit norm): o_t = w_t * v_t
and decays strong enough that the asymmetric factor exp(-G) of the chunk form would overflow (the kernels
then leave those channels out of the tensor-core pair products and sum their terms exactly):
  strong_decay     log_alpha = -1.2 per token (exp(-77) over a 64-token chunk)
  decay_3          log_alpha = -3 per token on every channel (exp(-192) over a chunk)
  mixed_20         three channels at -20 per token, the rest from the recipe's distribution
  spike            the recipe's distribution plus one token per chunk at -100 on every channel
  tame_edge        log_alpha = -0.9 per token (a chunk's decay mass 57.6, just inside the tensor-core range)
"""
import numpy as np
import pytest
import torch

from test_gpu_parity import NAMES, check_bwd, check_fwd, dev
from linear_attention_delta_gdn_b200 import binding
from linear_attention_delta_gdn_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

CASES = ("no_decay", "no_erase", "no_write", "exact_retrieval", "strong_decay", "decay_3", "mixed_20", "spike",
         "tame_edge")


def _inputs(case):
    x = make_inputs(2, 150, 3, 128, 128, seed=900 + CASES.index(case), dtype="bf16", with_do=True, with_S0=True)
    if case == "no_decay":
        x["log_alpha"].zero_()
    elif case == "no_erase":
        x["b"].zero_()
    elif case == "no_write":
        x["w"].zero_()
        del x["S0"]
    elif case == "exact_retrieval":
        x["b"].fill_(1.0)
        x["q"] = x["k"].clone()
    elif case == "strong_decay":
        x["log_alpha"].fill_(-1.2)
    elif case == "decay_3":
        x["log_alpha"].fill_(-3.0)
    elif case == "mixed_20":
        x["log_alpha"][..., [5, 77, 100]] = -20.0
    elif case == "spike":
        x["log_alpha"][:, 10::64] = -100.0
    elif case == "tame_edge":
        x["log_alpha"].fill_(-0.9)
    return x


@pytest.mark.parametrize("case", CASES)
def test_fwd_degenerate_cases(oracle_mod, case):
    x = _inputs(case)
    check_fwd(oracle_mod, x, 64, "bf16")
    if case == "no_write":   # nothing is ever written: exact zeros, not only within the tolerance
        o, ST = binding.gdn2_fwd(*(dev(x)[n] for n in NAMES), None)
        assert int(torch.count_nonzero(o)) == 0 and int(torch.count_nonzero(ST)) == 0


@pytest.mark.parametrize("case", CASES)
def test_bwd_degenerate_cases(oracle_mod, case):
    # With exact retrieval every read removes the state's component along k_t, so the gradient reaching S0
    # is a near-cancellation: its reference norm (~0.12) is ~1/2700 of the incoming dST's (~314). Its error
    # is then measured against that incoming gradient; the other gradients keep the relative check.
    check_bwd(oracle_mod, _inputs(case), 64, "bf16", with_dST=case != "no_write",
              ds0_vs_dST=case == "exact_retrieval")


def test_empty_sequence():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    x = make_inputs(2, 0, 3, 128, 128, seed=1, dtype="bf16", with_do=True, with_S0=True)
    d = dev(x)
    o, ST = binding.gdn2_fwd(*(d[n] for n in NAMES), d["S0"])
    assert tuple(o.shape) == (2, 0, 3, 128)
    assert torch.equal(ST, d["S0"])   # no tokens: the final state is the initial one
    dST = torch.randn((2, 3, 128, 128), generator=torch.Generator().manual_seed(2)).cuda()
    g = binding.gdn2_bwd(*(d[n] for n in NAMES), d["dout"], d["S0"], dST)
    torch.cuda.synchronize()
    assert torch.equal(g["dS0"], dST)
    for n in ("dq", "dk", "dv", "dlog_alpha", "db", "dw"):
        assert g[n].numel() == 0, n
    assert binding.gdn2_device_status() == binding.GDN2_OK
