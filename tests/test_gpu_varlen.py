"""Packed variable-length sequences (gdn2_varlen_fwd / gdn2_varlen_bwd) against the fp64 oracle run on each
sequence alone (its own S0 and dST), with lengths that put a ragged chunk at every sequence boundary and
include sequences of exactly one and two chunks and of one token. Tolerances as for the operator (relative
L2): fp32 1e-4; bf16 o, S_T 2e-2, gradients 3e-2; checked per sequence.
"""
import numpy as np
import pytest
import torch

from conftest import rel_l2
from linear_attention_delta_gdn_b200 import binding
from linear_attention_delta_gdn_b200.inputs import make_inputs, to_f64

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "log_alpha", "b", "w")
GRADS = ("dq", "dk", "dv", "dlog_alpha", "db", "dw")
TOL_OUT = {"f32": 1e-4, "bf16": 2e-2}
TOL_GRAD = {"f32": 1e-4, "bf16": 3e-2}
LENGTHS = [100, 1, 64, 37, 200, 65, 128]


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_attention_delta_gdn_b200 import build
    build.build()


def _packed(lengths, H, Dk, Dv, dtype, seed):
    seqs = [make_inputs(1, L, H, Dk, Dv, seed=seed + i, dtype=dtype, with_do=True, with_S0=True)
            for i, L in enumerate(lengths)]
    packed = {n: torch.cat([s[n][0] for s in seqs], 0) for n in NAMES + ("dout",)}
    S0 = torch.cat([s["S0"] for s in seqs], 0)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    return seqs, packed, S0, cu


@pytest.mark.parametrize("dtype,Dk,Dv,chunk", [("bf16", 128, 128, 64), ("bf16", 128, 128, 32), ("f32", 64, 64, 64),
                                               ("bf16", 64, 128, 16)])
def test_varlen_against_oracle_per_sequence(oracle_mod, dtype, Dk, Dv, chunk):
    H = 3
    seqs, packed, S0, cu = _packed(LENGTHS, H, Dk, Dv, dtype, seed=1500 + Dk)
    N, Tmax = len(LENGTHS), max(LENGTHS)
    dST = torch.randn((N, H, Dk, Dv), generator=torch.Generator().manual_seed(8))
    d = {n: t.cuda() for n, t in packed.items()}
    cu_d, S0_d, dST_d = cu.cuda(), S0.cuda(), dST.cuda()
    dt = binding._dt(d["q"])
    ws = torch.empty(binding.gdn2_varlen_workspace_size(binding.GDN2_OP_BWD, N, Tmax, H, Dk, Dv, chunk, dt),
                     dtype=torch.uint8, device="cuda")
    o, ST = binding.gdn2_varlen_fwd(*(d[n] for n in NAMES), cu_d, Tmax, S0_d, chunk=chunk, save_states=True, ws=ws)
    g = binding.gdn2_varlen_bwd(*(d[n] for n in NAMES), d["dout"], cu_d, Tmax, S0_d, dST_d, chunk=chunk,
                                states_saved=True, ws=ws)
    assert binding.gdn2_device_status() == binding.GDN2_OK, binding.last_error()
    o, ST = to_f64(o), to_f64(ST)
    got = {n: to_f64(g[n]) for n in GRADS + ("dS0",)}
    for i, s in enumerate(seqs):
        a, e = int(cu[i]), int(cu[i + 1])
        f = {n: to_f64(t) for n, t in s.items()}
        o_ref, ST_ref = oracle_mod.fwd(*(f[n] for n in NAMES), S0=f["S0"])
        ref = oracle_mod.bwd(*(f[n] for n in NAMES), dout=f["dout"], S0=f["S0"], dST=dST[i:i + 1].double().numpy())
        assert rel_l2(o[a:e], o_ref[0]) <= TOL_OUT[dtype], ("o", i)
        assert rel_l2(ST[i], ST_ref[0]) <= TOL_OUT[dtype], ("ST", i)
        for n in GRADS:
            assert np.all(np.isfinite(got[n][a:e])), (n, i)
            assert rel_l2(got[n][a:e], ref[n][0]) <= TOL_GRAD[dtype], (n, i, rel_l2(got[n][a:e], ref[n][0]))
        assert rel_l2(got["dS0"][i], ref["dS0"][0]) <= TOL_GRAD[dtype], ("dS0", i)


def test_varlen_inconsistent_lengths_are_reported():
    """A sequence longer than Tmax is cut (the copies stay inside the buffers) and gdn2_device_status reports it;
    so is a cu_seqlens that reaches past the packed length (that sequence is skipped)."""
    H, D = 2, 128
    _, packed, S0, cu = _packed([70, 30], H, D, D, "bf16", seed=1600)
    d = {n: t.cuda() for n, t in packed.items()}
    binding.gdn2_device_status()
    o, _ = binding.gdn2_varlen_fwd(*(d[n] for n in NAMES), cu.cuda(), 64, S0.cuda())
    assert binding.gdn2_device_status() == binding.GDN2_ERR_INVALID
    assert "cu_seqlens" in binding.last_error() and "Tmax" in binding.last_error()
    bad = cu.clone()
    bad[-1] = 200   # past the 100 packed tokens
    binding.gdn2_varlen_fwd(*(d[n] for n in NAMES), bad.cuda(), 128, S0.cuda())
    assert binding.gdn2_device_status() == binding.GDN2_ERR_INVALID
    assert "outside" in binding.last_error()
    binding.gdn2_varlen_fwd(*(d[n] for n in NAMES), cu.cuda(), 128, S0.cuda())
    assert binding.gdn2_device_status() == binding.GDN2_OK
