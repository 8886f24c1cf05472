"""GPU parity: libgdn2 (through its C ABI) against the fp64 oracle on the same
seeded inputs.

Tolerances (relative L2, ||x - ref|| / ||ref||), applied to the whole tensor AND to
every (batch, head) slice on its own, so that one bad head cannot hide among good ones:
  fp32 inputs: o, S_T and every gradient <= 1e-4
  bf16 inputs (fp32 state and accumulation): o, S_T <= 2e-2; gradients <= 3e-2
The oracle consumes exactly the dtype-rounded inputs, widened to fp64. The full-size
workloads are checked on every (batch, head) pair; the oracle computes each pair
independently of the others (heads never interact).
"""
import numpy as np
import pytest
import torch

from conftest import rel_l2, worst_head_rel_l2
from linear_attention_delta_gdn_b200 import binding
from linear_attention_delta_gdn_b200.inputs import WORKLOADS, make_inputs, make_workload_inputs, make_decode_stream, to_f64

pytestmark = pytest.mark.gpu

TOL_OUT = {"f32": 1e-4, "bf16": 2e-2}
TOL_GRAD = {"f32": 1e-4, "bf16": 3e-2}
GRADS = ("dq", "dk", "dv", "dlog_alpha", "db", "dw")
NAMES = ("q", "k", "v", "log_alpha", "b", "w")


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_attention_delta_gdn_b200 import build
    build.build()


def dev(x):
    return {n: (t.cuda() if t is not None else None) for n, t in x.items()}


def f64(x):
    return {n: to_f64(t) for n, t in x.items() if t is not None}


def heads_slice(a, heads, state=False):
    """Stack the (b, h) slices of a [B, T, H, D] (or [B, H, Dk, Dv]) array as batch entries."""
    if state:
        return np.stack([a[b, h] for b, h in heads])[:, None]
    return np.stack([a[b, :, h] for b, h in heads])[:, :, None]


def oracle_fwd(oracle_mod, x, heads=None):
    g = f64(x)
    S0 = g.get("S0")
    args = [g[n] for n in NAMES]
    if heads is not None:
        args = [heads_slice(a, heads) for a in args]
        S0 = None if S0 is None else heads_slice(S0, heads, state=True)
    return oracle_mod.fwd(*args, S0=S0)


def oracle_bwd(oracle_mod, x, dST=None, heads=None):
    g = f64(x)
    S0 = g.get("S0")
    args = [g[n] for n in NAMES]
    dout = g["dout"]
    if heads is not None:
        args = [heads_slice(a, heads) for a in args]
        dout = heads_slice(dout, heads)
        S0 = None if S0 is None else heads_slice(S0, heads, state=True)
        dST = None if dST is None else heads_slice(dST, heads, state=True)
    return oracle_mod.bwd(*args, dout=dout, S0=S0, dST=dST)


def gpu_fwd(x, chunk):
    d = dev(x)
    o, ST = binding.gdn2_fwd(*(d[n] for n in NAMES), d.get("S0"), chunk=chunk)
    torch.cuda.synchronize()
    return to_f64(o), to_f64(ST)


def pick(arr, heads, state=False):
    return heads_slice(arr, heads, state) if heads is not None else arr


def check_fwd(oracle_mod, x, chunk, dtype, heads=None):
    o, ST = gpu_fwd(x, chunk)
    o_ref, ST_ref = oracle_fwd(oracle_mod, x, heads)
    o, ST = pick(o, heads), pick(ST, heads, True)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(ST))
    eo, es = rel_l2(o, o_ref), rel_l2(ST, ST_ref)
    wo, ws = worst_head_rel_l2(o, o_ref), worst_head_rel_l2(ST, ST_ref, state=True)
    assert eo <= TOL_OUT[dtype] and wo <= TOL_OUT[dtype], "o rel err %.3g (worst head %.3g)" % (eo, wo)
    assert es <= TOL_OUT[dtype] and ws <= TOL_OUT[dtype], "S_T rel err %.3g (worst head %.3g)" % (es, ws)
    return eo, es


# ---------------------------------------------------------------- decode

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("Dk,Dv", [(128, 128), (64, 64), (32, 128), (128, 16)])
def test_decode_steps(oracle_mod, dtype, Dk, Dv):
    x = make_inputs(3, 5, 2, Dk, Dv, seed=7 + Dk + Dv, dtype=dtype, with_S0=True)
    d = dev(x)
    S = d["S0"].clone()
    Sref = to_f64(x["S0"])
    g = f64(x)
    for t in range(5):
        o = binding.gdn2_decode_step(*(d[n][:, t].contiguous() for n in NAMES), S)
        o_ref, Sref = oracle_mod.decode(*(g[n][:, t] for n in NAMES), Sref)
        assert rel_l2(to_f64(o), o_ref) <= TOL_OUT[dtype]
    assert rel_l2(to_f64(S), Sref) <= TOL_OUT[dtype] / 10


def test_decode_workload_sampled(oracle_mod):
    wl = WORKLOADS["decode-bf16-b256h16d128x1024"]
    xs = make_decode_stream(wl.T, wl.B, wl.H, wl.Dk, wl.Dv, wl.seed, wl.dtype, device="cuda")
    heads = [(0, 0), (17, 3), (100, 7), (128, 8), (200, 11), (255, 15), (64, 1), (31, 14)]
    bi = torch.tensor([b for b, _ in heads], device="cuda")
    hi = torch.tensor([h for _, h in heads], device="cuda")
    S = xs["S0"].clone()
    Sref = to_f64(xs["S0"][bi, hi])[:, None]
    o_gpu = []
    for t in range(wl.T):
        o = binding.gdn2_decode_step(*(xs[n][t] for n in NAMES), S)
        o_gpu.append(o[bi, hi])
    o_gpu = to_f64(torch.stack(o_gpu))                    # [steps, 8, Dv]
    sub = {n: to_f64(xs[n][:, bi, hi]) for n in NAMES}    # [steps, 8, D]
    o_ref = np.zeros_like(o_gpu)
    for t in range(wl.T):
        o_t, Sref = oracle_mod.decode(*(sub[n][t][:, None] for n in NAMES), Sref)
        o_ref[t] = o_t[:, 0]
    assert rel_l2(o_gpu, o_ref) <= TOL_OUT["bf16"]
    assert rel_l2(to_f64(S[bi, hi]), Sref[:, 0]) <= TOL_OUT["bf16"]


# ---------------------------------------------------------------- forward

@pytest.mark.parametrize("T", [1, 37, 64, 150])
@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("Dk,Dv", [(64, 64), (32, 128)])
def test_fwd_fp32_small(oracle_mod, T, chunk, Dk, Dv):
    x = make_inputs(2, T, 3, Dk, Dv, seed=T + chunk + Dk, dtype="f32", with_S0=(T % 2 == 1))
    check_fwd(oracle_mod, x, chunk, "f32")


@pytest.mark.parametrize("T", [1, 37, 64, 150, 333])
@pytest.mark.parametrize("with_S0", [False, True])
def test_fwd_bf16_d128(oracle_mod, T, with_S0):
    x = make_inputs(2, T, 3, 128, 128, seed=100 + T, dtype="bf16", with_S0=with_S0)
    check_fwd(oracle_mod, x, 64, "bf16")


# bf16 shapes off the tensor-core shape (d_k = d_v = 128) run on the recurrent kernels (bf16 in, fp32 math);
# bf16 at d = 128 with chunk 16 or 32 runs on the tensor-core kernels (64-token chunks inside).
BF16_SHAPES = [(64, 64, 64), (128, 128, 32), (128, 128, 16), (64, 128, 16), (128, 64, 32), (16, 16, 64),
               (32, 128, 64)]


@pytest.mark.parametrize("Dk,Dv,chunk", BF16_SHAPES)
def test_fwd_bf16_other_shapes(oracle_mod, Dk, Dv, chunk):
    x = make_inputs(2, 97, 2, Dk, Dv, seed=200 + Dk + chunk, dtype="bf16", with_S0=True)
    check_fwd(oracle_mod, x, chunk, "bf16")


@pytest.mark.parametrize("chunk", [16, 32])
def test_bf16_d128_small_chunk_runs_on_tensor_cores(oracle_mod, chunk):
    """The chunk length does not change the result, so bf16 d = 128 with chunk 16 or 32 takes the tensor-core
    kernels (64-token chunks) instead of the token-recurrent ones."""
    x = make_inputs(1, 150, 3, 128, 128, seed=210 + chunk, dtype="bf16", with_do=True, with_S0=True)
    binding.trace_read()
    binding.trace_enable(True)
    try:
        check_fwd(oracle_mod, x, chunk, "bf16")
        check_bwd(oracle_mod, x, chunk, "bf16", with_dST=True)
        check_bwd(oracle_mod, x, chunk, "bf16", with_dST=True, saved=True)
    finally:
        binding.trace_enable(False)
    names = set(binding.trace_read())
    assert {"chunk_fwd_kernel", "chunk_bwd_kernel"} <= names, names
    assert not names & {"recurrent_fwd_kernel", "recurrent_bwd_kernel"}, names


def test_fwd_workload_fp32(oracle_mod):
    wl = WORKLOADS["fwd-f32-b1h2t256d64"]
    check_fwd(oracle_mod, make_workload_inputs(wl), wl.chunk, wl.dtype)


@pytest.mark.parametrize("name", ["fwd-bf16-b4h16t4096d128", "fwd-bf16-b1h16t65536d128-s0"])
def test_fwd_workload_all_heads(oracle_mod, name):
    """The full-size forward workloads, every (batch, head) pair against the oracle."""
    wl = WORKLOADS[name]
    check_fwd(oracle_mod, make_workload_inputs(wl), wl.chunk, wl.dtype)


def test_fwd_resume_from_state(oracle_mod):
    """fwd over [0, T) equals fwd over [0, T1) then [T1, T) started from S_T1."""
    x = make_inputs(2, 200, 2, 128, 128, seed=300, dtype="bf16", with_S0=True)
    d = dev(x)
    o, ST = binding.gdn2_fwd(*(d[n] for n in NAMES), d["S0"])
    T1 = 128
    first = {n: d[n][:, :T1].contiguous() for n in NAMES}
    second = {n: d[n][:, T1:].contiguous() for n in NAMES}
    o1, S1 = binding.gdn2_fwd(*(first[n] for n in NAMES), d["S0"])
    o2, S2 = binding.gdn2_fwd(*(second[n] for n in NAMES), S1)
    assert rel_l2(to_f64(torch.cat([o1, o2], 1)), to_f64(o)) < 1e-2
    assert rel_l2(to_f64(S2), to_f64(ST)) < 1e-2


def test_fwd_state_in_place(oracle_mod):
    x = make_inputs(1, 70, 2, 128, 128, seed=301, dtype="bf16", with_S0=True)
    d = dev(x)
    _, ST = binding.gdn2_fwd(*(d[n] for n in NAMES), d["S0"])
    S = d["S0"].clone()
    binding.gdn2_fwd(*(d[n] for n in NAMES), S, ST=S)
    assert torch.equal(S, ST)


# ---------------------------------------------------------------- backward

# Exact retrieval (b = 1, q = k, unit keys): the outputs do not depend on the state, so the gradient reaching
# S0 is only the incoming dST carried back through the decays and erases, ~1/2700 of it at these shapes. There
# dS0 is ill-conditioned: perturbing the inputs by half a bf16 ulp moves the oracle's own dS0 by more than its
# norm, ~5e-4 of ||dST|| (tests/test_oracle_pins.py::test_exact_retrieval_dS0_is_ill_conditioned). Its error
# is therefore measured against ||dST||, with a bound a few times that input-level sensitivity.
DS0_VS_DST_TOL = 3e-3


def check_bwd(oracle_mod, x, chunk, dtype, heads=None, with_dST=False, saved=False, ds0_vs_dST=False):
    """Gradients against the oracle, whole tensor and worst (batch, head). With ds0_vs_dST the error of dS0 is
    measured against the norm of the incoming state gradient dST (see DS0_VS_DST_TOL)."""
    d = dev(x)
    dST = None
    if with_dST:
        B, _, H, Dk = x["q"].shape
        dST = torch.randn((B, H, Dk, x["v"].shape[-1]), generator=torch.Generator().manual_seed(5))
    if saved:
        B, T, H, Dk = x["q"].shape
        Dv = x["v"].shape[-1]
        need = binding.gdn2_workspace_size(binding.GDN2_OP_BWD, B, T, H, Dk, Dv, chunk, binding._dt(d["q"]))
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        binding.gdn2_fwd(*(d[n] for n in NAMES), d.get("S0"), chunk=chunk, save_states=True, ws=ws)
        g = binding.gdn2_bwd(*(d[n] for n in NAMES), d["dout"], d.get("S0"),
                             None if dST is None else dST.cuda(), chunk=chunk, states_saved=True, ws=ws)
    else:
        g = binding.gdn2_bwd(*(d[n] for n in NAMES), d["dout"], d.get("S0"),
                             None if dST is None else dST.cuda(), chunk=chunk)
    torch.cuda.synchronize()
    ref = oracle_bwd(oracle_mod, x, None if dST is None else dST.double().numpy(), heads)
    errs, worst = {}, {}
    for n in GRADS:
        got = pick(to_f64(g[n]), heads)
        assert np.all(np.isfinite(got)), n
        errs[n] = rel_l2(got, ref[n])
        worst[n] = worst_head_rel_l2(got, ref[n])
    got = pick(to_f64(g["dS0"]), heads, True)
    assert np.all(np.isfinite(got)), "dS0"
    if ds0_vs_dST:
        assert dST is not None
        dST_ref = pick(dST.double().numpy(), heads, True)
        e = float(np.linalg.norm((got - ref["dS0"]).ravel()) / np.linalg.norm(dST_ref.ravel()))
        assert e <= DS0_VS_DST_TOL, "dS0 error %.3g of ||dST|| (bound %g)" % (e, DS0_VS_DST_TOL)
    else:
        errs["dS0"] = rel_l2(got, ref["dS0"])
        worst["dS0"] = worst_head_rel_l2(got, ref["dS0"], state=True)
    bad = {n: (errs[n], worst[n]) for n in errs if max(errs[n], worst[n]) > TOL_GRAD[dtype]}
    assert not bad, "gradient rel errors (whole, worst head) above %g: %s (all: %s; worst heads: %s)" % (
        TOL_GRAD[dtype], bad, errs, worst)
    return errs


@pytest.mark.parametrize("T", [1, 37, 150])
@pytest.mark.parametrize("chunk", [16, 64])
def test_bwd_fp32_small(oracle_mod, T, chunk):
    x = make_inputs(2, T, 2, 32, 64, seed=400 + T + chunk, dtype="f32", with_do=True, with_S0=True)
    check_bwd(oracle_mod, x, chunk, "f32", with_dST=True)


@pytest.mark.parametrize("T", [1, 37, 64, 150, 300])
@pytest.mark.parametrize("with_S0", [False, True])
def test_bwd_bf16_d128(oracle_mod, T, with_S0):
    x = make_inputs(2, T, 2, 128, 128, seed=500 + T, dtype="bf16", with_do=True, with_S0=with_S0)
    check_bwd(oracle_mod, x, 64, "bf16", with_dST=with_S0)


@pytest.mark.parametrize("saved", [False, True])
def test_bwd_saved_states(oracle_mod, saved):
    x = make_inputs(1, 190, 3, 128, 128, seed=600, dtype="bf16", with_do=True, with_S0=True)
    check_bwd(oracle_mod, x, 64, "bf16", with_dST=True, saved=saved)


def test_bwd_workload_all_heads(oracle_mod):
    """The full-size training workload (the bench step: forward keeping the states, then the backward), every
    (batch, head) pair against the oracle."""
    wl = WORKLOADS["fwdbwd-bf16-b4h16t4096d128"]
    x = make_workload_inputs(wl)
    errs = check_bwd(oracle_mod, x, wl.chunk, wl.dtype, saved=True)
    print("gradient rel errors:", errs)


@pytest.mark.parametrize("Dk,Dv,chunk", BF16_SHAPES)
@pytest.mark.parametrize("saved", [False, True])
def test_bwd_bf16_other_shapes(oracle_mod, Dk, Dv, chunk, saved):
    """bf16 backward off the tensor-core shape (the bf16 instantiation of the recurrent backward), and bf16
    d = 128 with chunk 16 or 32 (tensor-core kernels)."""
    x = make_inputs(2, 97, 2, Dk, Dv, seed=220 + Dk + Dv + chunk, dtype="bf16", with_do=True, with_S0=True)
    check_bwd(oracle_mod, x, chunk, "bf16", with_dST=True, saved=saved)


def test_autograd_matches_direct():
    x = make_inputs(2, 100, 2, 128, 128, seed=700, dtype="bf16", with_do=True, with_S0=True)
    d = dev(x)
    leaves = {n: d[n].clone().requires_grad_(True) for n in NAMES}
    S0 = d["S0"].clone().requires_grad_(True)
    o, ST = binding.gated_delta_rule2(*(leaves[n] for n in NAMES), S0)
    (o.float() * d["dout"].float()).sum().backward()
    g = binding.gdn2_bwd(*(d[n] for n in NAMES), d["dout"], d["S0"])
    for n, gn in zip(NAMES, GRADS):
        assert rel_l2(to_f64(leaves[n].grad), to_f64(g[gn])) < 1e-6, n
    assert rel_l2(to_f64(S0.grad), to_f64(g["dS0"])) < 1e-6


@pytest.mark.parametrize("B,T,H,S0", [(1, 8192, 4, True), (1, 6000, 2, False), (2, 4100, 3, True)])
def test_long_sequence_segments(oracle_mod, B, T, H, S0):
    """With few heads and long sequences the forward cuts each head's chunks into segments (segment maps, a prefix
    over them, the segments again from their start states). Same results as one chain per head (GDN2_NO_SPLIT)
    and as the oracle, for the output, the final state and, through the backward's recompute and through the
    saved states, the gradients."""
    import os
    x = make_inputs(B, T, H, 128, 128, seed=1700 + T, dtype="bf16", with_do=True, with_S0=S0)
    d = dev(x)
    binding.trace_read()
    binding.trace_enable(True)
    try:
        o, ST = binding.gdn2_fwd(*(d[n] for n in NAMES), d.get("S0"))
    finally:
        binding.trace_enable(False)
    assert "split_prefix_kernel" in binding.trace_read()      # the segmented form ran
    os.environ["GDN2_NO_SPLIT"] = "1"
    try:
        o1, ST1 = binding.gdn2_fwd(*(d[n] for n in NAMES), d.get("S0"))
    finally:
        del os.environ["GDN2_NO_SPLIT"]
    torch.cuda.synchronize()
    assert rel_l2(to_f64(o), to_f64(o1)) < 1e-2 and rel_l2(to_f64(ST), to_f64(ST1)) < 1e-2
    check_fwd(oracle_mod, x, 64, "bf16")
    check_bwd(oracle_mod, x, 64, "bf16", with_dST=True)
    check_bwd(oracle_mod, x, 64, "bf16", with_dST=True, saved=True)
    assert binding.gdn2_device_status() == binding.GDN2_OK, binding.last_error()
