"""gdn2_bwd_no_alloc: the backward for callers that cannot allocate device memory.

It takes its scratch memory from a fixed array inside libgdn2.so instead of a
caller-supplied workspace. These tests call it through the C ABI and check it
against gdn2_bwd (the entry point with a caller workspace) on the same inputs,
twice in a row (the array keeps the previous call's contents), and check that
a problem larger than the array is refused before anything runs.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from conftest import rel_l2
from linear_attention_delta_gdn_b200 import binding
from linear_attention_delta_gdn_b200.inputs import make_inputs, to_f64

NAMES = ("q", "k", "v", "log_alpha", "b", "w")
GRADS = ("dq", "dk", "dv", "dlog_alpha", "db", "dw", "dS0")
TOL = {"f32": 1e-4, "bf16": 3e-2}


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _no_alloc(L, d, dST, dtype_code, chunk):
    B, T, H, Dk = d["q"].shape
    Dv = d["v"].shape[-1]
    g = {n: torch.full_like(d["q"], float("nan")) for n in ("dq", "dk", "dlog_alpha", "db")}
    g.update({n: torch.full_like(d["v"], float("nan")) for n in ("dv", "dw")})
    g["dS0"] = torch.full((B, H, Dk, Dv), float("nan"), dtype=torch.float32, device="cuda")
    rc = L.gdn2_bwd_no_alloc(*(_p(d[n]) for n in NAMES), _p(d.get("S0")), _p(d["dout"]), _p(dST),
                             _p(g["dq"]), _p(g["dk"]), _p(g["dv"]), _p(g["dlog_alpha"]), _p(g["db"]),
                             _p(g["dw"]), _p(g["dS0"]), B, T, H, Dk, Dv, chunk, dtype_code,
                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, L.gdn2_last_error()
    torch.cuda.synchronize()
    return g


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,B,T,H,D,chunk", [("bf16", 2, 200, 3, 128, 64), ("f32", 1, 70, 2, 64, 32)])
def test_no_alloc_matches_workspace_backward(dtype, B, T, H, D, chunk):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_attention_delta_gdn_b200 import build
    build.build()
    L = binding.lib()
    x = make_inputs(B, T, H, D, D, seed=900 + T, dtype=dtype, with_do=True, with_S0=True)
    d = {n: t.cuda() for n, t in x.items()}
    dST = torch.randn((B, H, D, D), generator=torch.Generator().manual_seed(3)).cuda()
    ref = binding.gdn2_bwd(*(d[n] for n in NAMES), d["dout"], d["S0"], dST, chunk=chunk)
    torch.cuda.synchronize()
    code = binding.GDN2_BF16 if dtype == "bf16" else binding.GDN2_F32
    for call in range(2):
        got = _no_alloc(L, d, dST, code, chunk)
        for n in GRADS:
            a = to_f64(got[n])
            assert np.all(np.isfinite(a)), (call, n)
            assert rel_l2(a, to_f64(ref[n])) <= TOL[dtype], (call, n)


def test_no_alloc_rejects_problems_larger_than_the_array():
    from linear_attention_delta_gdn_b200 import build
    build.build()
    L = binding.lib()
    cap = L.gdn2_no_alloc_scratch_bytes()
    assert cap == 64 * 1024 * 1024
    # 1.3B-layer shape: the backward needs far more scratch than the array holds
    need = binding.gdn2_workspace_size(binding.GDN2_OP_BWD, 4, 4096, 16, 128, 128, 64, binding.GDN2_BF16)
    assert need > cap
    p = ctypes.c_void_p(1 << 20)
    rc = L.gdn2_bwd_no_alloc(*([p] * 6), None, p, None, p, p, p, p, p, p, None,
                             4, 4096, 16, 128, 128, 64, binding.GDN2_BF16, None)
    assert rc == 3
    assert b"fixed array holds" in L.gdn2_last_error()


def test_no_alloc_accepts_exactly_the_problems_that_fit():
    """The size check sits exactly at the array's capacity: on the tensor-core shape (bf16, d = 128), the
    largest sequence of one head whose backward scratch fits passes the size check (on a host without a GPU
    the call then stops at the device lookup with GDN2_ERR_CUDA; with a GPU present that call is not made,
    since it would launch on the placeholder pointers), and one more 64-token chunk is refused with
    GDN2_ERR_WORKSPACE before anything runs."""
    from linear_attention_delta_gdn_b200 import build
    build.build()
    L = binding.lib()
    cap = L.gdn2_no_alloc_scratch_bytes()

    def need(n):   # backward scratch of one head of n 64-token chunks
        return binding.gdn2_workspace_size(binding.GDN2_OP_BWD, 1, 64 * n, 1, 128, 128, 64, binding.GDN2_BF16)

    n = 1
    while need(n + 1) <= cap:
        n += 1
    assert need(n) <= cap < need(n + 1)
    assert n >= 300      # a few hundred 64-token chunk-heads fit in the array
    p = ctypes.c_void_p(1 << 20)
    cases = [(n + 1, False)] + ([] if torch.cuda.is_available() else [(n, True)])
    for chunks, fits in cases:
        rc = L.gdn2_bwd_no_alloc(*([p] * 6), None, p, None, p, p, p, p, p, p, None,
                                 1, 64 * chunks, 1, 128, 128, 64, binding.GDN2_BF16, None)
        if fits:
            assert rc == 4, L.gdn2_last_error()      # past the size check, stopped at the device lookup
        else:
            assert rc == 3 and b"fixed array holds" in L.gdn2_last_error()
