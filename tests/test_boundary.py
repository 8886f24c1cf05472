"""Host-side tests of the C ABI (no GPU needed): the library loads, exports every
entry point that include/gdn2.h declares, sizes workspaces, and rejects bad
arguments with a status before launching anything."""
import ctypes
import os
import re
import threading

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "gdn2.h")


@pytest.fixture(scope="module")
def L():
    from linear_attention_delta_gdn_b200 import build, binding
    build.build()
    return binding.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn2_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert "gdn2_fwd" in names and "gdn2_bwd" in names and "gdn2_decode_step" in names
    for n in names:
        assert hasattr(L, n), n
        ctypes.cast(getattr(L, n), ctypes.c_void_p)


def test_binding_lists_all_exports():
    from linear_attention_delta_gdn_b200 import binding
    assert sorted(binding.EXPORTS) == declared_functions()


def test_version_and_status_strings(L):
    assert L.gdn2_version() >= 100
    for s in range(6):
        assert L.gdn2_status_string(s).startswith(b"GDN2_")


def test_workspace_sizes(L):
    from linear_attention_delta_gdn_b200.binding import gdn2_workspace_size as ws
    # fp32 recurrent path: checkpoints every chunk, fp32
    assert ws(0, 1, 256, 2, 64, 64, 64, 0) == 0
    fs = ws(1, 1, 256, 2, 64, 64, 64, 0)
    assert fs >= 1 * 2 * 4 * 64 * 64 * 4 and fs % 256 == 0
    assert ws(2, 1, 256, 2, 64, 64, 64, 0) > fs
    # bf16 shape of the 1.3B training layer: the inference forward keeps a WY image
    # (T | P | Wm | Qt | Kt | gC | untame mask, 65 KB, plus a 16 KB Kh tile used by chunks with untame channels)
    # and a ready flag per chunk; training adds the state (32 KB) and Delta (16 KB) images; the backward adds
    # the dZ (32 KB) and dDelta (16 KB) images, its ready flags, a work counter and an abort word
    units = 4 * 16 * 64
    i = ws(0, 4, 4096, 16, 128, 128, 64, 1)
    assert i == units * 82944 + units * 4
    f = ws(1, 4, 4096, 16, 128, 128, 64, 1)
    b = ws(2, 4, 4096, 16, 128, 128, 64, 1)
    assert f == units * (32768 + 16384) + i
    assert b == f + units * (32768 + 16384) + (units * 4 + 256)
    # ragged T rounds the chunk count up
    assert ws(1, 1, 65, 1, 128, 128, 64, 1) == ws(1, 1, 128, 1, 128, 128, 64, 1)
    # bf16 d = 128 runs the tensor-core kernels (64-token chunks) whatever chunk is requested
    for op in (0, 1, 2):
        for c in (16, 32):
            assert ws(op, 2, 300, 3, 128, 128, c, 1) == ws(op, 2, 300, 3, 128, 128, 64, 1)
    # the maps of a sequence piece: WY images, then flags with the work counter and abort word
    assert ws(3, 4, 4096, 16, 128, 128, 64, 1) == units * 82944 + units * 4 + 256
    # a long piece with few heads adds its segment maps (19 fp32 128 x 128 matrices per head)
    u1 = 1 * 2 * 256
    assert ws(3, 1, 16384, 2, 128, 128, 64, 1) == u1 * 82944 + u1 * 4 + 256 + 2 * 19 * 128 * 128 * 4
    assert ws(3, 1, 256, 2, 64, 64, 64, 0) == 0
    # invalid problems report zero
    assert ws(1, 0, 16, 1, 64, 64, 64, 1) == 0
    assert ws(1, 1, 16, 1, 96, 64, 64, 1) == 0
    assert ws(1, 1, 16, 1, 64, 64, 48, 1) == 0
    assert ws(1, 1, 16, 1, 64, 64, 64, 7) == 0


def _fwd(L, ptr=1 << 20, S0=None, ST=None, B=1, T=8, H=1, Dk=64, Dv=64, chunk=64, dt=1, save=0, ws=None, wsb=0,
         **over):
    args = dict(q=ptr, k=ptr, v=ptr, la=ptr, b=ptr, w=ptr, o=ptr)
    args.update(over)
    return L.gdn2_fwd(args["q"], args["k"], args["v"], args["la"], args["b"], args["w"], S0, args["o"], ST,
                      B, T, H, Dk, Dv, chunk, dt, save, ws, wsb, None)


def test_fwd_rejects_bad_arguments(L):
    assert _fwd(L, q=None) == 1
    assert b"q must not be NULL" in L.gdn2_last_error()
    assert _fwd(L, o=None) == 1
    assert _fwd(L, k=(1 << 20) + 2) == 1                  # misaligned
    assert b"16-byte aligned" in L.gdn2_last_error()
    assert _fwd(L, B=0) == 1
    assert _fwd(L, T=-1) == 1
    assert _fwd(L, Dk=96) == 2
    assert _fwd(L, chunk=128) == 2
    assert _fwd(L, dt=3) == 1
    assert _fwd(L, save=1) == 3                            # no workspace
    assert _fwd(L, save=1, ws=1 << 20, wsb=16) == 3        # too small
    assert b"workspace" in L.gdn2_last_error()
    # the tensor-core forward needs its WY workspace even without save_states
    assert _fwd(L, Dk=128, Dv=128) == 3
    assert _fwd(L, Dk=128, Dv=128, ws=(1 << 20) + 16, wsb=1 << 30) == 1   # misaligned workspace
    assert b"256-byte" in L.gdn2_last_error()


def test_bwd_and_decode_reject_bad_arguments(L):
    p = 1 << 20
    P = [p] * 6
    rc = L.gdn2_bwd(*P, None, p, None, p, p, p, p, p, p, None, 1, 8, 1, 64, 64, 64, 1, 0, None, 0, None)
    assert rc == 3                                         # workspace required
    rc = L.gdn2_bwd(*P, None, None, None, p, p, p, p, p, p, None, 1, 8, 1, 64, 64, 64, 1, 0, p, 1 << 30, None)
    assert rc == 1 and b"dout" in L.gdn2_last_error()
    rc = L.gdn2_bwd(*P, None, p, None, p, p, p, p, p, p, None, 1, 8, 1, 64, 64, 64, 1, 0, p + 16, 1 << 30, None)
    assert rc == 1 and b"256-byte" in L.gdn2_last_error()
    assert L.gdn2_decode_step(*P, None, p, 1, 1, 64, 64, 1, None) == 1
    assert L.gdn2_decode_step(*P, p, p, 1, 1, 64, 24, 1, None) == 2
    assert L.gdn2_decode_step(*P, p, p, 0, 1, 64, 64, 1, None) == 1


def test_error_detail_is_per_thread(L):
    assert _fwd(L, q=None) == 1
    seen = []

    def other():
        _fwd(L, Dk=96)
        seen.append(L.gdn2_last_error())

    th = threading.Thread(target=other)
    th.start()
    th.join()
    assert b"Dk=96" in seen[0]
    assert b"q must not be NULL" in L.gdn2_last_error()


def test_binding_refuses_cpu_tensors():
    import torch
    from linear_attention_delta_gdn_b200 import binding
    x = torch.zeros(1, 4, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        binding.gdn2_fwd(x, x, x, x, x, x)


def test_device_status_reports_a_cuda_error_without_a_device(L):
    """On a host without a usable GPU the status call returns GDN2_ERR_CUDA with a detail, not a crash."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present (the GPU tests cover the status call)")
    assert L.gdn2_device_status(None) == 4
    assert b"gdn2_device_status" in L.gdn2_last_error()


def test_maps_are_computed_on_the_tensor_core_path_only(L):
    from linear_attention_delta_gdn_b200 import binding
    for fn, nptr in ((L.gdn2_fwd_map, 8), (L.gdn2_bwd_map, 9)):
        rc = fn(*([None] * nptr), 1, 64, 2, 64, 64, 64, binding.GDN2_F32, None, 0, None)
        assert rc == binding.GDN2_ERR_UNSUPPORTED
        assert "tensor-core path" in L.gdn2_last_error().decode()
    # missing map outputs are refused before any launch
    rc = L.gdn2_fwd_map(*([None] * 8), 1, 64, 2, 128, 128, 64, binding.GDN2_BF16, None, 0, None)
    assert rc == binding.GDN2_ERR_INVALID
    rc = L.gdn2_state_affine(None, None, None, None, 1, 1, 128, 128, None)
    assert rc == binding.GDN2_ERR_INVALID


def test_reduced_gate_workspace_sizes_and_checks(L):
    """gdn2_beta_workspace_size: the GDN-2 workspace, then the broadcast gates (b, w and, for a scalar decay,
    log_alpha) and, for the backward, their gradients, each region 256-byte aligned. A forward that keeps its
    states takes the backward's GDN-2 size as its base, so the gates sit at the same offsets in both calls and one
    buffer of the backward's size serves both. Bad gates and missing pointers are refused before any launch."""
    from linear_attention_delta_gdn_b200.binding import gdn2_workspace_size as ws
    from linear_attention_delta_gdn_b200 import binding
    al = lambda x: (x + 255) // 256 * 256
    B, T, H, D = 4, 4096, 16, 128
    rows = B * T * H
    tile = al(rows * D * 2)
    for gate, ntiles in ((binding.GDN2_GATE_KDA, 2), (binding.GDN2_GATE_GDN, 3)):
        bws = lambda op: binding.gdn2_beta_workspace_size(gate, op, B, T, H, D, D, 64, binding.GDN2_BF16)
        assert bws(0) == al(ws(0, B, T, H, D, D, 64, 1)) + ntiles * tile
        assert bws(1) == al(ws(2, B, T, H, D, D, 64, 1)) + ntiles * tile
        assert bws(2) == al(ws(2, B, T, H, D, D, 64, 1)) + 2 * ntiles * tile
        assert bws(1) <= bws(2)
    assert binding.gdn2_beta_workspace_size(7, 2, B, T, H, D, D, 64, binding.GDN2_BF16) == 0
    assert binding.gdn2_beta_workspace_size(binding.GDN2_GATE_KDA, 2, B, T, H, 96, D, 64, binding.GDN2_BF16) == 0
    p = 1 << 20
    # gate 7 is neither KDA nor Gated DeltaNet; beta NULL
    rc = L.gdn2_beta_fwd(7, p, p, p, p, p, None, p, None, 1, 8, 1, 128, 128, 64, 1, 0, p, 1 << 30, None)
    assert rc == 1 and b"GDN2_GATE_KDA" in L.gdn2_last_error()
    rc = L.gdn2_beta_fwd(binding.GDN2_GATE_KDA, p, p, p, p, None, None, p, None, 1, 8, 1, 128, 128, 64, 1, 0, p,
                         1 << 30, None)
    assert rc == 1 and b"beta" in L.gdn2_last_error()
