"""Device-side waits of the tensor-core kernels are bounded and reported to the host.

Every wait inside the kernels (an mbarrier, a ready flag written by another CTA) gives up after ~2 s; the
kernel records it, skips the rest of its work and exits, and gdn2_device_status reports GDN2_ERR_TIMEOUT.
The failure is made on the host: GDN2_TEST_SKIP_PRODUCERS leaves out the producer launch of the forward's
two-launch form, so no ready flag of the consumers is ever set. The context stays usable afterwards.
"""
import os
import re

import pytest
import torch

from linear_attention_delta_gdn_b200 import binding
from linear_attention_delta_gdn_b200.inputs import make_inputs

NAMES = ("q", "k", "v", "log_alpha", "b", "w")


def _inputs(B, T, H, seed):
    x = make_inputs(B, T, H, 128, 128, seed=seed, dtype="bf16", with_do=True)
    return {n: t.cuda() for n, t in x.items()}


@pytest.mark.gpu
def test_status_ok_after_a_training_step():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    d = _inputs(2, 200, 3, seed=31)
    ws = torch.empty(binding.gdn2_workspace_size(binding.GDN2_OP_BWD, 2, 200, 3, 128, 128, 64, binding.GDN2_BF16),
                     dtype=torch.uint8, device="cuda")
    binding.gdn2_fwd(*(d[n] for n in NAMES), None, save_states=True, ws=ws)
    binding.gdn2_bwd(*(d[n] for n in NAMES), d["dout"], None, None, states_saved=True, ws=ws)
    assert binding.gdn2_device_status() == binding.GDN2_OK, binding.last_error()


@pytest.mark.gpu
def test_flag_that_nothing_sets_times_out_and_is_reported():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    d = _inputs(1, 128, 1, seed=32)
    assert binding.gdn2_device_status() == binding.GDN2_OK   # a clean record to start from
    os.environ["GDN2_TEST_SKIP_PRODUCERS"] = "1"
    try:
        binding.gdn2_fwd(*(d[n] for n in NAMES), None)   # the consumers wait ~2 s on a flag, then give up
        status = binding.gdn2_device_status()
    finally:
        del os.environ["GDN2_TEST_SKIP_PRODUCERS"]
    assert status == binding.GDN2_ERR_TIMEOUT
    msg = binding.last_error()
    fwd_bits = int(re.search(r"chunk_fwd_kernel bits (0x[0-9a-f]+)", msg).group(1), 16)
    assert fwd_bits & 4, msg   # the ready-flag wait
    # the record is cleared and the context still runs the operator correctly
    assert binding.gdn2_device_status() == binding.GDN2_OK
    o1, s1 = binding.gdn2_fwd(*(d[n] for n in NAMES), None)
    os.environ["GDN2_NO_COOPERATIVE"] = "1"
    try:
        o2, s2 = binding.gdn2_fwd(*(d[n] for n in NAMES), None)
    finally:
        del os.environ["GDN2_NO_COOPERATIVE"]
    assert binding.gdn2_device_status() == binding.GDN2_OK
    assert torch.equal(o1, o2) and torch.equal(s1, s2)
