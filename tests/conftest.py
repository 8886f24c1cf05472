"""pytest configuration: the ``gpu`` marker and shared helpers."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running")


def rel_l2(x, ref):
    """||x - ref||_2 / ||ref||_2 over the whole tensor (absolute L2 if ref is zero)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    num = np.linalg.norm((x - ref).ravel())
    den = np.linalg.norm(ref.ravel())
    return num / den if den > 0 else num


def worst_head_rel_l2(x, ref, state=False):
    """Largest per-(batch, head) relative L2 error: token tensors are [B, T, H, D], states [B, H, Dk, Dv].

    A whole-tensor figure can hide one bad head (or one bad stretch of chunks of one head); this one
    cannot. Heads whose reference is zero use the absolute L2, as rel_l2 does."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    worst = 0.0
    if state:
        for b in range(ref.shape[0]):
            for h in range(ref.shape[1]):
                worst = max(worst, rel_l2(x[b, h], ref[b, h]))
    else:
        if ref.shape[1] == 0:
            return 0.0
        for b in range(ref.shape[0]):
            for h in range(ref.shape[2]):
                worst = max(worst, rel_l2(x[b, :, h], ref[b, :, h]))
    return worst


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(autouse=True)
def _debug_build_index_checks(request):
    """Under the debug build (environment GDN2_DEBUG set), every GPU test ends with no failed index check."""
    yield
    if os.environ.get("GDN2_DEBUG", "") in ("", "0") or request.node.get_closest_marker("gpu") is None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    from linear_attention_delta_gdn_b200 import binding
    if binding.gdn2_device_status() != binding.GDN2_OK:
        assert "index check" not in binding.last_error(), binding.last_error()
