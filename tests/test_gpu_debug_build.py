"""The debug build of the library (compiled with -DGDN2_DEBUG: the kernels' index checks record a failure for
gdn2_device_status and skip the guarded access, never trap) runs the small-shape GPU suites in a child
process with GDN2_DEBUG set: the same tests must pass, and no index check may fire (conftest checks the
device status after every GPU test under that variable). The full-size workload tests stay with the release
build; the device-status tests, which make waits give up on purpose, are left out."""
import os
import subprocess
import sys

import pytest
import torch

from conftest import ROOT

pytestmark = pytest.mark.gpu


def test_small_suites_pass_on_the_debug_build():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_attention_delta_gdn_b200 import build
    lib = build.build(debug=True)
    assert lib.endswith("libgdn2_debug.so") and os.path.exists(lib)
    env = dict(os.environ, GDN2_DEBUG="1")
    files = ["tests/test_gpu_parity.py", "tests/test_gpu_edge_cases.py", "tests/test_gpu_varlen.py",
             "tests/test_gpu_reductions.py", "tests/test_gpu_context_parallel.py"]
    cmd = [sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider", *files,
           "-k", "not workload and not other_shapes"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=2400)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    # the child loaded the debug library
    probe = subprocess.run([sys.executable, "-c", "from linear_attention_delta_gdn_b200 import binding; "
                            "print(binding.lib()._name)"], cwd=ROOT, env=env, capture_output=True, text=True)
    assert probe.stdout.strip().endswith("libgdn2_debug.so"), probe.stdout + probe.stderr
