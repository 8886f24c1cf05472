"""Host-side helpers of bench.py (CPU): the sampled-head parity of the extra measurements reproduces zero error
when the "GPU outputs" are the oracle's own, including a start state; the roofline peaks come from the measured
file or the stated fallback; the source hash that guards the recorded DRAM traffic changes with the sources."""
import json
import os

import numpy as np
import torch

import bench
import oracle
from linear_attention_delta_gdn_b200.inputs import make_inputs, to_f64

NAMES = ("q", "k", "v", "log_alpha", "b", "w")
GRADS = ("dq", "dk", "dv", "dlog_alpha", "db", "dw")


def test_sample_parity_of_exact_outputs_is_zero():
    x = make_inputs(2, 150, 3, 16, 16, 5, "f32", with_do=True, with_S0=True)
    f = {n: to_f64(t) for n, t in x.items()}
    o, _ = oracle.fwd(*(f[n] for n in NAMES), S0=f["S0"])
    g = oracle.bwd(*(f[n] for n in NAMES), f["dout"], S0=f["S0"])
    outs = {"o": torch.from_numpy(o), **{n: torch.from_numpy(g[n]) for n in GRADS}}
    with_bwd = {"with_S0": True}
    bench.keep_sample(with_bwd, x, outs, 1, 2, True)
    fwd_only = {}
    o0, _ = oracle.fwd(*(f[n] for n in NAMES))
    bench.keep_sample(fwd_only, x, {"o": torch.from_numpy(o0)}, 0, 1, False)
    bench.sample_parity()
    assert with_bwd["parity"]["sampled_head"] == [1, 2]
    assert with_bwd["parity"]["o"] < 1e-12 and with_bwd["parity"]["gradients_worst"] < 1e-12
    assert fwd_only["parity"]["o"] < 1e-12 and "gradients_worst" not in fwd_only["parity"]
    assert bench.SAMPLES == []


def test_sample_parity_sees_a_wrong_head():
    x = make_inputs(1, 64, 2, 16, 16, 6, "f32", with_do=False)
    f = {n: to_f64(t) for n, t in x.items()}
    o, _ = oracle.fwd(*(f[n] for n in NAMES))
    e = {}
    bench.keep_sample(e, x, {"o": torch.from_numpy(o[:, :, ::-1].copy())}, 0, 0, False)   # heads swapped
    bench.sample_parity()
    assert e["parity"]["o"] > 0.1


def test_peaks_measured_or_fallback():
    pk = bench.peaks()
    assert pk["source"] in ("measured", "fallback")
    assert pk["hbm_gbs"] > 1000 and pk["bf16_tflops"] > 100
    p = os.path.join(bench.ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        assert pk["source"] == "measured" and pk["hbm_gbs"] == json.load(open(p))["hbm_gbs"]


def test_traffic_record_follows_the_sources():
    h = bench.kernel_source_hash("chunk_bwd_kernel")
    assert len(h) == 64 and h != bench.kernel_source_hash("chunk_fwd_kernel")
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "kernel_traffic.json")))
    for k in ("chunk_fwd_kernel", "chunk_bwd_kernel"):
        t = bench.recorded_traffic(k, 1000)
        if rec[k]["source_sha256"] == bench.kernel_source_hash(k):
            assert np.isclose(t, 1000 * rec[k]["dram_bytes_per_token_head"])
        else:   # sources changed since the capture: the bench reports no traffic rather than a stale figure
            assert t is None
