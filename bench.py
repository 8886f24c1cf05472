"""Throughput benchmark of the Gated Delta Rule-2 operator (forward + gate-aware backward).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = gdn2_fwd (keeping the chunk-start states) + gdn2_bwd on one batch of
the 1.3B training-layer shape: B=4, H=16, T=4096, d_k=d_v=128, bf16 inputs,
fp32 state, chunk 64, synthetic seeded inputs resident in HBM. For N > 1 (one
process per GPU under torchrun) every rank runs its own batch: heads and batch
entries never interact, so there is no data-path collective (weak scaling).
Rank 0 prints one JSON line.

Besides the headline step, the line carries (rank 0, N=1):
  * ``configs``: the forward-only 1.3B layer (B=4, H=16, T=4K, no saved states)
    and the long forward (B=1, H=16, T=64K, random S0), each with ms, tokens/s
    and the fraction of its HBM roofline;
  * ``sweep``: fwd+bwd at a fixed 64K tokens per step for T = 1K..64K
    (B = 64K / T), the same figures per point;
  * ``decode``: 1024 in-place decode steps (batch 256, 16 heads, d = 128);
  * ``kda_overhead``: the KDA and Gated DeltaNet reductions through the same
    kernels at the headline shape, against the GDN-2 step;
  * ``layer_gates``: the layer's gate-activation kernels (forward and backward)
    at the headline shape, against the HBM roofline;
  * ``layer_step``: the whole layer (projections on cuBLAS, gate kernels, the
    operator) forward + backward at d_model = 2048, with the library's share;
  * ``context_parallel_maps``: a context-parallel rank's map kernels on one
    16K-token piece, beside that piece's own forward and fwd+bwd;
  * ``host_overhead``: host time to issue one fwd + bwd step through the binding
    at a one-chunk problem, beside its device time;
  * ``cpu_baseline``: the fp64 oracle timed on a bounded sample of the headline
    workload on the host cores, with the GPU outputs of those same sequences
    compared against the oracle's (relative L2, whole sample and worst head);
    the same leg gives every ``configs`` and ``sweep`` entry a ``parity`` object
    (o and the worst gradient of one sampled head against the oracle).

``--impl reference`` times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN-2 fwd+bwd tokens/s (H16 d128 T4K bf16, 1×B200); % of roofline"
WORKLOAD = "fwdbwd-bf16-b4h16t4096d128"

# Algorithmic work per token and head (C = 64, d = 128, bf16 tensors of 256 B per
# token and head). The step: the forward reads q, k, v, log_alpha, b, w and writes
# o (7 x 256 B); the backward reads the six inputs and dout and writes six
# gradients (13 x 256 B); plus the fp32 final state and dS0 per head. Per kernel:
#   chunk_fwd_kernel      7 x 256 B  (its inputs and o)
#   chunk_bwd_kernel     13 x 256 B  (all backward inputs and gradients: reverse pass and
#                                     per-chunk gradients run in the same launch)
# Flops: forward 180,224 per token and head (the chunk contractions), backward
# counted as twice the forward.
STEP_BYTES_PER_TOKEN_HEAD = 1792 + 3328
STEP_FLOPS_PER_TOKEN_HEAD = 3 * 180224
KERNEL_BYTES_PER_TOKEN_HEAD = {"chunk_fwd_kernel": 1792, "chunk_bwd_kernel": 3328,
                               "recurrent_fwd_kernel": 1792, "recurrent_bwd_kernel": 3328}
KERNEL_SOURCES = {"chunk_fwd_kernel": ["chunk_fwd.cu"], "chunk_bwd_kernel": ["chunk_bwd.cu"]}
COMMON_SOURCES = ["chunk_common.cuh", "tc.cuh", "common.cuh", "internal.h"]


def kernel_source_hash(kernel):
    """sha256 over the CUDA sources a kernel is built from (to tell whether recorded counters still apply)."""
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kernel, []) + COMMON_SOURCES:
        with open(os.path.join(ROOT, "linear_attention_delta_gdn_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic(kernel, token_heads):
    """DRAM bytes per launch from profiles/kernel_traffic.json, scaled to this launch, if still valid."""
    p = os.path.join(ROOT, "profiles", "kernel_traffic.json")
    if not os.path.exists(p) or kernel not in KERNEL_SOURCES:
        return None
    with open(p) as f:
        rec = json.load(f).get(kernel)
    if not rec or rec.get("source_sha256") != kernel_source_hash(kernel):
        return None
    return rec["dram_bytes_per_token_head"] * token_heads


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index, path):
        self.path, self.index, self.proc = path, index, None

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def make_host_inputs(rank, B=None, T=None):
    import dataclasses
    from linear_attention_delta_gdn_b200.inputs import WORKLOADS, make_inputs
    wl = WORKLOADS[WORKLOAD]
    if B or T:
        wl = dataclasses.replace(wl, name="%s-B%d-T%d" % (wl.name, B or wl.B, T or wl.T), B=B or wl.B, T=T or wl.T)
    from linear_attention_delta_gdn_b200.replicas import rank_seed
    return wl, make_inputs(wl.B, wl.T, wl.H, wl.Dk, wl.Dv, rank_seed(wl.seed, rank), wl.dtype, with_do=True)


def cpu_baseline(wl, x, budget_s=20.0, steps=1, gpu=None):
    """Time the fp64 oracle (fwd + bwd) on a bounded sample of the workload.

    ``gpu`` (optional): the GPU's outputs of the same step (o and the gradients, CPU tensors of the full
    workload); the sampled sequences are then compared against the oracle's results on them (relative L2
    over the sample and the worst single sequence). The forward output is compared at any sample length
    (it is causal); the gradients only when the sample covers the whole sequence."""
    import oracle
    from linear_attention_delta_gdn_b200.inputs import to_f64
    cores = oracle.threads()
    nheads = max(1, min(wl.B * wl.H, 2 * cores))
    T = wl.T
    # pick nheads (b, h) sequences, first T tokens
    heads = [(i // wl.H, i % wl.H) for i in range(nheads)]
    g = {n: to_f64(t) for n, t in x.items()}
    sub = {n: np.stack([g[n][b, :T, h] for b, h in heads])[:, :, None] for n in g}
    names = ("q", "k", "v", "log_alpha", "b", "w")
    # shrink the sample until one step fits the budget (estimate from a short probe)
    t0 = time.perf_counter()
    probe_T = min(T, 256)
    probe = {n: np.ascontiguousarray(a[:, :probe_T]) for n, a in sub.items()}
    oracle.fwd(*(probe[n] for n in names))
    oracle.bwd(*(probe[n] for n in names), dout=probe["dout"])
    est = (time.perf_counter() - t0) * T / probe_T
    if est > budget_s:
        T = max(probe_T, int(T * budget_s / est) // 64 * 64)
        sub = {n: np.ascontiguousarray(a[:, :T]) for n, a in sub.items()}
    times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        o_ref, _ = oracle.fwd(*(sub[n] for n in names))
        g_ref = oracle.bwd(*(sub[n] for n in names), dout=sub["dout"])
        times.append(time.perf_counter() - t0)
    dt = statistics.median(times)
    tokens = nheads * T / wl.H            # token = one position of the 16-head layer
    out = {"value": tokens / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
           "sample": "fp64 oracle fwd+bwd on %d of %d (batch, head) sequences x %d tokens; tokens = "
                     "sequences x tokens / %d heads" % (nheads, wl.B * wl.H, T, wl.H),
           "seconds": dt}
    if gpu is not None:
        def rel(a, r):
            return float(np.linalg.norm((a - r).ravel()) / max(np.linalg.norm(r.ravel()), 1e-300))

        refs = {"o": o_ref}
        if T == wl.T:
            refs.update({n: g_ref[n] for n in ("dq", "dk", "dv", "dlog_alpha", "db", "dw")})
        par = {}
        for n, r in refs.items():
            a = np.stack([to_f64(gpu[n][b, :T, h]) for b, h in heads])[:, :, None]
            par[n] = {"rel_l2": rel(a, r), "worst_sequence": max(rel(a[i], r[i]) for i in range(len(heads)))}
        out["parity"] = {"sequences": nheads, "tokens": T, "errors": par,
                         "tolerance": {"o": 2e-2, "gradients": 3e-2}}
    return out


def bench_decode(binding, dev, steps=1024, pool=64):
    """Time the decode workload: 1024 consecutive single-token steps, batch 256, 16 heads, d = 128,
    fp32 state updated in place, bf16 inputs. Step inputs cycle through a pool of `pool` distinct draws
    (the state traffic, not the input values, sets the time). Returns per-step time and HBM figures."""
    import torch
    from linear_attention_delta_gdn_b200.inputs import WORKLOADS, make_decode_stream
    wl = WORKLOADS["decode-bf16-b256h16d128x1024"]
    xs = make_decode_stream(pool, wl.B, wl.H, wl.Dk, wl.Dv, wl.seed, wl.dtype, device=dev)
    names = ("q", "k", "v", "log_alpha", "b", "w")
    S = xs["S0"].clone()
    o = torch.empty((wl.B, wl.H, wl.Dv), dtype=torch.bfloat16, device=dev)
    step_in = [[xs[n][i] for n in names] for i in range(pool)]
    for i in range(8):
        binding.gdn2_decode_step(*step_in[i % pool], S, o=o)
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    binding.trace_read()
    binding.trace_enable(True)
    a.record()
    for i in range(steps):
        binding.gdn2_decode_step(*step_in[i % pool], S, o=o)
    b.record()
    binding.trace_enable(False)
    torch.cuda.synchronize(dev)
    kern = binding.trace_read().get("decode_kernel", (steps, 0.0))
    ms = a.elapsed_time(b) / steps
    kern_ms = kern[1] / max(1, kern[0])
    heads = wl.B * wl.H
    state_bytes = heads * wl.Dk * wl.Dv * 4
    io_bytes = heads * (4 * wl.Dk + 3 * wl.Dv) * 2       # q, k, log_alpha, b, v, w in; o out
    alg = 2 * state_bytes + io_bytes
    pk = peaks()
    return {"workload": wl.name, "steps": steps, "ms_per_step": ms, "kernel_ms": kern_ms,
            "alg_bytes_per_step": alg, "achieved_gbs": alg / (kern_ms / 1e3) / 1e9,
            "frac_of_hbm": alg / (kern_ms / 1e3) / 1e9 / pk["hbm_gbs"], "peak_gbs": pk["hbm_gbs"],
            "inputs": "%d-step input pool cycled; state evolves over all %d steps" % (pool, steps),
            "launches": kern[0]}


# One sampled (batch, head) sequence of each extra measurement: its inputs and the GPU's outputs, copied to the host
# during the measurement; the CPU-baseline leg compares them with the oracle (sample_parity).
SAMPLES = []


def keep_sample(entry, inputs, outputs, b, h, with_do):
    """Store sequence (b, h) of a measurement's inputs and outputs (host copies) for sample_parity."""
    names = ("q", "k", "v", "log_alpha", "b", "w") + (("dout",) if with_do else ())
    x = {n: inputs[n][b, :, h].detach().cpu() for n in names}
    if inputs.get("S0") is not None and entry.get("with_S0"):
        x["S0"] = inputs["S0"][b, h].detach().cpu()
    y = {n: t[b, :, h].detach().cpu() for n, t in outputs.items() if t is not None and t.dim() == 4}
    SAMPLES.append((entry, x, y, [b, h]))


def sample_parity():
    """Oracle results of every kept sample; each measurement's entry gets ``parity``: relative L2 of o (and of
    every gradient when the measurement ran the backward) on its sampled head."""
    import oracle
    from linear_attention_delta_gdn_b200.inputs import to_f64
    names = ("q", "k", "v", "log_alpha", "b", "w")

    def rel(a, r):
        return float(np.linalg.norm((a - r).ravel()) / max(np.linalg.norm(r.ravel()), 1e-300))

    for entry, x, y, bh in SAMPLES:
        f = {n: to_f64(t)[None, :, None] for n, t in x.items() if n != "S0"}
        S0 = to_f64(x["S0"])[None, None] if "S0" in x else None
        o_ref, _ = oracle.fwd(*(f[n] for n in names), S0=S0)
        par = {"sampled_head": bh, "o": rel(to_f64(y["o"])[None, :, None], o_ref)}
        if "dout" in f:
            g = oracle.bwd(*(f[n] for n in names), dout=f["dout"], S0=S0)
            par["gradients_worst"] = max(rel(to_f64(y[n])[None, :, None], g[n])
                                         for n in ("dq", "dk", "dv", "dlog_alpha", "db", "dw"))
        par["tolerance"] = {"o": 2e-2, "gradients": 3e-2}
        entry["parity"] = par
    SAMPLES.clear()


def device_inputs(B, T, H, D, seed, with_do, dev):
    """Token inputs drawn on the device with the recipe's distributions (seeded torch generator): the long
    and swept workloads hold up to ~2 GB of token tensors."""
    import torch
    from linear_attention_delta_gdn_b200.inputs import make_decode_stream
    names = ("q", "k", "v", "log_alpha", "b", "w")
    xs = make_decode_stream(T, B, H, D, D, seed, "bf16", device=dev)   # [T, B, H, D] -> [B, T, H, D]
    d = {n: xs[n].permute(1, 0, 2, 3).contiguous() for n in names}
    d["S0"] = xs["S0"]
    del xs
    if with_do:
        gen = torch.Generator(device=dev)
        gen.manual_seed(seed + 1)
        d["dout"] = torch.randn((B, T, H, D), generator=gen, device=dev).to(torch.bfloat16)
    return d


def timed_ms(fn, steps, dev, warmup=3):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize(dev)
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        fn()
    e.record()
    torch.cuda.synchronize(dev)
    return a.elapsed_time(e) / steps


def fwdbwd_point(binding, dev, B, T, H, steps, seed):
    """fwd (keeping the states) + bwd at one (B, T): ms per step, tokens/s and fraction of the HBM roofline."""
    import torch
    D = 128
    names = ("q", "k", "v", "log_alpha", "b", "w")
    pk = peaks()
    d = device_inputs(B, T, H, D, seed, True, dev)
    ws = torch.empty(binding.gdn2_workspace_size(binding.GDN2_OP_BWD, B, T, H, D, D, 64, binding.GDN2_BF16),
                     dtype=torch.uint8, device=dev)
    o = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
    ST = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    grads = {n: torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
             for n in ("dq", "dk", "dlog_alpha", "db", "dv", "dw")}
    grads["dS0"] = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)

    def step():
        binding.gdn2_fwd(*(d[n] for n in names), None, save_states=True, ws=ws, o=o, ST=ST)
        binding.gdn2_bwd(*(d[n] for n in names), d["dout"], None, None, states_saved=True, ws=ws, grads=grads)

    ms = timed_ms(step, steps, dev)
    alg = B * T * H * STEP_BYTES_PER_TOKEN_HEAD + 2 * B * H * D * D * 4
    out = {"workload": "fwdbwd-bf16-b%dh%dt%dd128" % (B, H, T), "B": B, "T": T, "H": H, "ms_per_step": ms,
           "tokens_per_s": B * T / (ms / 1e3), "frac_of_roofline": alg / (ms / 1e3) / 1e9 / pk["hbm_gbs"],
           "status": binding.gdn2_device_status()}
    keep_sample(out, d, dict(o=o, **{n: grads[n] for n in ("dq", "dk", "dv", "dlog_alpha", "db", "dw")}),
                B - 1, H // 2, True)
    del d, ws, o, ST, grads
    torch.cuda.empty_cache()
    return out


def measure_configs(binding, dev, args, fwd_inputs):
    """The forward-only 1.3B layer (the headline inputs, no saved states) and the long forward (B=1, H=16,
    T=64K, random S0): ms, tokens/s and the fraction of each one's HBM roofline (its inputs read, o written,
    the fp32 states read and written)."""
    import torch
    D = 128
    names = ("q", "k", "v", "log_alpha", "b", "w")
    pk = peaks()
    out = {}
    B, T, H = fwd_inputs["q"].shape[0], fwd_inputs["q"].shape[1], fwd_inputs["q"].shape[2]
    ws = torch.empty(binding.gdn2_workspace_size(binding.GDN2_OP_FWD, B, T, H, D, D, 64, binding.GDN2_BF16),
                     dtype=torch.uint8, device=dev)
    o = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
    ST = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    ms = timed_ms(lambda: binding.gdn2_fwd(*(fwd_inputs[n] for n in names), None, ws=ws, o=o, ST=ST),
                  max(5, args.steps), dev)
    alg = B * T * H * KERNEL_BYTES_PER_TOKEN_HEAD["chunk_fwd_kernel"] + B * H * D * D * 4
    out["fwd-bf16-b%dh%dt%dd128" % (B, H, T)] = {
        "mode": "forward only (no saved states), zero S0, o and S_T returned", "ms": ms,
        "tokens_per_s": B * T / (ms / 1e3), "frac_of_roofline": alg / (ms / 1e3) / 1e9 / pk["hbm_gbs"],
        "status": binding.gdn2_device_status()}
    keep_sample(out["fwd-bf16-b%dh%dt%dd128" % (B, H, T)], fwd_inputs, {"o": o}, B - 1, H // 2, False)
    del ws, o, ST

    B, T = 1, 65536
    d = device_inputs(B, T, H, D, 4000, False, dev)
    ws = torch.empty(binding.gdn2_workspace_size(binding.GDN2_OP_FWD, B, T, H, D, D, 64, binding.GDN2_BF16),
                     dtype=torch.uint8, device=dev)
    o = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
    ST = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    ms = timed_ms(lambda: binding.gdn2_fwd(*(d[n] for n in names), d["S0"], ws=ws, o=o, ST=ST),
                  max(5, args.steps // 2), dev)
    alg = B * T * H * KERNEL_BYTES_PER_TOKEN_HEAD["chunk_fwd_kernel"] + 2 * B * H * D * D * 4
    out["fwd-bf16-b1h16t65536d128-s0"] = {
        "mode": "forward, random S0 ~ N(0, 0.02^2), o and S_T returned", "ms": ms,
        "tokens_per_s": B * T / (ms / 1e3), "frac_of_roofline": alg / (ms / 1e3) / 1e9 / pk["hbm_gbs"],
        "status": binding.gdn2_device_status(), "with_S0": True}
    keep_sample(out["fwd-bf16-b1h16t65536d128-s0"], d, {"o": o}, 0, H // 2, False)
    del d, ws, o, ST
    torch.cuda.empty_cache()
    return out


def measure_reductions(binding, dev, d, args, gdn2_ms):
    """The pages' reductions through the same kernels at the headline shape: KDA (b = w = beta * 1) and Gated
    DeltaNet (also a scalar decay), fwd (keeping the states) + bwd, against the GDN-2 step. Both run the chunk
    kernels' scalar-gate instances (beta, and Gated DeltaNet's decay, read per token; dbeta and the decay's
    gradient summed in the gradient units). `overhead_of_gdn2` is gdn2_ms / reduced_ms - 1."""
    import torch
    names = ("q", "k", "v")
    B, T, H, D = d["q"].shape
    gen = torch.Generator(device=dev)
    gen.manual_seed(6000)
    beta = torch.sigmoid(torch.randn((B, T, H), generator=gen, device=dev)).to(torch.bfloat16)
    log_a = (-torch.nn.functional.softplus(torch.randn((B, T, H), generator=gen, device=dev)) / 16.0).to(torch.bfloat16)
    out = {"gdn2_ms": gdn2_ms}
    for name, gate, la in (("kda", binding.GDN2_GATE_KDA, d["log_alpha"]), ("gated_deltanet", binding.GDN2_GATE_GDN, log_a)):
        ws = torch.empty(binding.gdn2_beta_workspace_size(gate, binding.GDN2_OP_BWD, B, T, H, D, D, 64,
                                                          binding.GDN2_BF16), dtype=torch.uint8, device=dev)
        o = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
        ST = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
        grads = {"dq": torch.empty_like(d["q"]), "dk": torch.empty_like(d["k"]), "dv": torch.empty_like(d["v"]),
                 "dlog_alpha": torch.empty_like(la), "dbeta": torch.empty_like(beta),
                 "dS0": torch.empty((B, H, D, D), dtype=torch.float32, device=dev)}

        def step():
            binding.gdn2_beta_fwd(gate, *(d[n] for n in names), la, beta, None, save_states=True, ws=ws, o=o, ST=ST)
            binding.gdn2_beta_bwd(gate, *(d[n] for n in names), la, beta, d["dout"], None, None, states_saved=True,
                                  ws=ws, grads=grads)

        ms = timed_ms(step, max(5, args.steps), dev)
        out[name + "_ms"] = ms
        out["overhead_of_gdn2_over_" + name] = gdn2_ms / ms - 1.0
        out[name + "_status"] = binding.gdn2_device_status()
        del ws, o, ST, grads
    out["note"] = ("KDA and Gated DeltaNet run the chunk kernels' scalar-gate instances: no b or w tiles (nor a "
                   "log_alpha tile for Gated DeltaNet's scalar decay); dbeta (and dlog_a) summed in the gradient "
                   "units")
    torch.cuda.empty_cache()
    return out


def measure_layer_gates(binding, dev, args, B, T, H, D=128):
    """The layer's gate-activation kernels at the headline shape: z [B, T, H, 6 D] bf16 drawn on the device.
    Algorithmic bytes per token-head: forward z in + six outputs = 2 x 6D x 2 B; backward z and six gradients
    in, dz out = 3 x 6D x 2 B."""
    import torch
    pk = peaks()
    gen = torch.Generator(device=dev)
    gen.manual_seed(7000)
    z = torch.randn((B, T, H, 6 * D), generator=gen, device=dev).to(torch.bfloat16)
    bias = torch.full((H, D), -4.0, device=dev)
    outs = binding.gdn2_layer_gates_fwd(z, D, D, bias)
    steps = max(5, args.steps)
    f_ms = timed_ms(lambda: binding.gdn2_layer_gates_fwd(z, D, D, bias), steps, dev)
    b_ms = timed_ms(lambda: binding.gdn2_layer_gates_bwd(z, *outs, D, D, bias), steps, dev)
    th = B * T * H
    fb, bb = th * 2 * 6 * D * 2, th * 3 * 6 * D * 2
    out = {"workload": "layer-gates-bf16-b%dh%dt%dd%d" % (B, H, T, D), "fwd_ms": f_ms, "bwd_ms": b_ms,
           "fwd_frac_of_hbm": fb / (f_ms / 1e3) / 1e9 / pk["hbm_gbs"],
           "bwd_frac_of_hbm": bb / (b_ms / 1e3) / 1e9 / pk["hbm_gbs"], "status": binding.gdn2_device_status()}
    del z, outs
    torch.cuda.empty_cache()
    return out


def measure_layer_step(binding, dev, args, B, T, H, D=128):
    """The layer around the operator (Gdn2Layer: input projection on cuBLAS, gate kernels, the operator,
    output projection) forward + backward through autograd at d_model = H * D, bf16: ms per step, tokens/s, the
    projections' tensor-core throughput and the library kernels' share of the step (trace)."""
    import torch
    from linear_attention_delta_gdn_b200.layer import Gdn2Layer
    pk = peaks()
    torch.manual_seed(9000)
    dm = H * D
    layer = Gdn2Layer(dm, H, D, D, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(9001)
    x = torch.randn((B, T, dm), generator=gen, device=dev).to(torch.bfloat16).requires_grad_(True)
    dy = torch.randn((B, T, dm), generator=gen, device=dev).to(torch.bfloat16)

    def step():
        y, _ = layer(x)
        y.backward(dy)

    steps = max(3, args.steps // 4)
    for _ in range(3):
        step()
    torch.cuda.synchronize(dev)
    binding.trace_read()
    binding.trace_enable(True)
    ms = timed_ms(step, steps, dev, warmup=0)
    binding.trace_enable(False)
    kern = {k: v[1] / steps for k, v in binding.trace_read().items()}   # device ms per step of each library kernel
    ntok = B * T
    proj_flop = 3 * 2 * ntok * dm * (H * (4 * D + 2 * D) + dm)   # in + out projections, forward and two backward GEMMs
    lib_ms = sum(kern.values())
    out = {"workload": "layer-bf16-b%dt%dh%dd%d-dmodel%d" % (B, T, H, D, dm), "ms": ms, "tokens_per_s": ntok / (ms / 1e3),
           "library_kernels_ms": kern, "library_share": lib_ms / ms,
           "projection_tflops": proj_flop / ((ms - lib_ms) / 1e3) / 1e12 if ms > lib_ms else None,
           "peak_bf16_tflops": pk.get("bf16_tflops"), "status": binding.gdn2_device_status(),
           "note": "projections are cuBLAS GEMMs through torch.matmul (their throughput is over the step time the "
                   "library's kernels leave); the gates, the operator and their backward are the library's kernels"}
    del layer, x, dy
    torch.cuda.empty_cache()
    return out


def measure_host_overhead(binding, dev, calls=200):
    """Host time per call of the C ABI through the binding (gdn2_fwd keeping its states + gdn2_bwd on them) at a
    one-chunk problem, B=1 H=1 T=64, where the device work is a few microseconds: the wall time to issue `calls`
    steps back to back (no synchronisation inside; workspace, outputs and gradients preallocated), beside the
    device time per step from CUDA events. The entry points cache the tensor maps (per pointer and shape) and the
    launch facts, so a repeated call does argument checks, a flag memset and the launches."""
    import torch
    B, T, H, D = 1, 64, 1, 128
    d = device_inputs(B, T, H, D, 4242, True, dev)
    names = ("q", "k", "v", "log_alpha", "b", "w")
    ws = torch.empty(binding.gdn2_workspace_size(binding.GDN2_OP_BWD, B, T, H, D, D, 64, binding.GDN2_BF16),
                     dtype=torch.uint8, device=dev)
    o = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
    ST = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    grads = {n: torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
             for n in ("dq", "dk", "dv", "dlog_alpha", "db", "dw")}
    grads["dS0"] = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)

    def step():
        binding.gdn2_fwd(*(d[n] for n in names), None, save_states=True, ws=ws, o=o, ST=ST)
        binding.gdn2_bwd(*(d[n] for n in names), d["dout"], None, None, states_saved=True, ws=ws, grads=grads)

    for _ in range(10):
        step()
    torch.cuda.synchronize(dev)
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    t0 = time.perf_counter()
    for _ in range(calls):
        step()
    t1 = time.perf_counter()
    e.record()
    torch.cuda.synchronize(dev)
    return {"workload": "fwdbwd-bf16-b1h1t64d128", "steps": calls,
            "host_us_per_step": (t1 - t0) / calls * 1e6, "device_us_per_step": a.elapsed_time(e) / calls * 1e3,
            "status": binding.gdn2_device_status(),
            "note": "host time to issue one fwd (keeping its states) + bwd through the Python binding and the C ABI, "
                    "and the device time per step when the steps run back to back"}


def measure_context_maps(binding, dev, args, T=16384, H=16, D=128):
    """Per-rank cost of context parallelism on one piece (B = 1, T tokens, H heads): the piece's forward and
    reverse maps against its own forward and fwd+bwd (what a rank runs anyway)."""
    import torch
    names = ("q", "k", "v", "log_alpha", "b", "w")
    d = device_inputs(1, T, H, D, 8000, True, dev)
    steps = max(3, args.steps // 4)
    ws_map = torch.empty(binding.gdn2_workspace_size(binding.GDN2_OP_MAP, 1, T, H, D, D, 64, binding.GDN2_BF16),
                         dtype=torch.uint8, device=dev)
    x = [d[n] for n in names]
    fm = timed_ms(lambda: binding.gdn2_fwd_map(*x, ws=ws_map), steps, dev)
    bm = timed_ms(lambda: binding.gdn2_bwd_map(*x, d["dout"], ws=ws_map), steps, dev)
    M, N = binding.gdn2_fwd_map(*x, ws=ws_map)
    af = timed_ms(lambda: binding.gdn2_state_affine(M, N, d["S0"]), steps, dev)
    ws = torch.empty(binding.gdn2_workspace_size(binding.GDN2_OP_BWD, 1, T, H, D, D, 64, binding.GDN2_BF16),
                     dtype=torch.uint8, device=dev)
    f = timed_ms(lambda: binding.gdn2_fwd(*x, d["S0"], save_states=True, ws=ws), steps, dev)
    fb = timed_ms(lambda: (binding.gdn2_fwd(*x, d["S0"], save_states=True, ws=ws),
                           binding.gdn2_bwd(*x, d["dout"], d["S0"], None, states_saved=True, ws=ws)), steps, dev)
    out = {"piece": "b1h%dt%dd%d" % (H, T, D), "fwd_map_ms": fm, "bwd_map_ms": bm, "state_affine_ms": af,
           "piece_fwd_ms": f, "piece_fwdbwd_ms": fb, "status": binding.gdn2_device_status(),
           "note": "a rank of a context-parallel step runs its maps, one all-gather, P - 1 state_affine chain steps "
                   "and its piece's forward (and backward); one GPU per call here, so no multi-GPU time"}
    del d, ws, ws_map, M, N
    torch.cuda.empty_cache()
    return out


SWEEP_TOKENS = 65536
SWEEP_T = (1024, 2048, 4096, 8192, 16384, 32768, 65536)


def measure_sweep(binding, dev, args):
    """fwd+bwd throughput against sequence length at a fixed 64K tokens per step (B = 64K / T), H = 16."""
    return [fwdbwd_point(binding, dev, SWEEP_TOKENS // T, T, 16, max(3, args.steps // 4), 3000 + T)
            for T in SWEEP_T]


def run_sweep(args):
    """The sweep and the extra configs alone, one JSON line each (1 GPU)."""
    import torch
    from linear_attention_delta_gdn_b200 import binding, build
    build.build()
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    for pt in measure_sweep(binding, dev, args):
        print(json.dumps(dict(mode="sweep", **pt)), flush=True)
    d = device_inputs(4, 4096, 16, 128, 5000, False, dev)
    for name, r in measure_configs(binding, dev, args, d).items():
        print(json.dumps(dict(mode="config", workload=name, **r)), flush=True)
    return 0


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl, x = make_host_inputs(0)
    budget = float(os.environ.get("GDN2_REF_BUDGET_S", "8"))
    for _ in range(args.warmup):
        pass  # the oracle has no warm-up state; warm-up steps are not repeated on the CPU
    cb = cpu_baseline(wl, x, budget_s=budget, steps=max(1, args.steps))
    line = {"metric": METRIC, "impl": "reference", "value": cb["value"], "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": None, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": wl.B, "T": wl.T, "H": wl.H, "Dk": wl.Dk, "Dv": wl.Dv,
                       "chunk": wl.chunk, "global_batch": wl.B, "seq_len": wl.T, "parallelism": "host threads"},
            "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")},
            "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--no-decode", action="store_true", help="skip the decode-step measurement")
    ap.add_argument("--no-extra", action="store_true", help="skip the extra configs and the length sweep")
    ap.add_argument("--B", type=int, default=None, help="override the batch size (small profiling cases)")
    ap.add_argument("--T", type=int, default=None, help="override the sequence length (small profiling cases)")
    ap.add_argument("--sweep", action="store_true",
                    help="instead of the headline line: the length sweep (fwd+bwd at 64K tokens per step, "
                         "T = 1K..64K) and the extra configs, one JSON line each (1 GPU)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.sweep:
        return run_sweep(args)

    import torch
    import torch.distributed as dist
    from linear_attention_delta_gdn_b200 import binding, build

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    L = binding.lib()

    wl, xh = make_host_inputs(rank, args.B, args.T)
    B, T, H, Dk, Dv, chunk = wl.B, wl.T, wl.H, wl.Dk, wl.Dv, wl.chunk
    names = ("q", "k", "v", "log_alpha", "b", "w")
    pinned = {n: t.pin_memory() for n, t in xh.items()}
    d = {n: t.to(dev, non_blocking=True) for n, t in pinned.items()}
    o = torch.empty((B, T, H, Dv), dtype=torch.bfloat16, device=dev)
    ST = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=dev)
    grads = {n: torch.empty((B, T, H, Dk), dtype=torch.bfloat16, device=dev) for n in ("dq", "dk", "dlog_alpha", "db")}
    grads.update({n: torch.empty((B, T, H, Dv), dtype=torch.bfloat16, device=dev) for n in ("dv", "dw")})
    grads["dS0"] = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=dev)
    ws = torch.empty(binding.gdn2_workspace_size(binding.GDN2_OP_BWD, B, T, H, Dk, Dv, chunk, binding.GDN2_BF16),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(inp, o_=o, grads_=grads):
        binding.gdn2_fwd(*(inp[n] for n in names), None, chunk=chunk, save_states=True, ws=ws, o=o_, ST=ST)
        binding.gdn2_bwd(*(inp[n] for n in names), inp["dout"], None, None, chunk=chunk, states_saved=True,
                         ws=ws, grads=grads_)

    for _ in range(max(3, args.warmup)):
        step(d)
    torch.cuda.synchronize(dev)

    # ---- device-timed region: inputs resident in HBM (470 MB per step, larger than L2)
    # nvidia-smi samples of the timed region (summarised in the JSON line); GDN2_BENCH_LOG_DIR moves the CSV
    clock_log = os.path.join(os.environ.get("GDN2_BENCH_LOG_DIR", os.path.join(ROOT, "bench_logs")),
                             "bench_clocks_rank%d.csv" % rank)
    os.makedirs(os.path.dirname(clock_log), exist_ok=True)
    binding.trace_read()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local, clock_log) as clocks:
        time.sleep(0.3)
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        binding.trace_enable(True)
        start.record(stream)
        for i in range(args.steps):
            step(d)
        end.record(stream)
        binding.trace_enable(False)
        torch.cuda.synchronize(dev)
    kernels = binding.trace_read()       # {name: (launches, summed device ms)} of the timed region
    if world > 1:
        dist.barrier()
    from linear_attention_delta_gdn_b200.replicas import aggregate_tokens_per_s, max_over_ranks
    total_ms = max_over_ranks(start.elapsed_time(end), dist, dev)
    ms_per_step = total_ms / args.steps
    tokens_per_step = B * T
    value = aggregate_tokens_per_s(world, tokens_per_step, ms_per_step)

    # ---- end to end through host buffers: every step copies its inputs in from pinned host memory, runs fwd + bwd
    # and copies o and the six gradients back. A training loop's pipeline: two device buffer sets and three streams
    # (copy in, compute, copy out), so that one step's copies overlap the neighbouring steps' kernels and the two
    # copy directions overlap each other.
    gnames = ("dq", "dk", "dv", "dlog_alpha", "db", "dw")
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = (o.numel() + sum(grads[n].numel() for n in gnames)) * o.element_size()
    dsets = [d, {n: torch.empty_like(t) for n, t in d.items()}]
    osets = [(o, grads), (torch.empty_like(o), {n: torch.empty_like(t) for n, t in grads.items()})]
    host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in [o] + [grads[n] for n in gnames]]
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    nsteps = max(1, args.e2e_steps)
    ev = {k: [torch.cuda.Event() for _ in range(nsteps)] for k in ("in", "cmp", "out")}
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e_start.record(s_in)
    for i in range(nsteps):
        k = i % 2
        if i >= 2:
            s_in.wait_event(ev["cmp"][i - 2])    # the set's inputs have been consumed
        with torch.cuda.stream(s_in):
            for n in pinned:
                dsets[k][n].copy_(pinned[n], non_blocking=True)
            ev["in"][i].record(s_in)
        s_cmp.wait_event(ev["in"][i])
        if i >= 2:
            s_cmp.wait_event(ev["out"][i - 2])   # the set's outputs have been copied out
        with torch.cuda.stream(s_cmp):
            step(dsets[k], osets[k][0], osets[k][1])
            ev["cmp"][i].record(s_cmp)
        s_out.wait_event(ev["cmp"][i])
        with torch.cuda.stream(s_out):
            for h_, t in zip(host_out, [osets[k][0]] + [osets[k][1][n] for n in gnames]):
                h_.copy_(t, non_blocking=True)
            ev["out"][i].record(s_out)
    e_end.record(s_out)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end) / nsteps, dist, dev)
    e2e_value = aggregate_tokens_per_s(world, tokens_per_step, e2e_ms)

    # ---- roofline of the dominant kernel (device time summed over the timed region)
    pk = peaks()
    th = B * T * H
    dom = max(kernels, key=lambda k: kernels[k][1])
    n_launch, dom_ms = kernels[dom]
    per_launch_s = dom_ms / n_launch / 1e3
    alg_bytes = th * KERNEL_BYTES_PER_TOKEN_HEAD.get(dom, STEP_BYTES_PER_TOKEN_HEAD)
    achieved = alg_bytes / per_launch_s / 1e9
    traffic = recorded_traffic(dom, th)
    roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "traffic": traffic, "peak_source": pk["source"],
                "alg_bytes_per_launch": alg_bytes, "launch_ms": per_launch_s * 1e3,
                "kernels_ms_per_step": {k: v[1] / args.steps for k, v in kernels.items()},
                "step_alg_bytes": th * STEP_BYTES_PER_TOKEN_HEAD + 2 * B * H * Dk * Dv * 4,
                "step_frac": (th * STEP_BYTES_PER_TOKEN_HEAD + 2 * B * H * Dk * Dv * 4)
                / (ms_per_step / 1e3) / 1e9 / pk["hbm_gbs"]}
    launches_in_timed_region = sum(v[0] for v in kernels.values())

    decode = configs = sweep = None
    full = args.B is None and args.T is None
    if not args.no_decode and full:
        decode = bench_decode(binding, dev)
    reductions = layer_gates = cp_maps = layer_step = host = None
    if not args.no_extra and full and world == 1:
        configs = measure_configs(binding, dev, args, d)
        sweep = measure_sweep(binding, dev, args)
        reductions = measure_reductions(binding, dev, d, args, ms_per_step)
        layer_gates = measure_layer_gates(binding, dev, args, B, T, H)
        layer_step = measure_layer_step(binding, dev, args, B, T, H)
        cp_maps = measure_context_maps(binding, dev, args)
        host = measure_host_overhead(binding, dev)

    line = None
    if rank == 0:
        cb = None
        if not args.no_cpu_baseline and world == 1:
            gpu_out = {"o": o.cpu()}
            gpu_out.update({n: grads[n].cpu() for n in ("dq", "dk", "dv", "dlog_alpha", "db", "dw")})
            cb = cpu_baseline(wl, xh, gpu=gpu_out)
            cb = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample", "parity")}
            sample_parity()   # one sampled head of each extra measurement against the oracle
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": max(3, args.warmup), "ms_per_step": ms_per_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": wl.name, "B": B, "T": T, "H": H, "Dk": Dk, "Dv": Dv, "chunk": chunk,
                           "global_batch": world * B, "seq_len": T,
                           "parallelism": "dp%d (independent batches, no collective)" % world,
                           "l2": "inputs larger than L2 (%.0f MB read per step)" % (h2d / 1e6),
                           "kernels": sorted(kernels)},
                "roofline": roofline, "cpu_baseline": cb, "clocks": clocks.summary(),
                "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h},
                "gpu_launches": launches_in_timed_region,
                "decode": decode, "configs": configs, "sweep": sweep, "kda_overhead": reductions,
                "layer_gates": layer_gates, "layer_step": layer_step, "context_parallel_maps": cp_maps,
                "host_overhead": host}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
