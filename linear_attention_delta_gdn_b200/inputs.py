"""Seeded synthetic inputs for the Gated Delta Rule-2 operator.

This module only draws inputs. It holds none of the operator's arithmetic and
serves both the CUDA path and the fp64 oracle, which receive the same values.

Distributions (the shapes of the 1.3B training layer in "Gated DeltaNet-2:
Decoupling Erase and Write in Linear Attention", GitHub README training recipe:
16 heads, d_k = d_v = 128, sequence length 4K):
  q, k       ~ N(0, 1), then L2-normalised over d_k per token and head
  v          ~ N(0, 1)
  log_alpha  = -softplus(N(0, 1)) / 16          (channel-wise decay, log form)
  b          = sigmoid(N(0, 1)) over d_k          (erase gate in [0, 1])
  w          = sigmoid(N(0, 1)) over d_v          (write gate in [0, 1])
  dout       ~ N(0, 1)                            (upstream gradient)
  S0         ~ N(0, 0.02^2), float32              (initial state)
Draw order q, k, v, log_alpha, b, w, dout, S0 from numpy PCG64(seed); values
are then rounded to the workload dtype (float32 or bfloat16, round-to-nearest-
even). Decode streams (many single-token steps) are drawn with torch's
generator on the target device because they hold billions of values.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

_TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: operator mode, shapes, dtype and seed."""
    name: str
    mode: str            # "fwd", "fwd_bwd" or "decode"
    dtype: str           # "f32" or "bf16": dtype of q, k, v, gates, o and the token gradients
    B: int
    T: int               # sequence length; decode: number of consecutive steps
    H: int
    Dk: int
    Dv: int
    chunk: int
    with_S0: bool
    seed: int
    note: str = field(default="", compare=False)


WORKLOADS = {
    w.name: w
    for w in (
        Workload("fwd-f32-b1h2t256d64", "fwd", "f32", 1, 256, 2, 64, 64, 64, False, 1000,
                 "forward, fp32, zero initial state"),
        Workload("fwd-bf16-b4h16t4096d128", "fwd", "bf16", 4, 4096, 16, 128, 128, 64, False, 1001,
                 "forward, one 1.3B-shape training layer"),
        Workload("fwdbwd-bf16-b4h16t4096d128", "fwd_bwd", "bf16", 4, 4096, 16, 128, 128, 64, False, 1002,
                 "forward + gate-aware backward, one 1.3B-shape training layer"),
        Workload("fwd-bf16-b1h16t65536d128-s0", "fwd", "bf16", 1, 65536, 16, 128, 128, 64, True, 1003,
                 "long-sequence forward with a random initial state"),
        Workload("decode-bf16-b256h16d128x1024", "decode", "bf16", 256, 1024, 16, 128, 128, 64, True, 1004,
                 "1024 consecutive single-token decode steps, fp32 state in place"),
    )
}

#: the workload the throughput benchmark times
BENCH_WORKLOAD = "fwdbwd-bf16-b4h16t4096d128"


def _round(x: np.ndarray, dtype: str) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(_TORCH_DT[dtype])


def _softplus(x):
    return np.logaddexp(0.0, x)


def _sigmoid(x):
    return 0.5 * (1.0 + np.tanh(0.5 * x))


def make_inputs(B, T, H, Dk, Dv, seed, dtype="f32", with_do=False, with_S0=False):
    """Draw one batch of sequence inputs. Returns CPU torch tensors.

    Keys: q, k, log_alpha, b [B,T,H,Dk]; v, w [B,T,H,Dv] in ``dtype``;
    optionally dout [B,T,H,Dv] in ``dtype`` and S0 [B,H,Dk,Dv] float32.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    out = {}

    def normal(shape):
        return rng.standard_normal(size=shape)

    for name in ("q", "k"):
        x = normal((B, T, H, Dk))
        x /= np.linalg.norm(x, axis=-1, keepdims=True)
        out[name] = _round(x, dtype)
    out["v"] = _round(normal((B, T, H, Dv)), dtype)
    out["log_alpha"] = _round(-_softplus(normal((B, T, H, Dk))) / 16.0, dtype)
    out["b"] = _round(_sigmoid(normal((B, T, H, Dk))), dtype)
    out["w"] = _round(_sigmoid(normal((B, T, H, Dv))), dtype)
    if with_do:
        out["dout"] = _round(normal((B, T, H, Dv)), dtype)
    if with_S0:
        out["S0"] = torch.from_numpy((0.02 * normal((B, H, Dk, Dv))).astype(np.float32))
    return out


def make_reduced_gates(B, T, H, seed, dtype="f32"):
    """Gates of the two reductions (KDA, Gated DeltaNet), drawn with the recipe's distributions but one value
    per head and token: beta = sigmoid(N(0, 1)) and log_a = -softplus(N(0, 1)) / 16, both [B, T, H], from
    numpy PCG64(seed), in that order."""
    rng = np.random.Generator(np.random.PCG64(seed))
    beta = _sigmoid(rng.standard_normal(size=(B, T, H)))
    log_a = -_softplus(rng.standard_normal(size=(B, T, H))) / 16.0
    return {"beta": _round(beta, dtype), "log_a": _round(log_a, dtype)}


def make_workload_inputs(wl: Workload):
    """Inputs of a sequence workload (``mode`` fwd or fwd_bwd)."""
    return make_inputs(wl.B, wl.T, wl.H, wl.Dk, wl.Dv, wl.seed, wl.dtype,
                       with_do=(wl.mode == "fwd_bwd"), with_S0=wl.with_S0)


def make_decode_stream(steps, B, H, Dk, Dv, seed, dtype="bf16", device="cpu"):
    """Draw ``steps`` consecutive single-token inputs and an initial state.

    Same distributions as :func:`make_inputs`, drawn with a seeded torch
    generator on ``device`` (q, k, v, log_alpha, b, w then S0). Token tensors are
    [steps, B, H, D] in ``dtype``; S0 is [B, H, Dk, Dv] float32.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    tdt = _TORCH_DT[dtype]

    def normal(shape):
        return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)

    out = {}
    for name in ("q", "k"):
        x = normal((steps, B, H, Dk))
        out[name] = (x / x.norm(dim=-1, keepdim=True)).to(tdt)
    out["v"] = normal((steps, B, H, Dv)).to(tdt)
    out["log_alpha"] = (-torch.nn.functional.softplus(normal((steps, B, H, Dk))) / 16.0).to(tdt)
    out["b"] = torch.sigmoid(normal((steps, B, H, Dk))).to(tdt)
    out["w"] = torch.sigmoid(normal((steps, B, H, Dv))).to(tdt)
    out["S0"] = 0.02 * normal((B, H, Dk, Dv))
    return out


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a float32/bfloat16 tensor (for the oracle)."""
    return t.detach().to("cpu", torch.float64).numpy()
