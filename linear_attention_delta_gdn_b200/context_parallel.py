"""Context (sequence) parallelism: one sequence cut along T into pieces, piece r on rank r.

The state update of the Gated Delta Rule-2 (GitHub README introduction; arXiv abstract: a fixed-size
recurrent state) is affine in the state, ``S_t = (I - k_t (b_t*k_t)^T) Diag(alpha_t) S_{t-1} + k_t
(w_t*v_t)^T``. A piece therefore maps its start state to its end state as ``S_end = M S_start + N``, and
its backward maps the end gradient to the start gradient as ``dS_start = A dS_end + B``. The only data
that crosses ranks is those maps (fp32, ``[B, H, Dk, Dk]`` and ``[B, H, Dk, Dv]`` per rank):

forward   each rank computes its piece's (M, N) with ``gdn2_fwd_map``; one all-gather; every rank
          chains the maps of the pieces before it into its start state (``gdn2_state_affine``) and runs
          ``gdn2_fwd`` on its piece from there. Chaining all maps gives the sequence's final state.
backward  each rank computes (A, B) of its piece with ``gdn2_bwd_map``; one all-gather (which also sums
          the final-state gradients of the ranks); every rank chains the maps of the pieces after it into
          its end gradient and runs ``gdn2_bwd`` on its piece from its saved start state.

Conventions: ``S0`` is replicated (the same tensor value on every rank). The final state ``ST`` is
returned on every rank; the loss is the sum of the ranks' losses, so the ranks' ``dST`` are summed.
``dS0`` is the whole sequence's gradient on rank 0 and zero on the others, so that a sum over ranks
(as data-parallel gradient reduction does) gives it once. The per-piece work is the library's kernels
(``PieceOps``); the chaining here is host orchestration of device calls, nothing is computed in Python.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch

from . import binding


class PieceOps:
    """The per-piece operations: the CUDA library (bf16, Dk = Dv = 128 for the maps)."""

    def __init__(self, chunk: int = 64):
        self.chunk = chunk

    def fwd_map(self, q, k, v, la, b, w):
        return binding.gdn2_fwd_map(q, k, v, la, b, w, chunk=self.chunk)

    def bwd_map(self, q, k, v, la, b, w, dout):
        return binding.gdn2_bwd_map(q, k, v, la, b, w, dout, chunk=self.chunk)

    def affine(self, M, N, S):
        return binding.gdn2_state_affine(M, N, S)

    def fwd(self, q, k, v, la, b, w, S0):
        return binding.gdn2_fwd(q, k, v, la, b, w, S0, chunk=self.chunk, want_state=False)[0]

    def bwd(self, q, k, v, la, b, w, dout, S0, dST):
        return binding.gdn2_bwd(q, k, v, la, b, w, dout, S0, dST, chunk=self.chunk, want_dS0=False)


def chain_forward(Ms: Sequence[torch.Tensor], Ns: Sequence[torch.Tensor], S0: Optional[torch.Tensor],
                  ops) -> Tuple[List[Optional[torch.Tensor]], torch.Tensor]:
    """Start states of every piece (``None``: zero, for piece 0 without ``S0``) and the final state."""
    starts: List[Optional[torch.Tensor]] = []
    S = S0
    for M, N in zip(Ms, Ns):
        starts.append(S)
        S = ops.affine(M, N, S)
    return starts, S


def chain_backward(As: Sequence[torch.Tensor], Bs: Sequence[torch.Tensor], dST: Optional[torch.Tensor],
                   ops) -> Tuple[List[Optional[torch.Tensor]], torch.Tensor]:
    """End gradients of every piece (``None``: zero, for the last piece without ``dST``) and dS0."""
    ends: List[Optional[torch.Tensor]] = [None] * len(As)
    E = dST
    for j in range(len(As) - 1, -1, -1):
        ends[j] = E
        E = ops.affine(As[j], Bs[j], E)
    return ends, E


def _group_info(group):
    import torch.distributed as dist
    return dist.get_rank(group), dist.get_world_size(group)


def _all_gather_flat(parts: Sequence[torch.Tensor], group) -> List[List[torch.Tensor]]:
    """All-gather several tensors in one collective; returns, per rank, the tensors in ``parts``' shapes."""
    import torch.distributed as dist
    flat = torch.cat([p.reshape(-1) for p in parts])
    world = dist.get_world_size(group)
    bufs = [torch.empty_like(flat) for _ in range(world)]
    dist.all_gather(bufs, flat, group=group)
    out = []
    for buf in bufs:
        xs, o = [], 0
        for p in parts:
            xs.append(buf[o:o + p.numel()].view(p.shape))
            o += p.numel()
        out.append(xs)
    return out


def cp_forward(q, k, v, la, b, w, S0=None, group=None, ops=None):
    """Forward of this rank's piece. Returns ``(o, S_start, ST)``: the piece's output, its start state
    (``None`` for a zero state; keep it for :func:`cp_backward`) and the whole sequence's final state."""
    ops = ops or PieceOps()
    rank, world = _group_info(group)
    M, N = ops.fwd_map(q, k, v, la, b, w)
    gathered = _all_gather_flat([M, N], group)
    starts, ST = chain_forward([g[0] for g in gathered], [g[1] for g in gathered], S0, ops)
    o = ops.fwd(q, k, v, la, b, w, starts[rank])
    return o, starts[rank], ST


def cp_backward(q, k, v, la, b, w, dout, S_start, dST=None, group=None, ops=None):
    """Backward of this rank's piece from its saved start state. Returns the token gradients of the piece
    (dq, dk, dv, dlog_alpha, db, dw) and ``dS0`` (the sequence's on rank 0, zero elsewhere)."""
    ops = ops or PieceOps()
    rank, world = _group_info(group)
    A, Bm = ops.bwd_map(q, k, v, la, b, w, dout)
    dST_r = torch.zeros_like(Bm) if dST is None else dST.to(Bm.dtype)
    gathered = _all_gather_flat([A, Bm, dST_r], group)
    dST_sum = gathered[0][2].clone()
    for g in gathered[1:]:
        dST_sum += g[2]
    ends, dS0 = chain_backward([g[0] for g in gathered], [g[1] for g in gathered], dST_sum, ops)
    grads = dict(ops.bwd(q, k, v, la, b, w, dout, S_start, ends[rank]))
    grads["dS0"] = dS0 if rank == 0 else torch.zeros_like(dS0)
    return grads


class ContextParallelGDN2(torch.autograd.Function):
    """autograd wrapper of :func:`cp_forward` / :func:`cp_backward` (one collective each way)."""

    @staticmethod
    def forward(ctx, q, k, v, la, b, w, S0, group, ops):
        o, S_start, ST = cp_forward(q, k, v, la, b, w, S0, group, ops)
        ctx.save_for_backward(q, k, v, la, b, w, S_start if S_start is not None else torch.empty(0))
        ctx.has_start = S_start is not None
        ctx.has_S0 = S0 is not None
        ctx.group, ctx.ops = group, ops
        return o, ST

    @staticmethod
    def backward(ctx, do, dST):
        q, k, v, la, b, w, S_start = ctx.saved_tensors
        g = cp_backward(q, k, v, la, b, w, do.contiguous(), S_start if ctx.has_start else None,
                        None if dST is None else dST.contiguous(), ctx.group, ctx.ops)
        return (g["dq"], g["dk"], g["dv"], g["dlog_alpha"], g["db"], g["dw"],
                g["dS0"] if ctx.has_S0 else None, None, None)


def context_parallel_gdn2(q, k, v, la, b, w, S0=None, group=None, ops=None):
    """Differentiable Gated Delta Rule-2 over a sequence cut across the ranks of ``group`` (piece r on
    rank r, in order). Returns ``(o_piece, ST)``."""
    return ContextParallelGDN2.apply(q, k, v, la, b, w, S0, group, ops)


def pieces_forward(pieces, S0=None, ops=None):
    """All pieces of a sequence in one process (the same steps without a collective): returns the
    outputs, the start states and the final state."""
    ops = ops or PieceOps()
    maps = [ops.fwd_map(*p) for p in pieces]
    starts, ST = chain_forward([m[0] for m in maps], [m[1] for m in maps], S0, ops)
    outs = [ops.fwd(*p, S) for p, S in zip(pieces, starts)]
    return outs, starts, ST


def pieces_backward(pieces, douts, starts, dST=None, ops=None):
    """All pieces' backward in one process: returns the per-piece gradient dicts and dS0."""
    ops = ops or PieceOps()
    maps = [ops.bwd_map(*p, d) for p, d in zip(pieces, douts)]
    ends, dS0 = chain_backward([m[0] for m in maps], [m[1] for m in maps], dST, ops)
    grads = [dict(ops.bwd(*p, d, S, E)) for p, d, S, E in zip(pieces, douts, starts, ends)]
    return grads, dS0
