"""Context parallelism, host side (CPU): the orchestration of linear_attention_delta_gdn_b200.context_parallel
run with the oracle standing in for the per-piece kernels, in one process and as gloo ranks (world size 2
and 3). Every result must equal the oracle's on the whole, uncut sequence: the maps are exact in fp64, so
the tolerance is rounding only. A wrong order of the chained maps, a piece that starts from the wrong
state or a gradient that ends on the wrong rank fails here."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from linear_attention_delta_gdn_b200 import context_parallel as cp
from linear_attention_delta_gdn_b200.inputs import make_inputs, to_f64

NAMES = ("q", "k", "v", "log_alpha", "b", "w")
GRADS = ("dq", "dk", "dv", "dlog_alpha", "db", "dw")


class OracleOps:
    """The per-piece operations, computed by the fp64 oracle on CPU tensors (test stand-in for the kernels)."""

    @staticmethod
    def _np(x):
        return None if x is None else x.detach().numpy()

    def fwd_map(self, q, k, v, la, b, w):
        B, T, H, Dk = q.shape
        z = np.zeros((B, T, H, Dk))
        eye = np.broadcast_to(np.eye(Dk), (B, H, Dk, Dk)).copy()
        _, M = oracle.fwd(*map(self._np, (q, k)), z, *map(self._np, (la, b)), z, S0=eye)   # no input: M I
        _, N = oracle.fwd(*map(self._np, (q, k, v, la, b, w)))                      # zero start: N
        return torch.from_numpy(M), torch.from_numpy(N)

    def bwd_map(self, q, k, v, la, b, w, dout):
        B, T, H, Dk = q.shape
        z = np.zeros((B, T, H, Dk))
        eye = np.broadcast_to(np.eye(Dk), (B, H, Dk, Dk)).copy()
        A = oracle.bwd(*map(self._np, (q, k)), z, *map(self._np, (la, b)), z, z, dST=eye)["dS0"]
        Bm = oracle.bwd(*map(self._np, (q, k, v, la, b, w, dout)))["dS0"]
        return torch.from_numpy(A), torch.from_numpy(Bm)

    def affine(self, M, N, S):
        out = N.clone()
        if S is not None:
            out += M @ S
        return out

    def fwd(self, q, k, v, la, b, w, S0):
        o, _ = oracle.fwd(*map(self._np, (q, k, v, la, b, w)), S0=self._np(S0))
        return torch.from_numpy(o)

    def bwd(self, q, k, v, la, b, w, dout, S0, dST):
        g = oracle.bwd(*map(self._np, (q, k, v, la, b, w, dout)), S0=self._np(S0), dST=self._np(dST))
        return {n: torch.from_numpy(g[n]) for n in GRADS + ("dS0",)}


def _problem(T, seed, P):
    x = make_inputs(2, T, 2, 8, 6, seed, "f32", with_do=True, with_S0=True)
    g = {n: torch.from_numpy(to_f64(t)) for n, t in x.items()}
    rng = np.random.Generator(np.random.PCG64(seed + 1))
    dSTs = [torch.from_numpy(rng.standard_normal((2, 2, 8, 6))) for _ in range(P)]
    return g, dSTs


def _cuts(T, P):
    return [(r * T) // P for r in range(P + 1)]


def _whole(g, dST):
    o, ST = oracle.fwd(*(g[n].numpy() for n in NAMES), S0=g["S0"].numpy())
    gr = oracle.bwd(*(g[n].numpy() for n in NAMES), g["dout"].numpy(), S0=g["S0"].numpy(), dST=dST.numpy())
    return o, ST, gr


def _close(a, b):
    a, b = np.asarray(a), np.asarray(b)
    assert np.linalg.norm(a - b) <= 1e-10 * max(np.linalg.norm(b), 1e-30), (np.abs(a - b).max(), np.abs(b).max())


@pytest.mark.parametrize("P,T", [(3, 50), (4, 64), (2, 1)])
def test_pieces_in_one_process_equal_the_whole_sequence(P, T):
    g, dSTs = _problem(T, 31, 1)
    cuts = _cuts(T, P)
    pieces = [tuple(g[n][:, cuts[r]:cuts[r + 1]].contiguous() for n in NAMES) for r in range(P)]
    douts = [g["dout"][:, cuts[r]:cuts[r + 1]].contiguous() for r in range(P)]
    ops = OracleOps()
    outs, starts, ST = cp.pieces_forward(pieces, g["S0"], ops)
    grads, dS0 = cp.pieces_backward(pieces, douts, starts, dSTs[0], ops)
    o_ref, ST_ref, gr = _whole(g, dSTs[0])
    _close(torch.cat(outs, 1), o_ref)
    _close(ST, ST_ref)
    _close(dS0, gr["dS0"])
    for n in GRADS:
        _close(torch.cat([x[n] for x in grads], 1), gr[n])


def test_maps_are_adjoint():
    """A piece's reverse map is the transpose of its forward map (A = M^T), and the maps reproduce the
    piece's end state from any start state."""
    g, _ = _problem(40, 7, 1)
    ops = OracleOps()
    args = tuple(g[n] for n in NAMES)
    M, N = ops.fwd_map(*args)
    A, _ = ops.bwd_map(*args, g["dout"])
    _close(A, M.transpose(-1, -2))
    _, ST = oracle.fwd(*(t.numpy() for t in args), S0=g["S0"].numpy())
    _close(M @ g["S0"] + N, ST)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, T, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g, dSTs = _problem(T, 77, world)
        c = _cuts(T, world)
        mine = {n: g[n][:, c[rank]:c[rank + 1]].contiguous().requires_grad_(True) for n in NAMES}
        S0 = g["S0"].clone().requires_grad_(True)
        o, ST = cp.context_parallel_gdn2(*(mine[n] for n in NAMES), S0, None, OracleOps())
        loss = (o * g["dout"][:, c[rank]:c[rank + 1]]).sum() + (ST * dSTs[rank]).sum()
        loss.backward()
        out[rank] = {"o": o.detach().numpy(), "ST": ST.detach().numpy(), "dS0": S0.grad.numpy(),
                     **{"d" + n: mine[n].grad.numpy() for n in NAMES}}
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,T", [(2, 70), (3, 45)])
def test_context_parallel_gloo(world, T):
    mgr = mp.Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, T, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    g, dSTs = _problem(T, 77, world)
    dST = sum(dSTs[1:], dSTs[0].clone())   # the loss is the sum of the ranks' losses
    o_ref, ST_ref, gr = _whole(g, dST)
    res = [out[r] for r in range(world)]
    _close(np.concatenate([x["o"] for x in res], 1), o_ref)
    for x in res:
        _close(x["ST"], ST_ref)   # every rank holds the whole sequence's final state
    _close(sum(x["dS0"] for x in res), gr["dS0"])
    assert all(np.all(x["dS0"] == 0) for x in res[1:])   # dS0 only on rank 0
    for n in NAMES:
        _close(np.concatenate([x["d" + n] for x in res], 1), gr["d" + n])
