"""Replicas across processes (gloo, world size 2, CPU): each rank draws its own batch,
the slowest rank's time sets the job time, and every rank's result is the oracle's on
its own inputs (heads/batches never interact, so no data-path collective is needed)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from linear_attention_delta_gdn_b200.inputs import make_inputs, to_f64
        from linear_attention_delta_gdn_b200.replicas import aggregate_tokens_per_s, max_over_ranks, rank_seed
        x = make_inputs(1, 24, 2, 8, 8, rank_seed(5, rank), "f32", with_do=True)
        g = {n: to_f64(t) for n, t in x.items()}
        o, ST = oracle.fwd(*(g[n] for n in ("q", "k", "v", "log_alpha", "b", "w")))
        # fake per-rank step times: the job time must be the slowest rank's
        ms = max_over_ranks(10.0 + 5.0 * rank, dist)
        gathered = [None] * world
        dist.all_gather_object(gathered, (float(g["q"].sum()), float(o.sum())))
        out[rank] = (ms, aggregate_tokens_per_s(world, 24, ms), gathered)
    finally:
        dist.destroy_process_group()


def test_two_replicas_gloo():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    (ms0, v0, g0), (ms1, v1, g1) = out[0], out[1]
    assert ms0 == ms1 == 15.0
    assert v0 == v1 == pytest.approx(2 * 24 / 0.015)
    assert g0 == g1
    assert g0[0][0] != g0[1][0]            # the two ranks drew different batches


def test_single_process_helpers():
    from linear_attention_delta_gdn_b200.replicas import aggregate_tokens_per_s, max_over_ranks, rank_seed
    assert rank_seed(1002, 0) == 1002 and rank_seed(1002, 3) != rank_seed(1002, 2)
    assert max_over_ranks(3.5) == 3.5
    assert aggregate_tokens_per_s(1, 16384, 2.0) == pytest.approx(8.192e6)
    assert np.isfinite(aggregate_tokens_per_s(8, 16384, 1.6))
