"""The data-parallel exchange step of the bias update with two gloo ranks on CPU.

Each rank routes its own half of the tokens (oracle), builds its histogram and expert loads, and
the ranks sum histograms, token counts and loads with sum_qb_statistics.  The sums must equal the
statistics of all tokens on one rank exactly (integer sums are order-free), and both ranks must
then compute the same QB and sign-rule updates as a single rank that saw every token (the
per-rank bias drift of the e-book's capsule 27 Bug 2 cannot happen).
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import datagen
import oracle
import latent_routing_quantile_b200 as lq

SHAPE = datagen.LayerShape("dp", 512, 128, 64, 64, 4, 64, 0, "f32", seed=31, offset_var=0.5, beta=0.1)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = datagen.layer_weights(SHAPE)
        rows = np.arange(SHAPE.T)[rank::world]
        x = datagen.tokens(SHAPE, rows=rows)
        b = np.zeros(SHAPE.E)
        r = oracle.layer_routing(x, w, b, SHAPE.k)
        hist = torch.from_numpy(oracle.score_histogram(r["s"]).astype(np.int32))
        n = torch.tensor([len(rows)], dtype=torch.int64)
        load = torch.from_numpy(oracle.expert_counts(r["idx"], SHAPE.E).astype(np.int64))
        lq.sum_qb_statistics(hist, n, load)
        b1 = oracle.qb_update(b, hist.numpy().astype(np.int64), int(n.item()), SHAPE.k, SHAPE.beta)
        b2 = oracle.sign_rule_update(b, load.numpy(), 1e-2)
        out[rank] = (hist.numpy(), int(n.item()), b1, load.numpy(), b2)
    finally:
        dist.destroy_process_group()


def test_two_ranks_sum_to_the_single_rank_statistics():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=300)
            assert p.exitcode == 0
        res = dict(out)
    w = datagen.layer_weights(SHAPE)
    r_all = oracle.layer_routing(datagen.tokens(SHAPE), w, np.zeros(SHAPE.E), SHAPE.k)
    hist_all = oracle.score_histogram(r_all["s"])
    load_all = oracle.expert_counts(r_all["idx"], SHAPE.E)
    b_all = oracle.qb_update(np.zeros(SHAPE.E), hist_all, SHAPE.T, SHAPE.k, SHAPE.beta)
    b_sign = oracle.sign_rule_update(np.zeros(SHAPE.E), load_all, 1e-2)
    for r in range(2):
        hist, n, b1, load, b2 = res[r]
        assert n == SHAPE.T
        assert np.array_equal(hist, hist_all)
        assert np.array_equal(b1, b_all)
        assert np.array_equal(load, load_all)
        assert np.array_equal(b2, b_sign)
    # one rank's own loads would have moved some bias the other way (Bug 2 is not hypothetical)
    half = oracle.expert_counts(oracle.layer_routing(datagen.tokens(SHAPE, rows=np.arange(0, SHAPE.T, 2)), w,
                                                     np.zeros(SHAPE.E), SHAPE.k)["idx"], SHAPE.E)
    assert not np.array_equal(oracle.sign_rule_update(np.zeros(SHAPE.E), half, 1e-2), b_sign)
