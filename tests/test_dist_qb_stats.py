"""The data-parallel QB exchange step with two gloo ranks on CPU.

Each rank routes its own half of the tokens (oracle), builds its histogram, and the ranks sum
histograms and token counts with sum_qb_statistics.  The summed histogram must equal the
histogram of all tokens on one rank exactly (integer sums are order-free), and both ranks must
then compute the same bias update as a single rank that saw every token (the per-rank bias drift
of the e-book's capsule 27 Bug 2 cannot happen).
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
        s = oracle.layer_routing(x, w, b, SHAPE.k)["s"]
        hist = torch.from_numpy(oracle.score_histogram(s).astype(np.int32))
        n = torch.tensor([len(rows)], dtype=torch.int64)
        lq.sum_qb_statistics(hist, n)
        b1 = oracle.qb_update(b, hist.numpy().astype(np.int64), int(n.item()), SHAPE.k, SHAPE.beta)
        out[rank] = (hist.numpy(), int(n.item()), b1)
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
    s_all = oracle.layer_routing(datagen.tokens(SHAPE), w, np.zeros(SHAPE.E), SHAPE.k)["s"]
    hist_all = oracle.score_histogram(s_all)
    b_all = oracle.qb_update(np.zeros(SHAPE.E), hist_all, SHAPE.T, SHAPE.k, SHAPE.beta)
    for r in range(2):
        hist, n, b1 = res[r]
        assert n == SHAPE.T
        assert np.array_equal(hist, hist_all)
        assert np.array_equal(b1, b_all)
