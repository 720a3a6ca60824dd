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


class OracleLayer:
    """A stand-in for lq.Layer on the CPU with the calls dp_qb_update makes (hist, load, set_hist,
    set_load, qb_update): its statistics are those of the oracle's routing of this rank's tokens,
    and its update is the oracle's.  It records the order of the calls."""

    def __init__(self, x, w, b):
        r = oracle.layer_routing(x, w, b, SHAPE.k)
        self._hist = torch.from_numpy(oracle.score_histogram(r["s"]).astype(np.int32))
        self._n = torch.tensor([x.shape[0]], dtype=torch.int64)
        self._load = torch.from_numpy(oracle.expert_counts(r["idx"], SHAPE.E).astype(np.int64))
        self.b = np.asarray(b, dtype=np.float64)
        self.calls = []

    def hist(self, stream=None):
        self.calls.append("hist")
        return self._hist.clone(), self._n.clone()

    def load(self, stream=None):
        self.calls.append("load")
        return self._load.clone()

    def set_hist(self, hist, n, stream=None):
        self.calls.append("set_hist")
        self._hist, self._n = hist.clone(), n.clone()

    def set_load(self, load, stream=None):
        self.calls.append("set_load")
        self._load = load.clone()

    def qb_update(self, beta, literal=False, sign_rule=False, stream=None):
        self.calls.append("qb_update")
        if sign_rule:
            self.b = oracle.sign_rule_update(self.b, self._load.numpy(), beta)
        else:
            self.b = oracle.qb_update(self.b, self._hist.numpy().astype(np.int64), int(self._n.item()), SHAPE.k, beta,
                                      literal=literal)


def _rank_update(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = datagen.layer_weights(SHAPE)
        x = datagen.tokens(SHAPE, rows=np.arange(SHAPE.T)[rank::world])
        res = {}
        for rule in ("qb", "sign"):
            layer = OracleLayer(x, w, np.zeros(SHAPE.E))
            lq.dp_qb_update(layer, SHAPE.beta if rule == "qb" else 1e-2, sign_rule=(rule == "sign"))
            res[rule] = (layer.b, layer.calls)
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_dp_qb_update_sums_before_the_update_on_every_rank():
    """lq.dp_qb_update, the step bench.py runs between ranks: each rank reads its statistics,
    the ranks sum them, each sets the sums back and updates.  Driven on two gloo ranks through
    a CPU stand-in layer, both ranks end with the bias of one rank that saw every token, for
    QB and for the sign rule, and the calls come in the order read -> sum -> set -> update."""
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_update, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=300)
            assert p.exitcode == 0
        res = dict(out)
    w = datagen.layer_weights(SHAPE)
    r_all = oracle.layer_routing(datagen.tokens(SHAPE), w, np.zeros(SHAPE.E), SHAPE.k)
    b_qb = oracle.qb_update(np.zeros(SHAPE.E), oracle.score_histogram(r_all["s"]), SHAPE.T, SHAPE.k, SHAPE.beta)
    b_sign = oracle.sign_rule_update(np.zeros(SHAPE.E), oracle.expert_counts(r_all["idx"], SHAPE.E), 1e-2)
    for r in range(2):
        assert np.array_equal(res[r]["qb"][0], b_qb)
        assert np.array_equal(res[r]["sign"][0], b_sign)
        assert res[r]["qb"][1] == ["hist", "set_hist", "qb_update"]
        assert res[r]["sign"][1] == ["hist", "load", "set_hist", "set_load", "qb_update"]
    # a rank that updated from its own statistics alone would have another bias
    own = OracleLayer(datagen.tokens(SHAPE, rows=np.arange(0, SHAPE.T, 2)), w, np.zeros(SHAPE.E))
    own.qb_update(SHAPE.beta)
    assert not np.array_equal(own.b, b_qb)
