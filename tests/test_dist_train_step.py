"""The data-parallel training step (lq.dp_train_step) with two gloo ranks on CPU.

Each rank runs the layer's training step on its own half of the tokens through a CPU stand-in
layer whose forward_backward is the gradient oracle (oracle.backward) of those tokens; the ranks
then sum their weight gradients and their QB statistics.  The loss is a sum over all tokens, so
every rank must end with the weight gradients of one rank that saw every token (to fp64 rounding
of the two-term sums) and with the bias of one rank that saw every token (exactly), while dL/dx
stays each rank's own rows.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import datagen
import oracle
import oracle.backward as ob
import latent_routing_quantile_b200 as lq

SHAPE = datagen.LayerShape("dp_train", 96, 64, 32, 32, 4, 32, 48, "f32", seed=41, offset_var=0.5, beta=0.1)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleTrainLayer:
    """A CPU stand-in for lq.Layer with the calls dp_train_step makes: forward_backward (the
    oracle's output and gradients of this rank's tokens, gradients as fp64 tensors) and the
    statistics calls of dp_qb_update."""

    def __init__(self, w, b):
        self.w, self.b = w, np.asarray(b, dtype=np.float64)

    def forward_backward(self, x, dy, weights, record_stats=False, grads=None, stream=None):
        g = ob.layer_backward(x, self.w, self.b, SHAPE.k, dy)
        r = oracle.layer_routing(x, self.w, self.b, SHAPE.k)
        self._hist = torch.from_numpy(oracle.score_histogram(r["s"]).astype(np.int32))
        self._n = torch.tensor([x.shape[0]], dtype=torch.int64)
        y = oracle.layer_forward(x, self.w, self.b, SHAPE.k)["y"]
        return y, {n: torch.from_numpy(np.ascontiguousarray(v)) for n, v in g.items() if n != "idx"}

    def hist(self, stream=None):
        return self._hist.clone(), self._n.clone()

    def set_hist(self, hist, n, stream=None):
        self._hist, self._n = hist.clone(), n.clone()

    def qb_update(self, beta, literal=False, sign_rule=False, stream=None):
        self.b = oracle.qb_update(self.b, self._hist.numpy().astype(np.int64), int(self._n.item()), SHAPE.k, beta,
                                  literal=literal)


def _inputs(rows=None):
    x = datagen.tokens(SHAPE, rows=rows)
    dy = datagen.output_grad(SHAPE, seed=SHAPE.seed + 100)
    if rows is not None:
        dy = dy[torch.as_tensor(rows)]
    return x, dy


def _rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = {k: oracle.f64(v) for k, v in datagen.layer_weights(SHAPE, gain="random").items()}
        rows = np.arange(SHAPE.T)[rank::world]
        x, dy = _inputs(rows)
        layer = OracleTrainLayer(w, np.zeros(SHAPE.E))
        _, g = lq.dp_train_step(layer, x, dy, None, beta=SHAPE.beta)
        out[rank] = ({n: t.numpy() for n, t in g.items()}, layer.b, rows)
    finally:
        dist.destroy_process_group()


def test_two_ranks_sum_to_the_single_rank_gradients_and_bias():
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
    w = {k: oracle.f64(v) for k, v in datagen.layer_weights(SHAPE, gain="random").items()}
    x, dy = _inputs()
    g_all = ob.layer_backward(x, w, np.zeros(SHAPE.E), SHAPE.k, dy)
    r_all = oracle.layer_routing(x, w, np.zeros(SHAPE.E), SHAPE.k)
    b_all = oracle.qb_update(np.zeros(SHAPE.E), oracle.score_histogram(r_all["s"]), SHAPE.T, SHAPE.k, SHAPE.beta)
    for r in range(2):
        g, b, rows = res[r]
        for n in g:
            if n == "x":
                np.testing.assert_allclose(g[n], g_all["x"][rows], rtol=1e-12, atol=1e-15)
            else:
                np.testing.assert_allclose(g[n], g_all[n], rtol=1e-10, atol=1e-13 * np.max(np.abs(g_all[n])))
        assert np.array_equal(b, b_all)
    # one rank's gradients alone are not the batch's
    g_half = ob.layer_backward(*_inputs(np.arange(0, SHAPE.T, 2))[:1], w, np.zeros(SHAPE.E), SHAPE.k,
                               _inputs(np.arange(0, SHAPE.T, 2))[1])
    assert not np.allclose(g_half["w_up"], g_all["w_up"])
