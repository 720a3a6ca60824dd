"""The layer backward on the GPU (lmoe_forward_backward) against the CPU oracle of the gradients
(oracle.backward.layer_backward, float64), through the C ABI (needs a B200).

Tolerance.  The backward's products take bf16 operands and accumulate in fp32.  Along the
longest chain (dy -> dL/dz -> dL/do -> dL/dp -> dL/dh -> dL/dx_hat -> dL/dx) every gradient that
feeds a product is rounded to bf16 once, and the recomputed pre-activations, the gathered rows
of h and x_hat are bf16 too: at most 8 roundings of relative size 2^-9 each reach one gradient,
so max|G - G_ref| / max|G_ref| <= 8 * 2^-9 = 1.6e-2 to first order; the bound asserted is 2e-2
(the forward's own bf16 bound).  Each routed expert's weight gradient is checked on its own
(a wrong expert cannot hide behind the others' larger values), and an expert that received no
pair must get exactly zero.
"""
import dataclasses

import numpy as np
import pytest
import torch

import datagen
import oracle
import oracle.backward as ob
import latent_routing_quantile_b200 as lq

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from latent_routing_quantile_b200 import build
    build.build()
    yield


def _rel(g, ref):
    den = float(np.max(np.abs(ref)))
    return float(np.max(np.abs(g - ref))) / (den if den > 0 else 1.0)


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (1, 0), (0, 1), (1, 1)])
@pytest.mark.parametrize("k_split", [1, 3])
@pytest.mark.parametrize("M,N", [(200, 192), (392, 256)])
def test_engine_operand_layouts_and_split_k(a_mn, b_mn, k_split, M, N):
    """C = op(A) op(B)^T with either operand stored MN-major (the transposed reads of the
    backward's products), ragged M, N and K, against the float64 product of the same bf16
    values; M = 392 runs the two-CTA 256-row tiles.  fp32 accumulation over K = 200 terms: the
    error stays below 1e-5 of max|C|."""
    K = 200
    g = torch.Generator().manual_seed(7 + 2 * a_mn + b_mn)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    B = torch.randn(N, K, generator=g).to(torch.bfloat16)
    ref = A.double() @ B.double().T
    a_dev = (A.T.contiguous() if a_mn else A).cuda()
    b_dev = (B.T.contiguous() if b_mn else B).cuda()
    c = lq.gemm_bf16_ex(a_dev, b_dev, a_mn=bool(a_mn), b_mn=bool(b_mn), k_split=k_split)
    torch.cuda.synchronize()
    err = _rel(c.cpu().double().numpy(), ref.numpy())
    assert err <= 1e-5, err


SMALL = datagen.LayerShape("bwd_small", 300, 256, 128, 64, 4, 128, 256, "bf16", seed=71, offset_var=0.5)
NOSHARED = datagen.LayerShape("bwd_noshared", 200, 256, 128, 128, 6, 128, 0, "bf16", seed=72)
ONETOKEN = datagen.LayerShape("bwd_one", 1, 256, 128, 64, 4, 128, 128, "bf16", seed=73)


def run_backward(shape, gain="random", bias_std=0.0, weights_gain=True):
    w_cpu = datagen.layer_weights(shape, gain=gain)
    x = datagen.tokens(shape)
    dy = datagen.output_grad(shape, seed=shape.seed + 100)
    w_dev = {n: t.cuda() for n, t in w_cpu.items()}
    if not weights_gain:
        w_dev.pop("rms_gain")
    layer = lq.Layer(shape.d, shape.l, shape.E, shape.k, shape.h, shape.hs, lq.BF16, shape.T, w_dev,
                     rms_eps=shape.rms_eps)
    b = np.zeros(shape.E)
    if bias_std:
        b = datagen.normal_bias(shape.E, shape.seed, bias_std).astype(np.float32)
        layer.set_bias(torch.from_numpy(b).cuda())
        b = b.astype(np.float64)
    y, g = layer.forward_backward(x.cuda(), dy.cuda(), w_dev)
    torch.cuda.synchronize()
    assert layer.status() == 0
    r = layer.routing()
    layer.close()
    ref = ob.layer_backward(x, w_cpu, b, shape.k, dy, shape.rms_eps)
    return {n: t.cpu().double().numpy() for n, t in g.items()}, ref, r, y


def check_grads(shape, g, ref, r):
    idx = r["idx"].cpu().numpy()
    assert np.array_equal(np.sort(idx, 1), np.sort(ref["idx"], 1)), "the backward must be taken at the oracle's expert choice"
    errs = {}
    for n in ("x", "rms_gain", "w_down", "w_router", "router_bias", "w_up", "ws1", "ws3", "ws2"):
        if n in ref:
            errs[n] = _rel(g[n], ref[n])
    counts = np.bincount(idx.ravel(), minlength=shape.E)
    for n in ("w1", "w3", "w2"):
        worst = 0.0
        for e in range(shape.E):
            if counts[e] == 0:
                assert not np.any(g[n][e]), f"{n}[{e}]: an expert without pairs must get a zero gradient"
                continue
            worst = max(worst, _rel(g[n][e], ref[n][e]))
        errs[n] = worst
    bad = {n: v for n, v in errs.items() if not v <= TOL}
    assert not bad, f"gradients off the oracle: {bad} (all: {errs})"
    return errs


def test_backward_matches_the_oracle():
    """Ragged T (300 tokens: two full 128-row tiles and a tail), random gain, column offsets."""
    g, ref, r, _ = run_backward(SMALL)
    check_grads(SMALL, g, ref, r)


def test_backward_with_a_bias_that_reroutes():
    """A non-zero balancing bias moves the expert choice but gets no gradient of its own; the
    gates stay the renormalised unbiased scores."""
    g, ref, r, _ = run_backward(SMALL, bias_std=0.05)
    check_grads(SMALL, g, ref, r)


def test_backward_without_a_shared_expert_or_gain_tensor():
    g, ref, r, _ = run_backward(NOSHARED, gain="ones", weights_gain=False)
    check_grads(NOSHARED, g, ref, r)


def test_backward_of_one_token():
    """T = 1: most experts get no pair (their gradients must be exactly zero)."""
    g, ref, r, _ = run_backward(ONETOKEN)
    check_grads(ONETOKEN, g, ref, r)


def test_backward_rejects_unsupported_layers():
    shape = datagen.LayerShape("bwd_f32", 64, 256, 128, 64, 4, 128, 256, "f32", seed=74)
    w = {n: t.cuda() for n, t in datagen.layer_weights(shape).items()}
    layer = lq.Layer(shape.d, shape.l, shape.E, shape.k, shape.h, shape.hs, lq.F32, shape.T, w)
    x = datagen.tokens(shape).cuda()
    with pytest.raises(lq.LmoeError):
        layer.forward_backward(x, x.clone(), w)
    layer.close()
    # bf16 layer with 8-bit (MXFP8) routed experts: no backward either
    shape = datagen.LayerShape("bwd_mx", 64, 256, 128, 64, 4, 128, 256, "bf16", seed=74)
    w = {n: t.cuda() for n, t in datagen.layer_weights(shape).items()}
    layer = lq.Layer(shape.d, shape.l, shape.E, shape.k, shape.h, shape.hs, lq.BF16, shape.T, w,
                     experts=lq.EXPERTS_MXFP8)
    x = datagen.tokens(shape).cuda()
    with pytest.raises(lq.LmoeError):
        layer.forward_backward(x, x.clone(), w)
    layer.close()


def test_backward_at_the_training_bench_size():
    """mini_replica at full size (T = 8192, d = 1024, l = 256, E = 256, k = 6, h = 256,
    hs = 2048), the workload and launch configuration bench.py times as its training step: every
    gradient against the oracle on all tokens (the weight gradients sum over all of them)."""
    shape = datagen.WORKLOADS["mini_replica"]
    g, ref, r, _ = run_backward(shape, gain="ones")
    errs = check_grads(shape, g, ref, r)
    print("max error / max|ref| per gradient:", {n: f"{v:.2e}" for n, v in errs.items()})


def test_training_and_inference_calls_share_a_handle():
    """One handle, three calls: a training step on 300 tokens, an inference forward on the same
    tokens (its own cached graph; the output must equal the training step's bit for bit, since both
    run the same forward arithmetic), and a training step on the first 128 tokens only (the
    backward's per-call tensor maps and row extents follow T; its gradients must match the oracle
    on those 128 tokens)."""
    shape = SMALL
    w_cpu = datagen.layer_weights(shape, gain="random")
    x = datagen.tokens(shape)
    dy = datagen.output_grad(shape, seed=shape.seed + 100)
    w_dev = {n: t.cuda() for n, t in w_cpu.items()}
    layer = lq.Layer(shape.d, shape.l, shape.E, shape.k, shape.h, shape.hs, lq.BF16, shape.T, w_dev,
                     rms_eps=shape.rms_eps)
    y_train, _ = layer.forward_backward(x.cuda(), dy.cuda(), w_dev)
    y_inf = layer.forward(x.cuda())
    y_inf2 = layer.forward(x.cuda())  # the replay of the cached inference graph
    torch.cuda.synchronize()
    assert torch.equal(y_train, y_inf) and torch.equal(y_inf, y_inf2)
    T2 = 128
    sub = dataclasses.replace(shape, T=T2)
    _, g = layer.forward_backward(x[:T2].contiguous().cuda(), dy[:T2].contiguous().cuda(), w_dev)
    torch.cuda.synchronize()
    assert layer.status() == 0
    r = layer.routing()
    layer.close()
    ref = ob.layer_backward(x[:T2], w_cpu, np.zeros(shape.E), shape.k, dy[:T2], shape.rms_eps)
    check_grads(sub, {n: t.cpu().double().numpy() for n, t in g.items()}, ref, r)


def test_repeated_training_steps_replay_the_backward_graph():
    """A training loop with fixed buffers: the first step runs eagerly, the second captures the
    forward and the backward as graphs, the third replays them (same kernel count, same y bit for
    bit, gradients on the oracle).  Then new gradient buffers: the backward's graph is keyed by
    every pointer it writes, so steps with them run, capture and replay afresh, fill the new
    buffers, and leave the old ones as they were."""
    shape = SMALL
    w_cpu = datagen.layer_weights(shape, gain="random")
    x = datagen.tokens(shape).cuda()
    dy = datagen.output_grad(shape, seed=shape.seed + 100).cuda()
    w_dev = {n: t.cuda() for n, t in w_cpu.items()}
    layer = lq.Layer(shape.d, shape.l, shape.E, shape.k, shape.h, shape.hs, lq.BF16, shape.T, w_dev,
                     rms_eps=shape.rms_eps)
    y = torch.empty_like(x)
    _, ga = layer.forward_backward(x, dy, w_dev, y=y)
    grads_a = dict(ga)
    ys, counts = [], []
    for _ in range(3):
        before = layer.launches()
        layer.forward_backward(x, dy, w_dev, y=y, grads=grads_a)
        torch.cuda.synchronize()
        counts.append(layer.launches() - before)
        ys.append(y.clone())
    assert layer.status() == 0
    assert counts[0] == counts[1] == counts[2] > 0, counts
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])
    r = layer.routing()
    ref = ob.layer_backward(datagen.tokens(shape), w_cpu, np.zeros(shape.E), shape.k,
                            datagen.output_grad(shape, seed=shape.seed + 100), shape.rms_eps)
    check_grads(shape, {n: t.cpu().double().numpy() for n, t in grads_a.items()}, ref, r)
    # new gradient buffers (the old ones zeroed: they must stay zero)
    for t in grads_a.values():
        t.zero_()
    grads_b = {n: torch.full_like(t, float("nan")) for n, t in grads_a.items()}
    for _ in range(3):
        layer.forward_backward(x, dy, w_dev, y=y, grads=grads_b)
    torch.cuda.synchronize()
    assert layer.status() == 0
    assert all(not torch.any(t) for t in grads_a.values()), "a stale graph wrote the old gradient buffers"
    check_grads(shape, {n: t.cpu().double().numpy() for n, t in grads_b.items()}, ref, layer.routing())
    layer.close()
