"""Parity of the CUDA layer with the CPU oracle, through the C ABI (needs a B200).

Integer results (expert choice, counts, offsets, permutation, histogram) must match exactly;
where the GPU's fp32 scores and the oracle's fp64 scores may order two experts differently,
only tokens whose oracle k-th and (k+1)-th biased scores lie within 1e-5 of each other may
differ, and such tokens must stay under 1e-4 of all tokens.  Stage tests feed the kernels the
same fp32 scores the oracle sees, so there every decision is taken in the same precision.
Layer outputs: max|y - y_ref| / max|y_ref| <= 2e-2 for bf16, 1e-4 for fp32.
"""
import json
import os

import numpy as np
import pytest
import torch

import datagen
import oracle
import latent_routing_quantile_b200 as lq

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
NEAR_TIE = 1e-5
TOL = {"bf16": 2e-2, "f32": 1e-4}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from latent_routing_quantile_b200 import build
    build.build()
    yield


def normwise(y, ref):
    return float(np.max(np.abs(y - ref)) / np.max(np.abs(ref)))


def check_routing(gpu_idx, ora_idx, gap):
    """Returns the mismatch fraction; asserts every mismatch is a near-tie and the fraction < 1e-4."""
    mism = (gpu_idx != ora_idx).any(1)
    assert not (mism & ~(gap < NEAR_TIE)).any(), "a token that is not a near-tie was routed differently"
    frac = float(mism.mean())
    assert mism.sum() <= int(1e-4 * len(mism)), f"mismatch fraction {frac}"
    return frac


def check_permutation(r, T, k, E):
    idx = r["idx"].cpu().numpy()
    counts = r["counts"].cpu().numpy()
    off = r["offsets"].cpu().numpy()
    perm = r["perm"].cpu().numpy()
    inv = r["inv"].cpu().numpy().reshape(T, k)
    assert np.array_equal(counts, np.bincount(idx.ravel(), minlength=E))
    assert off[0] == 0 and np.array_equal(np.diff(off), counts)
    for e in range(E):
        seg = perm[off[e]:off[e + 1]]
        assert np.all(np.diff(seg) > 0)
        assert np.all((idx[seg] == e).any(1))
    t = np.repeat(np.arange(T), k)
    assert np.array_equal(perm[inv.ravel()], t)
    assert np.array_equal(np.sort(inv.ravel()), np.arange(T * k))


def make_layer(shape, w, max_tokens=None):
    return lq.layer_from_weights(shape, w, max_tokens=max_tokens)


# --------------------------------------------------------------------------- GEMM engine
@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 384, 320), (1, 64, 128), (647, 512, 1024)])
def test_tensor_core_gemm_matches_fp32_matmul(M, N, K):
    g = torch.Generator().manual_seed(M * 7 + N)
    a = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    b = torch.randn(N, K, generator=g).to(torch.bfloat16).cuda()
    c = lq.gemm_bf16(a, b)
    ref = a.double() @ b.double().T
    torch.cuda.synchronize()
    err = (c.double() - ref).abs().max().item()
    assert err <= 1e-5 * K ** 0.5 * ref.abs().max().item() + 1e-5, err


# --------------------------------------------------------------------------- routing stage
@pytest.mark.parametrize("T,E,k,quant", [(1000, 256, 6, 0), (777, 64, 8, 16), (300, 896, 16, 0), (129, 1024, 32, 64)])
def test_route_scores_stage_bit_exact(T, E, k, quant):
    s = datagen.uniform_scores(T, E, seed=T + E, quantise=quant)
    b = datagen.normal_bias(E, seed=E, std=0.02)
    u32 = (s + b[None, :]).astype(np.float32)   # the kernel decides on fp32 s + b
    shape = datagen.LayerShape("route", T, 64, 64, E, k, 64, 0, "bf16", seed=1)
    layer = make_layer(shape, datagen.layer_weights(shape))
    layer.set_bias(torch.from_numpy(b).cuda())
    layer.route_scores(torch.from_numpy(s).cuda(), record_stats=True)
    r = layer.routing()
    hist, ntok = layer.hist()
    torch.cuda.synchronize()
    s64 = s.astype(np.float64)
    idx = oracle.biased_topk(u32.astype(np.float64), np.zeros(E), k)
    assert np.array_equal(r["idx"].cpu().numpy(), idx)
    np.testing.assert_allclose(r["gates"].cpu().numpy(), oracle.gate_weights(s64, idx), rtol=2e-6)
    assert np.array_equal(r["counts"].cpu().numpy(), oracle.expert_counts(idx, E))
    assert np.array_equal(r["offsets"].cpu().numpy(), oracle.expert_offsets(oracle.expert_counts(idx, E)))
    pt, ps, inv = oracle.stable_permutation(idx, E)
    assert np.array_equal(r["perm"].cpu().numpy(), pt)
    assert np.array_equal(r["inv"].cpu().numpy(), inv.ravel())
    assert np.array_equal(hist.cpu().numpy(), oracle.score_histogram(s64))
    assert int(ntok.item()) == T
    assert layer.status() == 0
    layer.close()


def test_nan_score_is_flagged_and_never_chosen():
    T, E, k = 64, 64, 4
    s = datagen.uniform_scores(T, E, seed=3)
    s[5, 7] = np.nan
    s[5, 9] = 2.0  # would win; ensures the NaN row still routes
    shape = datagen.LayerShape("nan", T, 64, 64, E, k, 64, 0, "bf16", seed=1)
    layer = make_layer(shape, datagen.layer_weights(shape))
    layer.route_scores(torch.from_numpy(s).cuda())
    r = layer.routing()
    assert 7 not in r["idx"][5].cpu().tolist()
    assert layer.status() & lq.STATUS_NAN_SCORE
    assert layer.status() == 0  # cleared by the read
    layer.close()


# --------------------------------------------------------------------------- QB update stage
@pytest.mark.parametrize("literal", [False, True])
def test_qb_update_stage(literal):
    T, E, k, beta = 3000, 128, 8, 0.3
    rng = np.random.default_rng(5)
    s = oracle.sigmoid(rng.standard_normal((T, E)) + np.linspace(-1, 1, E)).astype(np.float32)
    b0 = datagen.normal_bias(E, seed=6, std=0.05)
    hist = oracle.score_histogram(s.astype(np.float64))
    shape = datagen.LayerShape("qb", T, 64, 64, E, k, 64, 0, "bf16", seed=1)
    layer = make_layer(shape, datagen.layer_weights(shape))
    layer.set_bias(torch.from_numpy(b0).cuda())
    layer.set_hist(torch.from_numpy(hist.astype(np.int32)).cuda(), torch.tensor([T], dtype=torch.int64).cuda())
    layer.qb_update(beta, literal=literal)
    b1 = layer.bias().cpu().numpy()
    ref = oracle.qb_update(b0.astype(np.float64), hist, T, k, beta, literal=literal)
    np.testing.assert_allclose(b1, ref, rtol=1e-6, atol=1e-7)
    h2, n2 = layer.hist()
    assert int(h2.abs().sum().item()) == 0 and int(n2.item()) == 0
    # nothing recorded: the bias stays
    layer.qb_update(beta)
    assert np.array_equal(layer.bias().cpu().numpy(), b1)
    layer.close()


# --------------------------------------------------------------------------- whole layer
def run_layer_check(shape, w, x, b=None, sample=None, record=True):
    """Forward on the GPU, oracle on all tokens (routing) and on `sample` rows (outputs)."""
    T, E, k = shape.T, shape.E, shape.k
    layer = make_layer(shape, w, max_tokens=T)
    if b is not None:
        layer.set_bias(torch.from_numpy(b.astype(np.float32)).cuda())
    xd = x.cuda()
    y = layer.forward(xd, record_stats=record)
    r = layer.routing()
    torch.cuda.synchronize()
    b64 = np.zeros(E) if b is None else b.astype(np.float64)
    ro = oracle.layer_routing(x, w, b64, k, shape.rms_eps)
    s_gpu = r["scores"].cpu().numpy()
    s_err = float(np.max(np.abs(s_gpu - ro["s"])))
    assert s_err < 2e-6, f"router scores off by {s_err}"
    frac = check_routing(r["idx"].cpu().numpy(), ro["idx"], ro["gap"])
    check_permutation(r, T, k, E)
    rows = np.arange(T) if sample is None else sample
    xs = x[torch.from_numpy(rows)]
    yo = oracle.layer_forward(xs, w, b64, k, shape.rms_eps)["y"]
    yg = y.float().cpu().numpy()[rows]
    err = normwise(yg, yo)
    assert err <= TOL[shape.dtype], f"output error {err}"
    assert layer.status() == 0
    return layer, y, ro, dict(score_err=s_err, mismatch=frac, out_err=err)


def test_tiny_fp32_layer_and_qb_update():
    shape = datagen.WORKLOADS["tiny_fp32"]
    w = datagen.layer_weights(shape)
    x = datagen.tokens(shape)
    layer, y, ro, stats = run_layer_check(shape, w, x)
    layer.qb_update(shape.beta)
    b_gpu = layer.bias().cpu().numpy()
    hist_o = oracle.score_histogram(ro["s"])
    b_ref = oracle.qb_update(np.zeros(shape.E), hist_o, shape.T, shape.k, shape.beta)
    np.testing.assert_allclose(b_gpu, b_ref, rtol=1e-5, atol=2 * shape.beta / 4096)
    layer.close()


@pytest.mark.parametrize("gain", ["ones", "random"])
def test_small_bf16_layer_ragged(gain):
    shape = datagen.LayerShape("small", 1000, 256, 128, 64, 4, 128, 256, "bf16", seed=21, offset_var=0.5)
    w = datagen.layer_weights(shape, gain=gain)
    x = datagen.tokens(shape)
    layer, y, ro, stats = run_layer_check(shape, w, x)
    # the histogram of the recorded forward: bins can differ only for scores on a bin edge
    hist, ntok = layer.hist()
    ho = oracle.score_histogram(ro["s"])
    edge = np.abs(ro["s"] * 4096 - np.round(ro["s"] * 4096)) < 1e-6 * 4096
    diff = np.abs(hist.cpu().numpy() - ho).sum(1)
    assert np.all(diff <= 2 * edge.sum(0))
    assert int(ntok.item()) == shape.T
    layer.close()


def test_forward_host_and_determinism():
    shape = datagen.LayerShape("host", 520, 256, 128, 64, 4, 128, 256, "bf16", seed=22, offset_var=0.5)
    w = datagen.layer_weights(shape)
    x = datagen.tokens(shape)
    layer = make_layer(shape, w)
    y1 = layer.forward(x.cuda())
    y2 = layer.forward(x.cuda())
    xh = x.pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    layer.forward_host(xh, yh)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert torch.equal(y1.cpu(), yh)
    # T = 0 is a no-op, T > max_tokens is rejected
    layer.forward(x[:0].cuda())
    with pytest.raises(lq.LmoeError, match="invalid"):
        layer.forward(torch.zeros((shape.T + 1, shape.d), dtype=torch.bfloat16, device="cuda"))
    layer.close()


def test_mini_replica_full_size():
    shape = datagen.WORKLOADS["mini_replica"]
    w = datagen.layer_weights(shape)
    x = datagen.tokens(shape)
    sample = np.arange(0, shape.T, 16)  # 512 tokens across all tiles
    layer, y, ro, stats = run_layer_check(shape, w, x, sample=sample)
    print("mini_replica", json.dumps(stats))
    layer.close()


def test_qb_skewed_router_run():
    """50 forward + QB steps on the skewed router, GPU and oracle each following their own bias.

    The two bias trajectories can drift apart by at most the histogram resolution: each side's
    quantile estimate lies within one bin (1/4096) of the exact quantile of its own scores, and
    the scores agree to ~1e-6, so |b_gpu - b_oracle| stays below 2/4096 (each update contracts
    the earlier difference by 1 - beta).  A token may then route differently only if its oracle
    margin is below 1e-5 plus twice the measured bias difference.
    """
    shape = datagen.WORKLOADS["qb_skewed"]
    a = json.load(open(os.path.join(GOLDEN, "qb_skew_offset.json")))["a"]
    c = np.zeros(shape.E, dtype=np.float32)
    c[0] = a
    w = datagen.layer_weights(shape, router_offsets=c)
    layer = make_layer(shape, w)
    b_ora = np.zeros(shape.E)
    ratios, qerr, berr, mism = [], [], [], []
    for step in range(shape.steps):
        db = float(np.max(np.abs(layer.bias().cpu().numpy() - b_ora)))
        berr.append(db)
        assert db <= 2 / 4096, (step, db)
        x = datagen.tokens(shape, seed=shape.seed + step)
        layer.forward(x.cuda(), record_stats=True)
        r = layer.routing()
        torch.cuda.synchronize()
        ro = oracle.layer_routing(x, w, b_ora, shape.k, shape.rms_eps)
        diff = (r["idx"].cpu().numpy() != ro["idx"]).any(1)
        assert not (diff & ~(ro["gap"] < NEAR_TIE + 2 * db)).any(), (step, db)
        mism.append(float(diff.mean()))
        cnt = r["counts"].cpu().numpy()
        ratios.append(oracle.load_ratio(cnt))
        hist_o = oracle.score_histogram(ro["s"])
        m = oracle.quantile_rank(shape.T, shape.k, shape.E)
        qerr.append(max(abs(oracle.histogram_quantile(hist_o[e], m) - oracle.exact_quantile(ro["s"][:, e], m))
                        for e in range(shape.E)))
        layer.qb_update(shape.beta)
        b_ora = oracle.qb_update(b_ora, hist_o, shape.T, shape.k, shape.beta)
    print("qb_skewed", json.dumps(dict(ratio_first=ratios[0], ratio_last=ratios[-1], ratios=ratios,
                                       max_q_err=max(qerr), max_bias_diff=max(berr),
                                       max_mismatch_frac=max(mism), mean_mismatch_frac=float(np.mean(mism)))))
    assert mism[0] <= 1e-4  # same bias (zero) on both sides at step 0
    assert ratios[0] >= 3.5 and ratios[-1] < 2.0
    assert max(qerr) <= 1 / 4096 + 1e-7
    layer.close()


@pytest.mark.slow
def test_wide_stress_sampled():
    shape = datagen.WORKLOADS["wide_stress"]
    w = datagen.layer_weights(shape)
    x = datagen.tokens(shape)
    sample = np.arange(0, shape.T, 64)  # 256 tokens
    layer, y, ro, stats = run_layer_check(shape, w, x, sample=sample)
    print("wide_stress", json.dumps(stats))
    layer.close()
