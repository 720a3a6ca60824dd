"""Pins of the CPU oracle to things other than itself (runs without a GPU).

Each test ties one oracle step to a closed form, a library routine, an
invariant the pages state, a brute force on tiny inputs, or a number the
pages print.  A plausible slip in the oracle (a dropped term, a wrong sign or
index, a transposed operand) fails at least one of them; test_oracle_mutants
plants such slips and checks that.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

import datagen
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# A worked example whose every value has a closed form.
# ---------------------------------------------------------------------------

def worked_example():
    """T=2, d=4, l=2, E=4, k=2, expert hidden 1, shared hidden 1, eps=0.

    x0=[2,2,2,2] -> r=1/2; x1=[3,-3,3,-3] -> r=1/3; gain [1,2,1,1], so
    x_hat0=[1,2,1,1], x_hat1=[1,-2,1,-1].  W_down picks h=[x_hat[0], x_hat[1]/4],
    so h0=[1, 1/2], h1=[1, -1/2].  Router columns give z = ln3, +-ln3, 0, ln4,
    i.e. s0=[3/4,3/4,1/2,4/5], s1=[3/4,1/4,1/2,4/5].  With b=[0,0,0,-1/4]:
    token 0 ties experts 0 and 1 at u=3/4 (lower index first) and drops
    expert 3 (s=4/5 but u=0.55); token 1 picks [0, 3] with gates 15/31, 16/31.
    Expert e: W1 row [ln(e+2), 0], W3 row [0, 1], W2 column [1, e+1].
    """
    ln = math.log
    w = {
        "rms_gain": np.array([1.0, 2.0, 1.0, 1.0]),
        "w_down": np.array([[1.0, 0, 0, 0], [0, 0.25, 0, 0]]),
        "w_router": np.array([[0.0, 0.0], [0.0, 2 * ln(3)], [ln(9), 0.0], [0.0, 0.0]]),
        "router_bias": np.array([ln(3), 0.0, -ln(9), ln(4)]),
        "w1": np.array([[[ln(e + 2), 0.0]] for e in range(4)]),
        "w3": np.array([[[0.0, 1.0]] for e in range(4)]),
        "w2": np.array([[[1.0], [e + 1.0]] for e in range(4)]),
        "w_up": np.array([[1.0, 0], [0, 1.0], [1.0, 1.0], [2.0, -1.0]]),
        "ws1": np.array([[1.0, 0, 0, 0]]),
        "ws3": np.array([[0, 1.0, 0, 0]]),
        "ws2": np.array([[1.0], [0], [0], [1.0]]),
    }
    x = np.array([[2.0, 2, 2, 2], [3.0, -3, 3, -3]])
    b = np.array([0.0, 0.0, 0.0, -0.25])
    return x, w, b


def test_worked_example_closed_forms():
    x, w, b = worked_example()
    out = oracle.layer_forward(x, w, b, k=2, eps=0.0)
    ln = math.log
    np.testing.assert_allclose(out["r"], [0.5, 1 / 3], rtol=1e-15)
    np.testing.assert_allclose(out["h"], [[1, 0.5], [1, -0.5]], rtol=1e-15)
    np.testing.assert_allclose(out["s"], [[0.75, 0.75, 0.5, 0.8], [0.75, 0.25, 0.5, 0.8]], rtol=1e-14)
    assert out["idx"].tolist() == [[0, 1], [0, 3]]
    np.testing.assert_allclose(out["gates"], [[0.5, 0.5], [15 / 31, 16 / 31]], rtol=1e-14)
    np.testing.assert_allclose(out["gap"], [0.2, 0.05], rtol=1e-12)
    np.testing.assert_allclose(out["order_gap"], [0.0, 0.05], atol=1e-15)  # token 0: exact tie
    # routed: silu(ln m) = ln m * m/(m+1); act = silu(a_e) * h[1]; o = act * [1, e+1]
    za0 = 0.5 * (ln(2) * 2 / 3 * 0.5) + 0.5 * (ln(3) * 3 / 4 * 0.5)
    zb0 = 0.5 * (ln(2) * 2 / 3 * 0.5) + 0.5 * 2 * (ln(3) * 3 / 4 * 0.5)
    za1 = -5 * ln(2) / 31 - 20 * ln(5) / 93
    zb1 = -5 * ln(2) / 31 - 80 * ln(5) / 93
    np.testing.assert_allclose(out["z"], [[za0, zb0], [za1, zb1]], rtol=1e-13)
    sh = 1 / (1 + math.exp(-1))  # silu(1)
    y_exp = [[za0 + 2 * sh, zb0, za0 + zb0, 2 * za0 - zb0 + 2 * sh],
             [za1 - 2 * sh, zb1, za1 + zb1, 2 * za1 - zb1 - 2 * sh]]
    np.testing.assert_allclose(out["y"], y_exp, rtol=1e-13)


def test_layer_routing_worked_example_closed_forms():
    """The routing half on its own (the routing oracle of every GPU layer test) takes the worked
    example's closed forms: the gain 2 on column 1 sets h0[1] = 1/2 and the router column offsets
    set s, so dropping either changes h, s and the choice."""
    x, w, b = worked_example()
    r = oracle.layer_routing(x, w, b, k=2, eps=0.0)
    np.testing.assert_allclose(r["h"], [[1, 0.5], [1, -0.5]], rtol=1e-15)
    np.testing.assert_allclose(r["s"], [[0.75, 0.75, 0.5, 0.8], [0.75, 0.25, 0.5, 0.8]], rtol=1e-14)
    assert r["idx"].tolist() == [[0, 1], [0, 3]]
    np.testing.assert_allclose(r["gates"], [[0.5, 0.5], [15 / 31, 16 / 31]], rtol=1e-14)
    np.testing.assert_allclose(r["gap"], [0.2, 0.05], rtol=1e-12)
    np.testing.assert_allclose(r["order_gap"], [0.0, 0.05], atol=1e-15)


def test_layer_routing_equals_the_forward_routing():
    """On a layer with a random gain, router offsets and a non-zero bias, the routing oracle's
    h, s, choice, gates and margins are those of the whole forward, bit for bit."""
    shape, w, x = small_layer()
    b = datagen.normal_bias(shape.E, seed=13, std=0.1).astype(np.float64)
    full = oracle.layer_forward(x, w, b, shape.k, shape.rms_eps)
    r = oracle.layer_routing(x, w, b, shape.k, shape.rms_eps)
    for name in ("h", "s", "idx", "gates", "gap", "order_gap"):
        assert np.array_equal(r[name], full[name]), name


# ---------------------------------------------------------------------------
# Library routines.
# ---------------------------------------------------------------------------

def test_rmsnorm_matches_torch_rms_norm():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((64, 96)) * 3
    g = 1 + 0.1 * rng.standard_normal(96)
    ref = F.rms_norm(torch.from_numpy(x), (96,), weight=torch.from_numpy(g), eps=1e-6).numpy()
    np.testing.assert_allclose(oracle.rmsnorm(x, g, 1e-6), ref, rtol=1e-13, atol=1e-14)


def test_sigmoid_and_silu_match_scipy():
    z = np.linspace(-30, 30, 2001)
    np.testing.assert_allclose(oracle.sigmoid(z), scipy.special.expit(z), rtol=1e-14, atol=1e-300)
    np.testing.assert_allclose(oracle.silu(z), z * scipy.special.expit(z), rtol=1e-14, atol=1e-300)


def test_swiglu_matches_torch_functional():
    rng = np.random.default_rng(1)
    a = rng.standard_normal((7, 16))
    w1, w3 = rng.standard_normal((2, 24, 16))
    w2 = rng.standard_normal((16, 24))
    ta = torch.from_numpy(a)
    ref = F.linear(F.silu(F.linear(ta, torch.from_numpy(w1))) * F.linear(ta, torch.from_numpy(w3)),
                   torch.from_numpy(w2)).numpy()
    np.testing.assert_allclose(oracle.swiglu(a, w1, w3, w2), ref, rtol=1e-12, atol=1e-12)


def test_histogram_matches_numpy_histogram():
    s = datagen.uniform_scores(5000, 6, seed=2).astype(np.float64)
    s[0, :] = 1.0            # the top edge goes to the last bin
    s[1, :] = 0.0
    s[2, :] = 2048 / 4096    # exactly on a bin edge
    hist = oracle.score_histogram(s)
    edges = np.linspace(0.0, 1.0, 4097)
    for e in range(6):
        np.testing.assert_array_equal(hist[e], np.histogram(s[:, e], bins=edges)[0])


@pytest.mark.parametrize("N,E,k", [(256, 32, 4), (1000, 128, 8), (8192, 256, 6), (16384, 896, 16),
                                   (5600, 896, 16), (7, 3, 1), (1, 8, 2)])
def test_quantile_rank_and_exact_quantile_match_inverted_cdf(N, E, k):
    m = oracle.quantile_rank(N, k, E)
    exact = Fraction(E - k, E) * N
    assert m == max(1, min(N, math.ceil(exact)))
    rng = np.random.default_rng(N)
    col = rng.random(N)
    p = float(Fraction(E - k, E))
    if Fraction(p) * N == exact:  # numpy's p*N is exact here, so its rank is the same
        assert oracle.exact_quantile(col, m) == np.quantile(col, p, method="inverted_cdf")


# ---------------------------------------------------------------------------
# Brute force on tiny inputs.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("quantise", [0, 8])
def test_topk_brute_force(quantise):
    T, E, k = 16, 32, 4
    s = datagen.uniform_scores(T, E, seed=5, quantise=quantise).astype(np.float64)
    b = np.zeros(E) if quantise else datagen.normal_bias(E, seed=5, std=0.05).astype(np.float64)
    idx = oracle.biased_topk(s, b, k)
    subsets = np.array(list(itertools.combinations(range(E), k)))
    for t in range(T):
        u = s[t] + b
        chosen = np.zeros((len(subsets), E), dtype=bool)
        np.put_along_axis(chosen, subsets, True, axis=1)
        # a subset is the top-k iff every chosen member beats every unchosen one:
        # larger u, or equal u and lower index
        beats = (u[:, None] > u[None, :]) | ((u[:, None] == u[None, :]) &
                                             (np.arange(E)[:, None] < np.arange(E)[None, :]))
        ok = np.array([beats[np.ix_(c, ~m)].all() for c, m in zip(subsets, chosen)])
        assert ok.sum() == 1
        best = subsets[ok][0]
        # rank order inside the set: each member preceded by those that beat it
        order = sorted(best, key=lambda e: sum(beats[o, e] for o in best))
        assert idx[t].tolist() == order


def test_permutation_brute_force():
    T, E, k = 12, 6, 3
    s = datagen.uniform_scores(T, E, seed=6, quantise=4).astype(np.float64)
    idx = oracle.biased_topk(s, np.zeros(E), k)
    pt, ps, inv = oracle.stable_permutation(idx, E)
    expect = [(t, i) for e in range(E) for t in range(T) for i in range(k) if idx[t, i] == e]
    assert list(zip(pt.tolist(), ps.tolist())) == expect
    for t in range(T):
        for i in range(k):
            assert pt[inv[t, i]] == t and ps[inv[t, i]] == i


# ---------------------------------------------------------------------------
# Invariants the pages state, and special cases.
# ---------------------------------------------------------------------------

def small_layer(E=8, k=3, d=32, l=16, h=8, hs=24, seed=11):
    shape = datagen.LayerShape("pin", 40, d, l, E, k, h, hs, "f32", seed=seed, offset_var=0.5)
    return shape, datagen.layer_weights(shape, gain="random"), datagen.tokens(shape)


def test_shapes_and_gate_sum():
    shape, w, x = small_layer()
    out = oracle.layer_forward(x, w, np.zeros(shape.E), shape.k)
    assert out["y"].shape == (shape.T, shape.d)
    assert out["idx"].shape == (shape.T, shape.k) and out["gates"].shape == (shape.T, shape.k)
    assert np.all(np.abs(out["gates"].sum(1) - 1) <= 1e-15)
    assert np.all(np.diff(np.sort(out["idx"], 1), axis=1) > 0)  # distinct experts per token


def test_bias_reroutes_but_never_changes_gate_magnitudes():
    shape, w, x = small_layer()
    b0 = np.zeros(shape.E)
    b1 = datagen.normal_bias(shape.E, seed=3, std=0.2).astype(np.float64)
    r0 = oracle.layer_routing(x, w, b0, shape.k)
    r1 = oracle.layer_routing(x, w, b1, shape.k)
    s = r0["s"]
    assert np.array_equal(r0["s"], r1["s"])          # scores do not see b
    moved = (np.sort(r0["idx"], 1) != np.sort(r1["idx"], 1)).any(1)
    assert moved.any() and not moved.all()            # the bias reroutes some tokens
    for r in (r0, r1):
        chosen = np.take_along_axis(s, r["idx"], 1)
        np.testing.assert_array_equal(r["gates"], chosen / chosen.sum(1, keepdims=True))
    same = ~moved
    g0 = {(t, e): g for t in np.nonzero(same)[0] for e, g in zip(r0["idx"][t], r0["gates"][t])}
    g1 = {(t, e): g for t in np.nonzero(same)[0] for e, g in zip(r1["idx"][t], r1["gates"][t])}
    assert g0 == g1                                   # bit-identical where the set is unchanged


def test_all_experts_chosen_and_top1():
    shape, w, x = small_layer(E=4, k=4)
    out = oracle.layer_forward(x, w, np.zeros(4), 4)
    np.testing.assert_allclose(out["gates"], np.take_along_axis(out["s"], out["idx"], 1) /
                               out["s"].sum(1, keepdims=True), rtol=1e-15)
    assert np.all(np.isinf(out["gap"]))
    out1 = oracle.layer_forward(x, w, np.zeros(4), 1)
    assert np.all(out1["gates"] == 1.0)


def test_identical_experts_make_routing_irrelevant():
    shape, w, x = small_layer()
    for name in ("w1", "w3", "w2"):
        w[name] = w[name][:1].repeat(shape.E, 1, 1)
    y0 = oracle.layer_forward(x, w, np.zeros(shape.E), shape.k)["y"]
    y1 = oracle.layer_forward(x, w, datagen.normal_bias(shape.E, 4, 0.3).astype(np.float64), shape.k)["y"]
    np.testing.assert_allclose(y0, y1, rtol=1e-12, atol=1e-12)


def test_zero_routed_experts_reduce_to_a_swiglu_mlp():
    shape, w, x = small_layer()
    for name in ("w1", "w3", "w2"):
        w[name] = torch.zeros_like(w[name])
    y = oracle.layer_forward(x, w, np.zeros(shape.E), shape.k)["y"]
    tx = oracle.f64(x)
    t = lambda n: torch.from_numpy(oracle.f64(w[n]))  # noqa: E731
    xn = F.rms_norm(torch.from_numpy(tx), (shape.d,), weight=t("rms_gain"), eps=shape.rms_eps)
    ref = F.linear(F.silu(F.linear(xn, t("ws1"))) * F.linear(xn, t("ws3")), t("ws2")).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_identity_projections_reduce_to_a_plain_moe():
    """l = d, W_down = I, W_up = I, no shared expert: a plain sigmoid top-k MoE on x_hat,
    written here token by token with torch.topk and torch.nn.functional."""
    d = 16
    shape = datagen.LayerShape("moe", 24, d, d, 6, 2, 8, 0, "f32", seed=12, offset_var=0.5)
    w = datagen.layer_weights(shape)
    w["w_down"] = torch.eye(d)
    w["w_up"] = torch.eye(d)
    x = datagen.tokens(shape)
    y = oracle.layer_forward(x, w, np.zeros(6), 2)["y"]
    xn = F.rms_norm(x.double(), (d,), eps=shape.rms_eps)
    for t in range(shape.T):
        s = torch.sigmoid(xn[t] @ w["w_router"].double().T + w["router_bias"].double())
        val, sel = torch.topk(s, 2)
        yt = torch.zeros(d, dtype=torch.float64)
        for g, e in zip(val / val.sum(), sel):
            w1, w3, w2 = (w[n][e].double() for n in ("w1", "w3", "w2"))
            yt += g * F.linear(F.silu(F.linear(xn[t], w1)) * F.linear(xn[t], w3), w2)
        np.testing.assert_allclose(y[t], yt.numpy(), rtol=1e-12, atol=1e-12)


def test_counts_offsets_permutation_invariants():
    shape, w, x = small_layer(E=16, k=4)
    idx = oracle.layer_routing(x, w, np.zeros(16), 4)["idx"]
    cnt = oracle.expert_counts(idx, 16)
    off = oracle.expert_offsets(cnt)
    pt, ps, inv = oracle.stable_permutation(idx, 16)
    assert off[0] == 0 and off[-1] == idx.size and np.all(np.diff(off) == cnt)
    for e in range(16):
        seg = pt[off[e]:off[e + 1]]
        assert np.all(np.diff(seg) > 0)
        assert set(seg.tolist()) == set(np.nonzero((idx == e).any(1))[0].tolist())
        assert np.all(idx[seg, ps[off[e]:off[e + 1]]] == e)
    assert sorted(inv.ravel().tolist()) == list(range(idx.size))


# ---------------------------------------------------------------------------
# Quantile Balancing.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("case", ["uniform", "sigmoid", "duplicates", "one_bin", "edges"])
def test_histogram_quantile_within_one_bin_of_exact(case):
    rng = np.random.default_rng(7)
    N, E, k = 3000, 16, 3
    if case == "uniform":
        s = rng.random((N, E))
    elif case == "sigmoid":
        s = oracle.sigmoid(rng.standard_normal((N, E)) * 3)
    elif case == "duplicates":
        s = np.round(rng.random((N, E)) * 7) / 7
    elif case == "one_bin":
        s = 0.5 + rng.random((N, E)) / 8192
    else:
        s = np.floor(rng.random((N, E)) * 4097) / 4096
    s = np.clip(s, 0, 1).astype(np.float32).astype(np.float64)  # bins are taken on fp32 scores
    hist = oracle.score_histogram(s)
    m = oracle.quantile_rank(N, k, E)
    for e in range(E):
        q = oracle.exact_quantile(s[:, e], m)
        qh = oracle.histogram_quantile(hist[e], m)
        assert abs(qh - q) <= 1 / 4096 + 1e-15


def test_histogram_error_bound_consistent_with_pages():
    pages = json.load(open(os.path.join(GOLDEN, "pages_qb_demo.json")))
    # The demo's 0.0027 histogram error sits above one bin of a 4096-bin [0,1]
    # histogram, so the bound used here is the tighter of the two.
    assert 1 / 4096 < pages["histogram_vs_exact_quantile_max_error"]


def test_qb_update_mean_preserving_and_sign():
    rng = np.random.default_rng(8)
    N, E, k = 2000, 32, 4
    s = oracle.sigmoid(rng.standard_normal((N, E)) + np.linspace(-1, 1, E))
    b = rng.standard_normal(E) * 0.1
    hist = oracle.score_histogram(s)
    for literal in (False, True):
        b1 = oracle.qb_update(b, hist, N, k, 0.3, literal=literal)
        assert abs(b1.mean() - b.mean()) < 1e-14
    # [blog] raise the bar for the hot expert: the most loaded one gets the lowest step
    cnt = oracle.expert_counts(oracle.biased_topk(s, b, k), E)
    b1 = oracle.qb_update(b, hist, N, k, 0.3)
    assert (b1 - b)[np.argmax(cnt)] < 0 < (b1 - b)[np.argmin(cnt)]


def test_qb_single_step_at_beta_one():
    """beta = 1 on fixed scores: every biased column's exact quantile lands within one bin of the
    same level after one update ([demo] Tab 11, single-step convergence)."""
    rng = np.random.default_rng(9)
    N, E, k = 4000, 64, 4
    s = oracle.sigmoid(rng.standard_normal((N, E)) + rng.standard_normal(E))
    b = np.zeros(E)
    hist = oracle.score_histogram(s)
    b1 = oracle.qb_update(b, hist, N, k, 1.0)
    m = oracle.quantile_rank(N, k, E)
    level = np.array([oracle.exact_quantile(s[:, e] + b1[e], m) for e in range(E)])
    assert level.max() - level.min() <= 2 / 4096 + 1e-7  # + fp32 rounding of the binned scores
    before = oracle.load_ratio(oracle.expert_counts(oracle.biased_topk(s, b, k), E))
    after = oracle.load_ratio(oracle.expert_counts(oracle.biased_topk(s, b1, k), E))
    assert after < before / 3


def test_sign_rule_worked_example():
    """Hand-computed: loads (3, 1, 2, 2) have mean 2, so expert 0 (hot) steps down by gamma,
    expert 1 (cold) up, experts 2 and 3 (at the mean) stay ([ebook] capsule 16)."""
    b = np.array([0.5, -0.25, 0.0, 0.125])
    got = oracle.sign_rule_update(b, np.array([3, 1, 2, 2]), 0.01)
    np.testing.assert_array_equal(got, [0.49, -0.24, 0.0, 0.125])
    # equal loads: nothing moves
    np.testing.assert_array_equal(oracle.sign_rule_update(b, np.array([5, 5, 5, 5]), 0.01), b)


@pytest.mark.parametrize("seed", range(4))
def test_sign_rule_sign_against_exact_rational_mean(seed):
    """Brute force with exact rationals: the step is +gamma below the mean load, -gamma above it,
    0 at it, for small integer loads that often sit exactly on the mean."""
    from fractions import Fraction
    rng = np.random.default_rng(seed)
    E = int(rng.integers(2, 9))
    load = rng.integers(0, 4, E)
    b = rng.standard_normal(E)
    got = oracle.sign_rule_update(b, load, 0.25)
    mean = Fraction(int(load.sum()), E)
    for e in range(E):
        want = b[e] + (0.25 if load[e] < mean else (-0.25 if load[e] > mean else 0.0))
        assert got[e] == want


def test_sign_rule_revives_a_collapsed_router():
    """[ebook] capsule 16: most experts dead (never selected) and the sign rule as the fix.  On
    fixed scores where 4 of 32 experts take every token, repeated steps of gamma = 1e-2 bring
    every expert back; each step moves each bias by exactly 0 or gamma."""
    rng = np.random.default_rng(11)
    N, E, k = 2048, 32, 2
    off = np.zeros(E)
    off[:4] = 3.0
    s = oracle.sigmoid(rng.standard_normal((N, E)) * 0.5 + off)
    b = np.zeros(E)
    dead0 = int((oracle.expert_counts(oracle.biased_topk(s, b, k), E) == 0).sum())
    assert dead0 >= 24
    for _ in range(200):
        load = oracle.expert_counts(oracle.biased_topk(s, b, k), E)
        b1 = oracle.sign_rule_update(b, load, 1e-2)
        assert set(np.round(np.abs(b1 - b), 12)) <= {0.0, 0.01}
        b = b1
    assert int((oracle.expert_counts(oracle.biased_topk(s, b, k), E) == 0).sum()) == 0


@pytest.mark.slow
def test_qb_skewed_router_converges_like_the_demo():
    """50 steps, beta 0.05, fresh tokens each step: max/min load starts at >= 3.5 and ends near
    the demo's 1.5 ([demo] Tab 2 Figure 2(a): 3.7 -> 1.5)."""
    pages = json.load(open(os.path.join(GOLDEN, "pages_qb_demo.json")))
    shape = datagen.WORKLOADS["qb_skewed"]
    a = json.load(open(os.path.join(GOLDEN, "qb_skew_offset.json")))["a"]
    c = np.zeros(shape.E, dtype=np.float32)
    c[0] = a
    w = datagen.layer_weights(shape, router_offsets=c)
    b = np.zeros(shape.E)
    ratios = []
    for step in range(shape.steps):
        x = datagen.tokens(shape, seed=shape.seed + step)
        r = oracle.layer_routing(x, w, b, shape.k)
        cnt = oracle.expert_counts(r["idx"], shape.E)
        ratios.append(oracle.load_ratio(cnt))
        if step == 0:
            assert cnt[0] / (shape.T * shape.k / shape.E) == pytest.approx(3.7, abs=0.1)
        b = oracle.qb_update(b, oracle.score_histogram(r["s"]), shape.T, shape.k, shape.beta)
    assert ratios[0] >= 3.5
    assert min(ratios[-5:]) <= pages["max_min_load_ratio_after_qb"] * 1.1
    assert max(ratios[-5:]) < ratios[0] / 2.5


def test_topk_margins_by_repeated_maximum():
    """The near-tie margins the parity checks lean on: u_(k) - u_(k+1) and the smallest gap among
    the top k+1, found here by taking the maximum k+1 times (no sort)."""
    rng = np.random.default_rng(91)
    for trial in range(40):
        E = int(rng.integers(2, 12))
        k = int(rng.integers(1, E + 1))
        s = rng.uniform(0, 1, (5, E))
        if trial % 4 == 0:
            s = np.round(s * 8) / 8  # exact ties
        b = rng.normal(0, 0.1, E)
        gap, ogap = oracle.topk_gap(s, b, k), oracle.topk_order_gap(s, b, k)
        for t in range(5):
            u = list(s[t] + b)
            tops = []
            for _ in range(min(k + 1, E)):
                m = max(u)
                tops.append(m)
                u.remove(m)
            want_gap = tops[k - 1] - tops[k] if k < E else np.inf
            diffs = [tops[i] - tops[i + 1] for i in range(len(tops) - 1)]
            want_ogap = min(diffs) if diffs else np.inf
            assert gap[t] == want_gap and ogap[t] == want_ogap
