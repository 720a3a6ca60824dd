"""Plants plausible mistakes in the CPU oracle and checks that a pin catches each one.

Every mutant replaces one oracle function (on the CPU only, through pytest's
monkeypatch) and reruns the pin that should reject it.
"""
import numpy as np
import pytest

import oracle
import test_oracle_pins as pins


MUTANTS = {
    # rmsnorm: sum instead of mean
    "rms_sum": ("rms_reciprocal", lambda x, eps: 1 / np.sqrt(np.sum(x * x, 1) + eps),
                [pins.test_rmsnorm_matches_torch_rms_norm, pins.test_worked_example_closed_forms]),
    # rmsnorm: gain dropped
    "no_gain": ("rmsnorm", lambda x, g, eps: x * oracle.rms_reciprocal(x, eps)[:, None],
                [pins.test_rmsnorm_matches_torch_rms_norm]),
    # router: sign of the logit flipped
    "router_sign": ("router_scores", lambda h, w, c: oracle.sigmoid(-(h @ w.T + c[None, :])),
                    [pins.test_worked_example_closed_forms]),
    # top-k: ties go to the higher index
    "ties_high": ("biased_topk",
                  lambda s, b, k: (s.shape[1] - 1 - np.argsort(-(s + b)[:, ::-1], 1, kind="stable"))[:, :k],
                  [lambda: pins.test_topk_brute_force(8), pins.test_worked_example_closed_forms]),
    # top-k: selects on s, ignoring the bias
    "unbiased_select": ("biased_topk", lambda s, b, k: np.argsort(-s, 1, kind="stable")[:, :k],
                        [pins.test_bias_reroutes_but_never_changes_gate_magnitudes]),
    # gates: renormalise but forget to divide
    "gate_unnormalised": ("gate_weights", lambda s, idx: np.take_along_axis(s, idx, 1),
                          [pins.test_shapes_and_gate_sum]),
    # SwiGLU: silu on the wrong branch
    "swiglu_swapped": ("swiglu", lambda a, w1, w3, w2: ((a @ w1.T) * oracle.silu(a @ w3.T)) @ w2.T,
                       [pins.test_swiglu_matches_torch_functional, pins.test_worked_example_closed_forms]),
    # combine: only the first slot
    "combine_first": ("combine", lambda g, o: g[:, 0, None] * o[:, 0],
                      [pins.test_worked_example_closed_forms, pins.test_identity_projections_reduce_to_a_plain_moe]),
    # shared expert: the W3 (linear) branch dropped
    "shared_no_gate": ("shared_expert", lambda xh, w1, w3, w2: oracle.silu(xh @ w1.T) @ w2.T,
                       [pins.test_zero_routed_experts_reduce_to_a_swiglu_mlp,
                        pins.test_worked_example_closed_forms]),
    # histogram: off by one bin at the top edge
    "bins_no_clamp": ("score_bins", lambda s, nbins=4096: np.floor(s * nbins).astype(np.int64) % nbins,
                      [pins.test_histogram_matches_numpy_histogram]),
    # quantile rank: floor instead of ceiling
    "rank_floor": ("quantile_rank", lambda N, k, E: max(1, ((E - k) * N) // E),
                   [lambda: pins.test_quantile_rank_and_exact_quantile_match_inverted_cdf(1000, 128, 8)]),
    # QB: wrong sign of the step
    "qb_sign": ("qb_update",
                lambda b, hist, N, k, beta, literal=False, nbins=4096:
                2 * oracle.f64(b) - _QB(b, hist, N, k, beta, literal, nbins),
                [pins.test_qb_update_mean_preserving_and_sign, pins.test_qb_single_step_at_beta_one]),
    # QB: no mean centring
    "qb_no_centre": ("qb_update",
                     lambda b, hist, N, k, beta, literal=False, nbins=4096:
                     _QB(b, hist, N, k, beta, literal, nbins) - beta * _QMEAN(b, hist, N, k, literal, nbins),
                     [pins.test_qb_update_mean_preserving_and_sign]),
    # QB: crossing bin found with > instead of >=
    "qb_crossing": ("histogram_quantile",
                    lambda hist_e, m, nbins=4096: _HQ(hist_e, m + 1, nbins),
                    [lambda: [pins.test_histogram_quantile_within_one_bin_of_exact(c)
                              for c in ("uniform", "sigmoid", "duplicates", "one_bin", "edges")]]),
    # sign rule: direction flipped (hot experts pushed further up)
    "sign_rule_flipped": ("sign_rule_update",
                          lambda b, load, gamma: 2 * oracle.f64(b) - _SR(b, load, gamma),
                          [pins.test_sign_rule_worked_example, pins.test_sign_rule_revives_a_collapsed_router]),
    # sign rule: compared with the largest load instead of the mean (no bias ever falls)
    "sign_rule_vs_max": ("sign_rule_update",
                         lambda b, load, gamma: oracle.f64(b) + gamma * np.sign(np.max(load) - np.asarray(load)),
                         [pins.test_sign_rule_worked_example,
                          lambda: pins.test_sign_rule_sign_against_exact_rational_mean(0)]),
    # routing oracle: RMSNorm gain dropped
    "routing_no_gain": ("layer_routing",
                        lambda x, w, b, k, eps=1e-6: _LR(x, {**w, "rms_gain": np.ones(len(w["rms_gain"]))}, b, k, eps),
                        [pins.test_layer_routing_worked_example_closed_forms,
                         pins.test_layer_routing_equals_the_forward_routing]),
    # routing oracle: router column offsets dropped
    "routing_no_offsets": ("layer_routing",
                           lambda x, w, b, k, eps=1e-6:
                           _LR(x, {**w, "router_bias": np.zeros(len(w["router_bias"]))}, b, k, eps),
                           [pins.test_layer_routing_worked_example_closed_forms,
                            pins.test_layer_routing_equals_the_forward_routing]),
    # routing oracle: the bias ignored in the choice
    "routing_no_bias": ("layer_routing",
                        lambda x, w, b, k, eps=1e-6: _LR(x, w, np.zeros_like(oracle.f64(b)), k, eps),
                        [pins.test_layer_routing_worked_example_closed_forms,
                         pins.test_layer_routing_equals_the_forward_routing]),
}

_SR = oracle.sign_rule_update
_LR = oracle.layer_routing
_QB = oracle.qb_update
_HQ = oracle.histogram_quantile


def _QMEAN(b, hist, N, k, literal, nbins):
    m = oracle.quantile_rank(N, k, hist.shape[0])
    q = np.array([_HQ(hist[e], m, nbins) for e in range(hist.shape[0])])
    u = q if literal else q + oracle.f64(b)
    return u.mean()


def _fails(pin):
    try:
        pin()
    except (AssertionError, ValueError, IndexError):
        return True
    return False


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_a_pin_catches_the_mutant(name, monkeypatch):
    target, mutant, pin_list = MUTANTS[name]
    monkeypatch.setattr(oracle, target, mutant)
    assert any(_fails(p) for p in pin_list), f"no pin caught mutant {name}"
