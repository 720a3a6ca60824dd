"""Pins of the CPU oracle for the layer's gradients (oracle.backward), on the CPU only.

Each gradient is checked against something other than itself: central finite differences of
the forward oracle (oracle.layer_forward, the function whose derivative it claims to be), the
autograd of torch's own RMSNorm and SiLU, and invariants of the gate renormalisation.  Planted
mistakes in the backward (a dropped term, a wrong sign, a transposed operand) must fail a pin.
"""
import numpy as np
import pytest
import torch

import datagen
import oracle
import oracle.backward as ob

SHAPE = datagen.LayerShape("bwd", 10, 16, 8, 6, 2, 8, 12, "f32", seed=61, offset_var=0.5)


def _problem(hs=SHAPE.hs):
    shape = SHAPE if hs == SHAPE.hs else datagen.LayerShape("bwd", 10, 16, 8, 6, 2, 8, hs, "f32", seed=61,
                                                            offset_var=0.5)
    w = {k: oracle.f64(v) for k, v in datagen.layer_weights(shape, gain="random").items()}
    x = oracle.f64(datagen.tokens(shape))
    rng = np.random.default_rng(62)
    b = rng.normal(0.0, 0.05, shape.E)
    dy = rng.standard_normal((shape.T, shape.d))
    return shape, w, x, b, dy


def _loss(x, w, b, k, dy):
    out = oracle.layer_forward(x, w, b, k)
    return float((out["y"] * dy).sum()), out["idx"]


def _fd_check(shape, w, x, b, dy, eps=1e-5, rtol=1e-6, ndir=3):
    """<grad, V> against (L(P + eps V) - L(P - eps V)) / (2 eps) for random directions V of every
    input and weight; the expert choice must stay the same at both points."""
    g = ob.layer_backward(x, w, b, shape.k, dy)
    rng = np.random.default_rng(63)
    _, idx0 = _loss(x, w, b, shape.k, dy)
    assert np.array_equal(g["idx"], idx0)
    for name in ["x"] + sorted(w):
        base = x if name == "x" else w[name]
        assert g[name].shape == base.shape, name
        for _ in range(ndir):
            v = rng.standard_normal(base.shape)
            vals = []
            for sgn in (1.0, -1.0):
                p = base + sgn * eps * v
                if name == "x":
                    loss, idx = _loss(p, w, b, shape.k, dy)
                else:
                    loss, idx = _loss(x, dict(w, **{name: p}), b, shape.k, dy)
                assert np.array_equal(idx, idx0), f"{name}: the expert choice moved; use a smaller step"
                vals.append(loss)
            num = (vals[0] - vals[1]) / (2 * eps)
            ana = float((g[name] * v).sum())
            assert abs(num - ana) <= rtol * max(1.0, abs(num)), f"{name}: analytic {ana}, differences {num}"


def test_backward_matches_central_differences_of_the_forward():
    _fd_check(*_problem())


def test_backward_without_a_shared_expert():
    shape, w, x, b, dy = _problem(hs=0)
    assert "ws1" not in w
    _fd_check(shape, w, x, b, dy)


def test_no_gradient_reaches_the_qb_bias():
    """The bias only reroutes: moving it without changing the choice leaves y unchanged, so the
    loss's derivative along any bias direction is zero ([demo] Tab 8-10)."""
    shape, w, x, b, dy = _problem()
    base, idx0 = _loss(x, w, b, shape.k, dy)
    v = np.random.default_rng(64).standard_normal(shape.E)
    for eps in (1e-6, -1e-6):
        loss, idx = _loss(x, w, b + eps * v, shape.k, dy)
        assert np.array_equal(idx, idx0)
        assert loss == base
    assert "b" not in ob.layer_backward(x, w, b, shape.k, dy)


def test_gate_gradient_is_blind_to_a_common_scale_of_the_chosen_scores():
    """g = s / sum s does not change when every chosen score is scaled by one factor, so the
    score gradient is orthogonal to the chosen scores: sum_j s_j dL/ds_j = 0."""
    rng = np.random.default_rng(65)
    s_sel = rng.uniform(0.05, 1.0, (50, 6))
    dg = rng.standard_normal((50, 6))
    ds = ob.gate_backward(s_sel, dg)
    np.testing.assert_allclose((s_sel * ds).sum(1), 0.0, atol=1e-12)
    # and equals the Jacobian written out element by element on one token
    S = s_sel[0].sum()
    jac = (np.eye(6) - (s_sel[0] / S)[:, None]) / S  # jac[i, j] = d g_i / d s_j
    np.testing.assert_allclose(ds[0], dg[0] @ jac, rtol=1e-12)


def test_swiglu_backward_matches_torch_autograd():
    rng = np.random.default_rng(66)
    a, w1, w3, w2, dout = (rng.standard_normal(s) for s in [(7, 5), (9, 5), (9, 5), (4, 9), (7, 4)])
    ta, t1, t3, t2 = (torch.tensor(m, requires_grad=True) for m in (a, w1, w3, w2))
    out = (torch.nn.functional.silu(ta @ t1.T) * (ta @ t3.T)) @ t2.T
    out.backward(torch.tensor(dout))
    got = ob.swiglu_backward(a, w1, w3, w2, dout)
    for mine, ref in zip(got, (ta, t1, t3, t2)):
        np.testing.assert_allclose(mine, ref.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_rmsnorm_backward_matches_torch_autograd():
    rng = np.random.default_rng(67)
    x = rng.standard_normal((6, 16))
    gain = 1.0 + 0.1 * rng.standard_normal(16)
    dxh = rng.standard_normal((6, 16))
    tx, tg = torch.tensor(x, requires_grad=True), torch.tensor(gain, requires_grad=True)
    torch.nn.functional.rms_norm(tx, (16,), weight=tg, eps=1e-6).backward(torch.tensor(dxh))
    dx, dg = ob.rmsnorm_backward(x, gain, 1e-6, dxh)
    np.testing.assert_allclose(dx, tx.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dg, tg.grad.numpy(), rtol=1e-10, atol=1e-12)


_SG = ob.silu_grad
_GB = ob.gate_backward
_RB = ob.rmsnorm_backward
_SB = ob.swiglu_backward

BACKWARD_MUTANTS = {
    # silu': the v (1 - sigmoid) term dropped
    "silu_grad_short": ("silu_grad", lambda v: oracle.sigmoid(v),
                        [test_swiglu_backward_matches_torch_autograd]),
    # gates: the renormalisation term dropped (as if g = s)
    "gate_no_renorm": ("gate_backward", lambda s_sel, dg: dg / s_sel.sum(1, keepdims=True),
                       [test_gate_gradient_is_blind_to_a_common_scale_of_the_chosen_scores,
                        test_backward_matches_central_differences_of_the_forward]),
    # gates: the renormalisation term with the wrong sign
    "gate_sign": ("gate_backward",
                  lambda s_sel, dg: (dg + (s_sel / s_sel.sum(1, keepdims=True) * dg).sum(1, keepdims=True))
                  / s_sel.sum(1, keepdims=True),
                  [test_gate_gradient_is_blind_to_a_common_scale_of_the_chosen_scores]),
    # RMSNorm: the derivative of r dropped
    "rms_no_dr": ("rmsnorm_backward",
                  lambda x, gain, eps, dxh: (dxh * gain[None, :] * oracle.rms_reciprocal(x, eps)[:, None],
                                             _RB(x, gain, eps, dxh)[1]),
                  [test_rmsnorm_backward_matches_torch_autograd,
                   test_backward_matches_central_differences_of_the_forward]),
    # router: the sigmoid's derivative dropped (logit gradient taken as ds)
    "router_no_sigmoid_grad": ("router_backward",
                               lambda ds, s, h, w_r: (ds.T @ h, ds.sum(0), ds @ w_r),
                               [test_backward_matches_central_differences_of_the_forward]),
    # routed experts: the linear branch's share of the input gradient dropped
    "expert_da_gate_only": ("swiglu_backward",
                            lambda a, w1, w3, w2, dout: (
                                ((dout @ w2) * (a @ w3.T) * _SG(a @ w1.T)) @ w1,) + _SB(a, w1, w3, w2, dout)[1:],
                            [test_backward_matches_central_differences_of_the_forward]),
    # SwiGLU: the W2 gradient transposed (act^T dout in place of dout^T act)
    "w2_transposed": ("swiglu_backward",
                      lambda a, w1, w3, w2, dout: _SB(a, w1, w3, w2, dout)[:3]
                      + (_SB(a, w1, w3, w2, dout)[3].reshape(w2.shape[::-1]).T,),
                      [test_swiglu_backward_matches_torch_autograd]),
}


def _fails(pin):
    try:
        pin()
    except (AssertionError, ValueError, IndexError):
        return True
    return False


@pytest.mark.parametrize("name", sorted(BACKWARD_MUTANTS))
def test_a_backward_pin_catches_the_mutant(name, monkeypatch):
    target, mutant, pin_list = BACKWARD_MUTANTS[name]
    monkeypatch.setattr(ob, target, mutant)
    assert any(_fails(p) for p in pin_list), f"no pin caught mutant {name}"
