"""CPU oracle for the gradients of the Stable-LatentMoE layer forward.

TEST INFRASTRUCTURE, under the same rule as the rest of this package: only
tests/, __graft_entry__.smoke() and the CPU legs of bench.py may import it,
and it imports nothing from the CUDA library.

What it is: the exact derivative of oracle.layer_forward (float64 numpy), for
a loss whose gradient with respect to the output y is the given dy, written
out step by step in the reverse order of the forward.  The expert choice is
piecewise constant in every input, so, as the layer's training use asks
("Pretraining a Mini Kimi K3", capsule 16: the bias only reroutes; "KimiK3MoE
架构轻量化复刻演示上线", Tab 8-10: the gate weights are the renormalised
unbiased scores), no gradient flows through the top-k selection or into the
QB bias b; the gate weights g_i = s_i / sum_j s_j pass theirs to the router
scores through the renormalisation.

Notation (per token t; the forward's own):
  r = (mean_j x_j^2 + eps)^(-1/2)    x_hat = gain * x * r    h = x_hat W_down^T
  s = sigmoid(h W_r^T + c)           g_i = s_{e_i} / S,  S = sum_i s_{e_i}
  p1 = h W1_e^T, p3 = h W3_e^T       a = silu(p1) * p3      o_i = a W2_e^T
  z = sum_i g_i o_i                  y = z W_up^T + (silu(x_hat Ws1^T) * x_hat Ws3^T) Ws2^T

Parity unpinned beyond SwiGLU: the routed and shared experts are the SwiGLU
stand-in for SiTU-GLU (the pages give no formula for it), so these gradients
are those of SwiGLU.
"""
from __future__ import annotations

import numpy as np

from . import f64, layer_forward, rms_reciprocal, rmsnorm, sigmoid, silu


def silu_grad(v: np.ndarray) -> np.ndarray:
    """d silu(v) / dv = sigmoid(v) (1 + v (1 - sigmoid(v)))."""
    sg = sigmoid(v)
    return sg * (1.0 + v * (1.0 - sg))


def swiglu_backward(a: np.ndarray, w1: np.ndarray, w3: np.ndarray, w2: np.ndarray, dout: np.ndarray):
    """Gradients of out = (silu(a W1^T) * (a W3^T)) W2^T for rows a and output gradient dout.

    Returns (da, dW1, dW3, dW2)."""
    p1, p3 = a @ w1.T, a @ w3.T
    act = silu(p1) * p3
    dact = dout @ w2
    dp1 = dact * p3 * silu_grad(p1)
    dp3 = dact * silu(p1)
    return dp1 @ w1 + dp3 @ w3, dp1.T @ a, dp3.T @ a, dout.T @ act


def gate_backward(s_sel: np.ndarray, dg: np.ndarray) -> np.ndarray:
    """Gradient with respect to the chosen scores of g_i = s_i / sum_j s_j, given dL/dg.

    d g_i / d s_j = (delta_ij - g_i) / S, so dL/ds_j = (dL/dg_j - sum_i g_i dL/dg_i) / S."""
    S = s_sel.sum(axis=1, keepdims=True)
    g = s_sel / S
    return (dg - (g * dg).sum(axis=1, keepdims=True)) / S


def router_backward(ds: np.ndarray, s: np.ndarray, h: np.ndarray, w_r: np.ndarray):
    """Gradients of s = sigmoid(h W_r^T + c) given dL/ds: the logit gradient is ds * s (1 - s).

    Returns (dW_r, dc, dh)."""
    dlogit = ds * s * (1.0 - s)
    return dlogit.T @ h, dlogit.sum(axis=0), dlogit @ w_r


def rmsnorm_backward(x: np.ndarray, gain: np.ndarray, eps: float, dx_hat: np.ndarray):
    """Gradients of x_hat = gain * x * r, r = (mean_j x_j^2 + eps)^(-1/2).

    dr/dx_j = -r^3 x_j / d, so dx = gain * dx_hat * r - x r^3 / d * sum_m gain_m dx_hat_m x_m.
    Returns (dx, dgain)."""
    d = x.shape[1]
    r = rms_reciprocal(x, eps)[:, None]
    gdx = dx_hat * gain[None, :]
    dx = gdx * r - x * (r ** 3) / d * (gdx * x).sum(axis=1, keepdims=True)
    dgain = (dx_hat * x * r).sum(axis=0)
    return dx, dgain


def layer_backward(x, w: dict, b, k: int, dy, eps: float = 1e-6) -> dict:
    """Gradients of sum(y * dy) for y = layer_forward(x, w, b, k, eps)["y"], in float64.

    Returns dx and one entry per weight of `w` (rms_gain, w_down, w_router, router_bias, w1, w3,
    w2, w_up, and ws1, ws3, ws2 when the shared expert exists), each of its weight's shape, plus
    idx (the expert choice the gradients are taken at).  b receives no gradient."""
    x = f64(x)
    dy = f64(dy)
    gain = f64(w["rms_gain"])
    w_down, w_r, w_up = f64(w["w_down"]), f64(w["w_router"]), f64(w["w_up"])
    T = x.shape[0]
    E = w_r.shape[0]
    # the forward's own intermediates: h, s, the choice, the gates, the expert outputs, z
    fwd = layer_forward(x, w, b, k, eps)
    h, s, idx, g, o, zc = fwd["h"], fwd["s"], fwd["idx"], fwd["gates"], fwd["o"], fwd["z"]
    x_hat = rmsnorm(x, gain, eps)
    rows = np.arange(T)[:, None]
    grads = dict(idx=idx)
    grads["w_up"] = dy.T @ zc
    dz = dy @ w_up
    # shared expert on x_hat
    dx_hat = np.zeros_like(x_hat)
    if "ws1" in w:
        dxs, grads["ws1"], grads["ws3"], grads["ws2"] = swiglu_backward(
            x_hat, f64(w["ws1"]), f64(w["ws3"]), f64(w["ws2"]), dy)
        dx_hat += dxs
    # combine: z = sum_i g_i o_i
    dg = np.einsum("tl,tkl->tk", dz, o)
    do = g[:, :, None] * dz[:, None, :]
    # routed experts, each over the (token, slot) pairs routed to it
    dh = np.zeros_like(h)
    dw1 = np.zeros((E,) + tuple(np.shape(w["w1"])[1:]))
    dw3 = np.zeros_like(dw1)
    dw2 = np.zeros((E,) + tuple(np.shape(w["w2"])[1:]))
    for e in np.unique(idx):
        t, i = np.nonzero(idx == e)
        dh_e, dw1[e], dw3[e], dw2[e] = swiglu_backward(h[t], f64(w["w1"][e]), f64(w["w3"][e]),
                                                       f64(w["w2"][e]), do[t, i])
        np.add.at(dh, t, dh_e)
    grads["w1"], grads["w3"], grads["w2"] = dw1, dw3, dw2
    # gates -> chosen scores -> router logits (unchosen scores get nothing)
    ds = np.zeros_like(s)
    ds[rows, idx] = gate_backward(s[rows, idx], dg)
    grads["w_router"], grads["router_bias"], dh_router = router_backward(ds, s, h, w_r)
    dh += dh_router
    # latent down-projection and RMSNorm
    grads["w_down"] = dh.T @ x_hat
    dx_hat += dh @ w_down
    grads["x"], grads["rms_gain"] = rmsnorm_backward(x, gain, eps, dx_hat)
    return grads
