"""Pins of the CPU oracle for block-scaled 8-bit operands (oracle.lowp), on the CPU only.

The element format is pinned to torch's own float8_e4m3fn type (every code decoded, and the cast
of values across all binades, midpoints included); the block scale to its defining inequality by
brute force over powers of two; the dequantised operands to the format's half-step error bound.
Planted mistakes (ties away from zero, a scale one binade off, no saturation) must fail a pin.
"""
import numpy as np
import pytest
import torch

import oracle.lowp as lp


def test_every_e4m3_code_decodes_like_torch():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([lp.e4m3_decode(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan) and nan.sum() == 2  # 0x7f and 0xff
    assert np.array_equal(mine[~nan], ref[~nan])
    assert np.nanmax(mine) == lp.E4M3_MAX and np.nanmin(np.abs(mine[mine != 0])) == 2.0 ** -9


def _grid():
    v = np.array([lp.e4m3_decode(c) for c in range(127)])  # 0 .. 448
    return v


def test_rounding_matches_torch_cast_below_saturation():
    rng = np.random.default_rng(71)
    mags = np.exp2(rng.uniform(-13, np.log2(463.9), 200000))
    x = np.concatenate([mags * rng.choice([-1, 1], mags.size), _grid(), -_grid()])
    # every midpoint between neighbours: ties must go to the even mantissa
    g = _grid()
    mids = (g[:-1] + g[1:]) / 2
    x = np.concatenate([x, mids, -mids, [0.0, -0.0, 2.0 ** -10, 3 * 2.0 ** -10]])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = lp.round_e4m3(x)
    assert np.array_equal(mine, ref)


def test_saturation_reading_above_448():
    # torch's cast gives NaN from 464 up; the reading here saturates every magnitude at 448
    x = np.array([448.0, 463.9, 464.0, 500.0, 1e6, -1e30])
    assert np.array_equal(lp.round_e4m3(x), np.array([448, 448, 448, 448, 448, -448.0]))


def test_scale_exponent_is_the_binade_of_the_block_max_minus_8():
    rng = np.random.default_rng(72)
    amax = np.exp2(rng.uniform(-100, 100, 5000))
    X = lp.mx_scale_exponent(amax)
    # brute force: the unique integer with 2^(X+8) <= amax < 2^(X+9)
    lo = np.array([2.0 ** (int(t) + 8) for t in X])
    assert np.all((lo <= amax) & (amax < 2 * lo))
    assert lp.mx_scale_exponent(0.0) == -127
    assert lp.mx_scale_exponent(2.0 ** 200) == 127 and lp.mx_scale_exponent(2.0 ** -200) == -127


def test_block_quantisation_error_bound_and_round_trip():
    rng = np.random.default_rng(73)
    a = rng.standard_normal((64, 256)) * np.exp2(rng.integers(-20, 20, (64, 1)))
    a[3, 32:64] = 0.0                                           # an all-zero block
    q, X = lp.mxfp8_quantize(a)
    assert X.shape == (64, 8) and X[3, 1] == -127
    deq = lp.mxfp8_dequantize(q, X)
    scaled = np.ldexp(a.reshape(64, 8, 32), -X[..., None]).reshape(64, 256)
    # the block max lands in [256, 512) before rounding; below 448 the error is at most half a step
    bmax = np.abs(scaled.reshape(64, 8, 32)).max(-1)
    assert np.all((bmax[X > -127] >= 256) & (bmax[X > -127] < 512))
    ok = np.abs(scaled) <= lp.E4M3_MAX
    err = np.abs(q - scaled)
    assert np.all(err[ok] <= lp.e4m3_half_step(scaled)[ok])
    assert np.all(np.abs(q[~ok]) == lp.E4M3_MAX)
    assert np.array_equal(deq[3, 32:64], np.zeros(32))
    # values already on a block's grid come back unchanged
    q2, X2 = lp.mxfp8_quantize(deq)
    assert np.array_equal(lp.mxfp8_dequantize(q2, X2), deq)


def test_block_scaled_product_matches_the_dequantised_operands():
    rng = np.random.default_rng(74)
    a, b = rng.standard_normal((24, 128)), rng.standard_normal((40, 128))
    c = lp.mxfp8_matmul(a, b)
    qa, xa = lp.mxfp8_quantize(a)
    qb, xb = lp.mxfp8_quantize(b)
    ref = torch.from_numpy(lp.mxfp8_dequantize(qa, xa)) @ torch.from_numpy(lp.mxfp8_dequantize(qb, xb)).T
    np.testing.assert_allclose(c, ref.numpy(), rtol=1e-13, atol=1e-13)
    # and sits within the quantisation bound of the exact product: each element moves by at most
    # 1/8 of its magnitude (half a step, 2^-4, below 448 in scaled units; at most 64/512 where
    # (448, 512) saturates) or by half the subnormal step 2^-10 of its block's scale
    def err_bound(m, X):
        return np.maximum(2.0 ** -3 * np.abs(m), np.repeat(np.ldexp(1.0, X - 10), 32, axis=-1))
    ea, eb = err_bound(a, xa), err_bound(b, xb)
    bound = ea @ np.abs(b).T + np.abs(a) @ eb.T + ea @ eb.T
    assert np.all(np.abs(c - a @ b.T) <= bound)


_ROUND = lp.round_e4m3
_SCALE = lp.mx_scale_exponent

LOWP_MUTANTS = {
    # ties away from zero instead of to even
    "ties_away": ("round_e4m3",
                  lambda x: np.copysign(np.minimum(
                      np.floor(np.abs(np.asarray(x, float)) / (2 * lp.e4m3_half_step(x)) + 0.5)
                      * (2 * lp.e4m3_half_step(x)), lp.E4M3_MAX), x),
                  [test_rounding_matches_torch_cast_below_saturation]),
    # the scale one binade too small: block maxima land in [512, 1024) and saturate
    "scale_minus_7": ("mx_scale_exponent", lambda amax: _SCALE(amax) + 1,
                      [test_scale_exponent_is_the_binade_of_the_block_max_minus_8,
                       test_block_quantisation_error_bound_and_round_trip]),
    # no saturation: magnitudes above 448 keep their rounded value
    "no_saturation": ("round_e4m3",
                      lambda x: np.copysign(np.round(np.abs(np.asarray(x, float)) / (2 * lp.e4m3_half_step(x)))
                                            * (2 * lp.e4m3_half_step(x)), x),
                      [test_saturation_reading_above_448]),
}


def _fails(pin):
    try:
        pin()
    except (AssertionError, ValueError, IndexError):
        return True
    return False


@pytest.mark.parametrize("name", sorted(LOWP_MUTANTS))
def test_a_lowp_pin_catches_the_mutant(name, monkeypatch):
    target, mutant, pin_list = LOWP_MUTANTS[name]
    monkeypatch.setattr(lp, target, mutant)
    assert any(_fails(p) for p in pin_list), f"no pin caught mutant {name}"


def _expert_problem(seed=75):
    rng = np.random.default_rng(seed)
    T, l, h, E, k = 40, 64, 96, 5, 2
    hid = rng.standard_normal((T, l))
    w1, w3 = rng.standard_normal((E, h, l)) / 8, rng.standard_normal((E, h, l)) / 8
    w2 = rng.standard_normal((E, l, h)) / 10
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    return hid, idx, w1, w3, w2


def test_mxfp8_experts_are_exact_under_power_of_two_scaling_of_w2():
    """A power-of-two factor on W2 moves every block scale by the same power and no element:
    the 8-bit expert output scales by exactly that factor."""
    hid, idx, w1, w3, w2 = _expert_problem()
    o = lp.routed_outputs_mxfp8(hid, idx, w1, w3, w2)
    for j in (-5, 3):
        assert np.array_equal(lp.routed_outputs_mxfp8(hid, idx, w1, w3, np.ldexp(w2, j)), np.ldexp(o, j))


def test_mxfp8_experts_ignore_the_order_of_k_blocks():
    """Quantisation acts on 32-element blocks along K only: permuting whole blocks of l in h, W1
    and W3 together (and of h in W1, W3 rows and W2 columns together) changes no output beyond
    the float64 summation order."""
    hid, idx, w1, w3, w2 = _expert_problem()
    o = lp.routed_outputs_mxfp8(hid, idx, w1, w3, w2)
    pl = np.concatenate([np.arange(32, 64), np.arange(0, 32)])            # swap the two blocks of l
    ph = np.concatenate([np.arange(64, 96), np.arange(0, 32), np.arange(32, 64)])  # rotate h's blocks
    o2 = lp.routed_outputs_mxfp8(hid[:, pl], idx, w1[:, ph][:, :, pl], w3[:, ph][:, :, pl], w2[:, :, ph])
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-12)


def test_mxfp8_experts_stay_near_the_full_precision_experts():
    """A check of the wiring against the forward oracle's float64 experts: each 8-bit operand is
    within 1/8 of its value (the element pins above); through two GEMMs and the SwiGLU the outputs
    stay within 30% of the output scale (about 10% here), while a lost block scale or a misplaced
    operand moves them by orders of magnitude."""
    import oracle
    hid, idx, w1, w3, w2 = _expert_problem()
    o8 = lp.routed_outputs_mxfp8(hid, idx, w1, w3, w2)
    o = oracle.routed_outputs(hid, idx, w1, w3, w2)
    rel = np.max(np.abs(o8 - o)) / np.max(np.abs(o))
    assert 0 < rel < 0.3, rel


def test_layer_forward_mxfp8_with_an_identity_quantiser_is_the_forward_oracle():
    """With the quantiser replaced by the identity (elements = values, every scale 2^0), the
    8-bit layer is the forward oracle's layer: routing, combine, up-projection and shared expert
    are wired exactly as there, and only the experts' operands change with the format."""
    import datagen
    import oracle
    shape = datagen.LayerShape("mx_pin", 24, 64, 64, 8, 2, 64, 96, "f32", seed=77, offset_var=0.5)
    w = datagen.layer_weights(shape, gain="random")
    x = datagen.tokens(shape)
    b = datagen.normal_bias(shape.E, seed=77, std=0.1).astype(np.float64)
    real = lp.mxfp8_quantize
    try:
        lp.mxfp8_quantize = lambda a, block=32: (np.asarray(a, dtype=np.float64),
                                                 np.zeros(np.shape(a)[:-1] + (np.shape(a)[-1] // block,), int))
        y8 = lp.layer_forward_mxfp8(x, w, b, shape.k)
    finally:
        lp.mxfp8_quantize = real
    ref = oracle.layer_forward(x, w, b, shape.k)
    assert np.array_equal(y8["idx"], ref["idx"])
    np.testing.assert_allclose(y8["y"], ref["y"], rtol=1e-12, atol=1e-12)
    # and with the real quantiser it moves, within the 8-bit bound of the experts' part
    y8 = lp.layer_forward_mxfp8(x, w, b, shape.k)["y"]
    rel = np.max(np.abs(y8 - ref["y"])) / np.max(np.abs(ref["y"]))
    assert 0 < rel < 0.2, rel
