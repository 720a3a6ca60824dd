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
