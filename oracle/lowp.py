"""CPU oracle for block-scaled 8-bit operands (MXFP8: E4M3 elements, power-of-two block scales).

TEST INFRASTRUCTURE, under the same rule as the rest of this package: only tests/,
__graft_entry__.smoke() and the CPU legs of bench.py may import it, and it imports nothing from
the CUDA library.

The pages say only that the K3 model runs its experts with 4-bit weights and 8-bit activations
("Kimi K3登顶开源第一，靠的是把浪费逼到墙角", the QAT paragraph) and that the replica's FP8 attempt
lost on H200 (the wink.run summary of "Pretraining a Mini Kimi K3": 0.19x).  They fix no format,
block size or scale rule.  Readings taken (the plainest that block-scaled tensor-core operands
support):
  * Elements are E4M3: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no infinities,
    largest finite magnitude 448 (exponent field 15, mantissa 110), subnormals down to 2^-9.
    A value is rounded to the nearest element, ties to the even mantissa, and magnitudes beyond
    448 saturate to 448.
  * One power-of-two scale 2^X per 32 consecutive elements along K, the reduction axis, with
    X = floor(log2(max |v| of the block)) - 8 (8 is the exponent of E4M3's largest binade), so the
    block's largest magnitude lands in [256, 512) before rounding (and saturates above 448);
    X is clamped to [-127, 127] (the range of an 8-bit exponent-only scale); an all-zero block
    takes X = -127.
  * A product of two such operands is the float64 product of their dequantised values
    (element * 2^X): the tensor core multiplies the elements exactly and accumulates in fp32; this
    oracle is that product without the accumulation's rounding.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_MIN_NORMAL = 2.0 ** -6
E4M3_SUBNORMAL_STEP = 2.0 ** -9
E4M3_EMAX = 8        # exponent of the largest binade, [256, 512)
MX_BLOCK = 32
SCALE_EXP_MIN, SCALE_EXP_MAX = -127, 127


def e4m3_decode(code: int) -> float:
    """Value of one E4M3 byte from its bit fields (sign, 4-bit exponent with bias 7, 3-bit
    mantissa); exponent field 15 with mantissa 111 is NaN, there are no infinities."""
    sign = -1.0 if code & 0x80 else 1.0
    e, m = (code >> 3) & 0xF, code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * m * 2.0 ** -9            # subnormal: m/8 * 2^(1-7)
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def round_e4m3(x) -> np.ndarray:
    """Nearest E4M3 value of each element (ties to the even mantissa), saturating at +-448."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    # the spacing of the grid at |a|: 2^(e-3) in the binade [2^e, 2^(e+1)), 2^-9 below 2^-6
    _, ex = np.frexp(np.where(a > 0, a, 1.0))   # a = m 2^ex with m in [0.5, 1): binade e = ex - 1
    step = np.where(a >= E4M3_MIN_NORMAL, np.ldexp(1.0, ex - 1 - 3), E4M3_SUBNORMAL_STEP)
    q = np.round(a / step) * step              # np.round rounds halves to even; a / step is exact
    return np.copysign(np.minimum(q, E4M3_MAX), x)


def mx_scale_exponent(block_amax) -> np.ndarray:
    """X = floor(log2(amax)) - 8, clamped to [-127, 127]; -127 for an all-zero block."""
    amax = np.asarray(block_amax, dtype=np.float64)
    _, ex = np.frexp(np.where(amax > 0, amax, 1.0))
    X = np.where(amax > 0, ex - 1 - E4M3_EMAX, SCALE_EXP_MIN)
    return np.clip(X, SCALE_EXP_MIN, SCALE_EXP_MAX).astype(np.int64)


def mxfp8_quantize(a, block: int = MX_BLOCK):
    """Block-scaled E4M3 encoding of `a` along its last axis (K, a multiple of `block`).

    Returns (elements, X): elements are float64 values on the E4M3 grid, shape of `a`; X holds one
    scale exponent per block, shape a.shape[:-1] + (K / block,)."""
    a = np.asarray(a, dtype=np.float64)
    K = a.shape[-1]
    if K % block:
        raise ValueError("K must be a multiple of the block size")
    blocks = a.reshape(a.shape[:-1] + (K // block, block))
    X = mx_scale_exponent(np.abs(blocks).max(axis=-1))
    elems = round_e4m3(np.ldexp(blocks, -X[..., None]))
    return elems.reshape(a.shape), X


def mxfp8_dequantize(elems, X, block: int = MX_BLOCK) -> np.ndarray:
    """element * 2^X of its block."""
    elems = np.asarray(elems, dtype=np.float64)
    K = elems.shape[-1]
    blocks = elems.reshape(elems.shape[:-1] + (K // block, block))
    return np.ldexp(blocks, np.asarray(X)[..., None]).reshape(elems.shape)


def mxfp8_matmul(a, b, block: int = MX_BLOCK) -> np.ndarray:
    """C = A B^T for A [M, K] and B [N, K], each quantised to MXFP8 along K first."""
    qa, xa = mxfp8_quantize(a, block)
    qb, xb = mxfp8_quantize(b, block)
    return mxfp8_dequantize(qa, xa, block) @ mxfp8_dequantize(qb, xb, block).T


def e4m3_half_step(v) -> np.ndarray:
    """Half the E4M3 grid spacing at |v| (the largest rounding error there, below saturation)."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    step = np.where(a >= E4M3_MIN_NORMAL, np.ldexp(1.0, ex - 1 - 3), E4M3_SUBNORMAL_STEP)
    return step / 2




def routed_outputs_mxfp8(h, idx, w1, w3, w2, block: int = MX_BLOCK) -> np.ndarray:
    """o[t, i] = SwiGLU_{idx[t,i]}(h[t]) with every GEMM operand in MXFP8, for each chosen pair.

    The same expert FFN as the forward oracle's routed_outputs (SwiGLU, the stand-in for SiTU-GLU),
    with 8-bit operands: the expert's rows of h and its W1, W3 are quantised along l (their K),
    act = silu(p1) * p3 and W2 along h; each product is the float64 product of the dequantised
    operands, and silu and the elementwise product are float64 as well."""
    h = _f64(h)
    T, k = idx.shape
    o = np.zeros((T, k, np.shape(w2)[1]), dtype=np.float64)
    for e in np.unique(idx):
        t, i = np.nonzero(idx == e)
        a = h[t]
        p1 = mxfp8_matmul(a, _f64(w1[e]), block)
        p3 = mxfp8_matmul(a, _f64(w3[e]), block)
        act = p1 / (1.0 + np.exp(-p1)) * p3
        o[t, i] = mxfp8_matmul(act, _f64(w2[e]), block)
    return o


def _f64(a) -> np.ndarray:
    """An input (numpy array, or a CPU torch tensor of any float type) widened exactly to float64."""
    if hasattr(a, "detach"):
        import torch
        return a.detach().to(torch.float64).numpy()
    return np.asarray(a, dtype=np.float64)


def layer_forward_mxfp8(x, w: dict, b, k: int, eps: float = 1e-6, block: int = MX_BLOCK) -> dict:
    """The whole layer with MXFP8 routed experts: the forward oracle's steps in its order, with
    routed_outputs replaced by routed_outputs_mxfp8 (the routing, the gates, the combine, the
    up-projection and the shared expert stay float64).  Returns y and the routing."""
    import oracle
    xf = oracle.f64(x)
    x_hat = oracle.rmsnorm(xf, oracle.f64(w["rms_gain"]), eps)
    r = oracle.layer_routing(x, w, b, k, eps)
    o = routed_outputs_mxfp8(r["h"], r["idx"], w["w1"], w["w3"], w["w2"], block)
    z = oracle.combine(r["gates"], o)
    y = oracle.up_projection(z, oracle.f64(w["w_up"]))
    if "ws1" in w:
        y = y + oracle.shared_expert(x_hat, oracle.f64(w["ws1"]), oracle.f64(w["ws3"]), oracle.f64(w["ws2"]))
    return dict(r, o=o, z=z, y=y)


__all__ = ["E4M3_MAX", "MX_BLOCK", "e4m3_decode", "round_e4m3", "mx_scale_exponent", "mxfp8_quantize",
           "mxfp8_dequantize", "mxfp8_matmul", "e4m3_half_step", "routed_outputs_mxfp8",
           "layer_forward_mxfp8"]
