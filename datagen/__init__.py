"""Seeded synthetic inputs for the Stable-LatentMoE layer.

This module only draws random numbers and rounds them to the storage type
(fp32, or bf16 by round-to-nearest-even through torch's cast).  It holds none
of the layer's arithmetic, so both the CPU oracle (test infrastructure) and
the CUDA library take their inputs from here and from nowhere else.

Every stream is keyed by (seed, tensor id, sub-index), so one expert's
weights or one 1024-row chunk of tokens can be regenerated on its own: the
oracle recomputes a token subset of the 16384-token, 896-expert workload
without holding every expert in fp64.

Distributions follow the layer's five synthetic workloads (the pages give
only 896-choose-16 and top-6 routing): tokens x ~ N(0, 1); every weight ~ N(0, 1/fan_in) where
fan_in is the input width of that projection; RMSNorm gain 1; router column
offsets c_e ~ N(0, 0.5) (variance 0.5) where the workload says so.
"""
from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np
import torch

TOKEN_CHUNK = 1024  # rows of x drawn from one stream

# stream ids, one per tensor
_TID = {
    "w_down": 1, "w_router": 2, "w1": 3, "w3": 4, "w2": 5, "w_up": 6,
    "ws1": 7, "ws3": 8, "ws2": 9, "router_bias": 10, "x": 11, "rms_gain": 12,
    "bias": 13, "scores": 14, "dy": 15,
}


@dataclass(frozen=True)
class LayerShape:
    """Sizes of one LatentMoE layer workload.

    T tokens, backbone width d, latent width l, E routed experts, top-k,
    routed-expert SwiGLU hidden h, shared-expert hidden hs (0 = none).
    dtype is the storage/arithmetic type of activations and of every weight
    except the router, which is always fp32.
    """

    name: str
    T: int
    d: int
    l: int
    E: int
    k: int
    h: int
    hs: int
    dtype: str  # "f32" | "bf16"
    seed: int
    offset_var: float = 0.0   # variance of the router column offsets c_e
    beta: float = 0.0         # QB step size used by the workload
    steps: int = 1            # forward + QB-update steps of the workload
    rms_eps: float = 1e-6
    nbins: int = 4096

    def with_tokens(self, T: int) -> "LayerShape":
        return dataclasses.replace(self, T=T, name=f"{self.name}_T{T}")


WORKLOADS = {
    # fp32 throughout; one forward plus one QB update.
    "tiny_fp32": LayerShape("tiny_fp32", 256, 256, 64, 32, 4, 128, 512, "f32", seed=0, beta=0.01),
    # mini-replica scale: batch 4 x seq 2048, bf16, router offsets N(0, 0.5).
    "mini_replica": LayerShape("mini_replica", 8192, 1024, 256, 256, 6, 256, 2048, "bf16",
                               seed=1, offset_var=0.5),
    # full-width routing stress, 896 experts choose 16.
    "wide_stress": LayerShape("wide_stress", 16384, 7168, 2048, 896, 16, 512, 4096, "bf16", seed=2),
    # QB convergence run on a skewed router: 50 steps, beta 0.05, fresh x from seed 3+step.
    "qb_skewed": LayerShape("qb_skewed", 4096, 1024, 256, 128, 8, 256, 2048, "bf16",
                            seed=3, beta=0.05, steps=50),
    # the wide layer's routed-expert shape (l = 2048, h = 512, k = 16, about 292 rows per expert)
    # with 128 experts and d = 1024: the small case on which ncu captures the expert GEMMs.
    "wide_experts": LayerShape("wide_experts", 2336, 1024, 2048, 128, 16, 512, 1024, "bf16", seed=2),
    # large-batch sweep, T in SWEEP_T.
    "sweep": LayerShape("sweep", 262144, 1024, 256, 256, 6, 256, 2048, "bf16", seed=4, offset_var=0.5),
}
SWEEP_T = (1024, 4096, 16384, 65536, 262144)


def torch_dtype(shape: LayerShape) -> torch.dtype:
    return torch.float32 if shape.dtype == "f32" else torch.bfloat16


def _normal(seed: int, tid: int, sub: int, n: int) -> np.ndarray:
    rng = np.random.default_rng([seed, tid, sub])
    return rng.standard_normal(n, dtype=np.float32)


def _store(a: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    t = torch.from_numpy(a)
    return t if dtype == torch.float32 else t.to(dtype)


def _matrix(seed, name, rows, cols, fan_in, dtype, sub=0):
    v = _normal(seed, _TID[name], sub, rows * cols).reshape(rows, cols)
    v *= np.float32(1.0 / math.sqrt(fan_in))
    return _store(v, dtype)


def _experts(seed, name, E, rows, cols, fan_in, dtype):
    """Expert e's matrix comes from its own stream (sub-index e), so the experts are drawn on
    several host threads (numpy and torch release the GIL) with the same values as one by one."""
    out = torch.empty((E, rows, cols), dtype=dtype)

    def fill(e):
        out[e] = _matrix(seed, name, rows, cols, fan_in, dtype, sub=e)

    workers = min(16, os.cpu_count() or 1, E)
    if workers <= 1 or E * rows * cols < (1 << 22):
        for e in range(E):
            fill(e)
    else:
        with ThreadPoolExecutor(workers) as ex:
            list(ex.map(fill, range(E)))
    return out


def layer_weights(shape: LayerShape, seed: int | None = None, *, gain: str = "ones",
                  router_offsets: np.ndarray | None = None) -> dict[str, torch.Tensor]:
    """All weights of one layer as CPU tensors in the storage dtype.

    Layouts are (out, in), the nn.Linear convention:
      rms_gain [d]; w_down [l,d]; w_router [E,l] fp32; router_bias [E] fp32;
      w1, w3 [E,h,l]; w2 [E,l,h]; w_up [d,l]; ws1, ws3 [hs,d]; ws2 [d,hs].
    gain="random" draws g = 1 + 0.1 N(0,1) instead of ones.
    router_offsets, if given, replaces the drawn column offsets c.
    """
    s = shape.seed if seed is None else seed
    dt = torch_dtype(shape)
    d, l, E, h, hs = shape.d, shape.l, shape.E, shape.h, shape.hs
    w = {}
    if gain == "ones":
        w["rms_gain"] = torch.ones(d, dtype=dt)
    else:
        g = 1.0 + 0.1 * _normal(s, _TID["rms_gain"], 0, d)
        w["rms_gain"] = _store(g.astype(np.float32), dt)
    w["w_down"] = _matrix(s, "w_down", l, d, d, dt)
    w["w_router"] = _matrix(s, "w_router", E, l, l, torch.float32)
    if router_offsets is not None:
        w["router_bias"] = torch.from_numpy(np.asarray(router_offsets, dtype=np.float32).copy())
    elif shape.offset_var > 0:
        c = _normal(s, _TID["router_bias"], 0, E) * np.float32(math.sqrt(shape.offset_var))
        w["router_bias"] = torch.from_numpy(c)
    else:
        w["router_bias"] = torch.zeros(E, dtype=torch.float32)
    w["w1"] = _experts(s, "w1", E, h, l, l, dt)
    w["w3"] = _experts(s, "w3", E, h, l, l, dt)
    w["w2"] = _experts(s, "w2", E, l, h, h, dt)
    w["w_up"] = _matrix(s, "w_up", d, l, l, dt)
    if hs > 0:
        w["ws1"] = _matrix(s, "ws1", hs, d, d, dt)
        w["ws3"] = _matrix(s, "ws3", hs, d, d, dt)
        w["ws2"] = _matrix(s, "ws2", d, hs, hs, dt)
    return w


def tokens(shape: LayerShape, seed: int | None = None, rows=None, T: int | None = None) -> torch.Tensor:
    """x ~ N(0,1) of shape [T, d] (or only `rows`, any iterable of row ids).

    Rows are drawn in chunks of TOKEN_CHUNK from per-chunk streams, so a row
    subset regenerates exactly the same values as the full matrix.
    """
    s = shape.seed if seed is None else seed
    dt = torch_dtype(shape)
    T = shape.T if T is None else T
    d = shape.d
    if rows is None:
        out = np.empty((T, d), dtype=np.float32)
        for c0 in range(0, T, TOKEN_CHUNK):
            n = min(TOKEN_CHUNK, T - c0)
            out[c0:c0 + n] = _normal(s, _TID["x"], c0 // TOKEN_CHUNK, TOKEN_CHUNK * d).reshape(
                TOKEN_CHUNK, d)[:n]
        return _store(out, dt)
    rows = np.asarray(list(rows), dtype=np.int64)
    out = np.empty((len(rows), d), dtype=np.float32)
    for c in np.unique(rows // TOKEN_CHUNK):
        blk = _normal(s, _TID["x"], int(c), TOKEN_CHUNK * d).reshape(TOKEN_CHUNK, d)
        sel = np.nonzero(rows // TOKEN_CHUNK == c)[0]
        out[sel] = blk[rows[sel] - c * TOKEN_CHUNK]
    return _store(out, dt)


def output_grad(shape: LayerShape, seed: int | None = None, T: int | None = None,
                scale: float = 1.0) -> torch.Tensor:
    """dL/dy ~ scale * N(0,1) of shape [T, d] in the layer's dtype (the output gradient of a
    backward pass), drawn in chunks of TOKEN_CHUNK rows like tokens()."""
    s = shape.seed if seed is None else seed
    T = shape.T if T is None else T
    d = shape.d
    out = np.empty((T, d), dtype=np.float32)
    for c0 in range(0, T, TOKEN_CHUNK):
        n = min(TOKEN_CHUNK, T - c0)
        out[c0:c0 + n] = _normal(s, _TID["dy"], c0 // TOKEN_CHUNK, TOKEN_CHUNK * d).reshape(TOKEN_CHUNK, d)[:n]
    if scale != 1.0:
        out *= np.float32(scale)
    return _store(out, torch_dtype(shape))


def uniform_scores(T: int, E: int, seed: int, quantise: int = 0) -> np.ndarray:
    """Router-score-like fp32 values in [0,1] for stage tests that start from scores.

    quantise > 0 snaps them to a grid of that many steps, which plants exact ties.
    """
    rng = np.random.default_rng([seed, _TID["scores"], 0])
    s = rng.random((T, E), dtype=np.float32)
    if quantise:
        s = (np.floor(s * quantise) / quantise).astype(np.float32)
    return s


def normal_bias(E: int, seed: int, std: float) -> np.ndarray:
    """A per-expert fp32 bias b ~ N(0, std^2), for routing tests with a non-zero bias."""
    return (_normal(seed, _TID["bias"], 0, E) * np.float32(std)).astype(np.float32)
