"""Python binding of liblmoe.so, the B200 Stable-LatentMoE layer with Quantile Balancing.

Argument marshalling only: every step of the layer runs in the CUDA kernels behind the C ABI
(include/lmoe.h).  torch supplies device memory and streams.  If the library is not built the
import of the binding still works, but the first call raises: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int, c_int32, c_size_t, c_uint32, c_void_p

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblmoe.so")

F32, BF16 = 0, 1
EXPERTS_BF16, EXPERTS_MXFP8 = 0, 1
RECORD_STATS = 1
UPDATE_BIAS = 4
ASYNC_OUTPUT = 8
QB_LITERAL = 1
BIAS_SIGN = 2
STATUS_NAN_SCORE, STATUS_WATCHDOG, STATUS_BAD_INDEX = 1, 2, 4
NBINS = 4096

EXPORTED = (
    "lmoe_create", "lmoe_destroy", "lmoe_workspace_bytes", "lmoe_forward", "lmoe_forward_host", "lmoe_host_wait",
    "lmoe_qb_update", "lmoe_set_update", "lmoe_route_scores", "lmoe_get_routing", "lmoe_get_bias", "lmoe_set_bias",
    "lmoe_get_hist", "lmoe_set_hist", "lmoe_get_load", "lmoe_set_load", "lmoe_get_status", "lmoe_strerror", "lmoe_gemm_bf16",
    "lmoe_profile_enable", "lmoe_profile_read", "lmoe_stage_name", "lmoe_launch_count",
    "lmoe_route_noalloc", "lmoe_watchdog_selftest", "lmoe_gemm_bf16_ex", "lmoe_forward_backward",
)
NUM_STAGES = 14


class LmoeError(RuntimeError):
    pass


class lmoe_config(ctypes.Structure):
    _fields_ = [("d", c_int32), ("l", c_int32), ("E", c_int32), ("k", c_int32), ("h", c_int32),
                ("hs", c_int32), ("dtype", c_int32), ("nbins", c_int32), ("rms_eps", c_float),
                ("max_tokens", c_int32), ("experts", c_int32)]


class lmoe_weights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in ("rms_gain", "w_down", "w_router", "router_bias", "w1", "w3",
                                         "w2", "w_up", "ws1", "ws3", "ws2")]


class lmoe_grads(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in ("dx", "rms_gain", "w_down", "w_router", "router_bias", "w1", "w3", "w2",
                                         "w_up", "ws1", "ws3", "ws2")]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise LmoeError(f"{LIB_PATH} is missing: build it with `python -m latent_routing_quantile_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, u32 = c_void_p, c_int32, c_uint32
        sig = {
            "lmoe_create": [POINTER(lmoe_config), POINTER(lmoe_weights), vp, POINTER(vp)],
            "lmoe_destroy": [vp],
            "lmoe_workspace_bytes": [POINTER(lmoe_config), POINTER(c_size_t)],
            "lmoe_forward": [vp, vp, vp, i32, u32, vp],
            "lmoe_forward_host": [vp, vp, vp, i32, u32, vp],
            "lmoe_host_wait": [vp, vp],
            "lmoe_qb_update": [vp, c_float, u32, vp],
            "lmoe_set_update": [vp, c_float, u32],
            "lmoe_route_scores": [vp, vp, i32, u32, vp],
            "lmoe_get_routing": [vp, vp, vp, vp, vp, vp, vp, vp, vp],
            "lmoe_get_bias": [vp, vp, vp],
            "lmoe_set_bias": [vp, vp, vp],
            "lmoe_get_hist": [vp, vp, vp, vp],
            "lmoe_set_hist": [vp, vp, vp, vp],
            "lmoe_get_load": [vp, vp, vp],
            "lmoe_set_load": [vp, vp, vp],
            "lmoe_get_status": [vp, POINTER(u32)],
            "lmoe_gemm_bf16": [vp, vp, vp, i32, i32, i32, vp],
            "lmoe_gemm_bf16_ex": [vp, i32, vp, i32, vp, i32, i32, i32, i32, vp],
            "lmoe_forward_backward": [vp, POINTER(lmoe_weights), vp, vp, vp, i32, u32, POINTER(lmoe_grads), vp],
            "lmoe_profile_enable": [vp, i32],
            "lmoe_profile_read": [vp, POINTER(c_float), i32, POINTER(i32)],
            "lmoe_launch_count": [vp, POINTER(ctypes.c_int64)],
            "lmoe_route_noalloc": [vp, vp, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp],
            "lmoe_watchdog_selftest": [vp, i32, vp],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = c_int
        L.lmoe_strerror.argtypes = [c_int]
        L.lmoe_strerror.restype = ctypes.c_char_p
        L.lmoe_stage_name.argtypes = [c_int32]
        L.lmoe_stage_name.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(rc: int, what: str):
    if rc != 0:
        raise LmoeError(f"{what}: {lib().lmoe_strerror(rc).decode()} ({rc})")


def _ptr(t):
    return None if t is None else c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return c_void_p(s.cuda_stream)


def _dev(t: torch.Tensor, dtype=None, shape=None, name="tensor"):
    if not t.is_cuda or not t.is_contiguous():
        raise LmoeError(f"{name} must be a contiguous CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise LmoeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise LmoeError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


class Layer:
    """One LatentMoE layer handle (lmoe_create ... lmoe_destroy).

    weights: dict of CUDA tensors named as in lmoe_weights (rms_gain, w_down, w_router,
    router_bias, w1, w3, w2, w_up, ws1, ws3, ws2), layouts (out, in).
    """

    def __init__(self, d, l, E, k, h, hs, dtype, max_tokens, weights, rms_eps=1e-6, stream=None,
                 experts=EXPERTS_BF16):
        self.cfg = lmoe_config(d, l, E, k, h, hs, dtype, NBINS, rms_eps, max_tokens, experts)
        self.dtype = torch.float32 if dtype == F32 else torch.bfloat16
        dt = self.dtype
        shapes = {"rms_gain": ((d,), dt), "w_down": ((l, d), dt), "w_router": ((E, l), torch.float32),
                  "router_bias": ((E,), torch.float32), "w1": ((E, h, l), dt), "w3": ((E, h, l), dt),
                  "w2": ((E, l, h), dt), "w_up": ((d, l), dt)}
        if hs:
            shapes.update({"ws1": ((hs, d), dt), "ws3": ((hs, d), dt), "ws2": ((d, hs), dt)})
        w = lmoe_weights()
        for name, (shape, tdt) in shapes.items():
            t = weights.get(name)
            if t is not None:
                _dev(t, tdt, shape, name)
                setattr(w, name, t.data_ptr())
        self._keep = dict(weights)
        self.handle = c_void_p()
        _check(lib().lmoe_create(ctypes.byref(self.cfg), ctypes.byref(w), _stream(stream),
                                 ctypes.byref(self.handle)), "lmoe_create")
        (torch.cuda.current_stream() if stream is None else stream).synchronize()
        self._keep = None
        self.last_T = 0

    # ---------------------------------------------------------------- forward
    @staticmethod
    def _fwd_flags(record_stats, update_bias):
        # update_bias records this forward's statistics too (the update counts them)
        return (RECORD_STATS if (record_stats or update_bias) else 0) | (UPDATE_BIAS if update_bias else 0)

    def forward(self, x, y=None, record_stats=False, update_bias=False, stream=None):
        """update_bias=True also runs the bias update set by set_update inside this forward."""
        T = x.shape[0]
        _dev(x, self.dtype, (T, self.cfg.d), "x")
        if y is None:
            y = torch.empty_like(x)
        _dev(y, self.dtype, (T, self.cfg.d), "y")
        _check(lib().lmoe_forward(self.handle, _ptr(x), _ptr(y), T, self._fwd_flags(record_stats, update_bias),
                                  _stream(stream)), "lmoe_forward")
        self.last_T = T
        return y

    GRAD_NAMES = ("x", "rms_gain", "w_down", "w_router", "router_bias", "w1", "w3", "w2", "w_up", "ws1", "ws3",
                  "ws2")

    def forward_backward(self, x, dy, weights, y=None, record_stats=False, grads=None, stream=None):
        """One training step's layer work (lmoe_forward_backward): y = forward(x) and the fp32
        gradients of sum(y * dy) with respect to x and every weight, returned as a dict keyed like
        the weights (plus "x").  `weights` are the device tensors the layer was created from.
        `grads` may pass preallocated fp32 buffers."""
        c = self.cfg
        T = x.shape[0]
        _dev(x, self.dtype, (T, c.d), "x")
        _dev(dy, self.dtype, (T, c.d), "dy")
        if y is None:
            y = torch.empty_like(x)
        _dev(y, self.dtype, (T, c.d), "y")
        shapes = {"x": (T, c.d), "rms_gain": (c.d,), "w_down": (c.l, c.d), "w_router": (c.E, c.l),
                  "router_bias": (c.E,), "w1": (c.E, c.h, c.l), "w3": (c.E, c.h, c.l), "w2": (c.E, c.l, c.h),
                  "w_up": (c.d, c.l)}
        if c.hs:
            shapes.update({"ws1": (c.hs, c.d), "ws3": (c.hs, c.d), "ws2": (c.d, c.hs)})
        g = dict(grads or {})
        for n, shp in shapes.items():
            if n not in g:
                g[n] = torch.empty(shp, dtype=torch.float32, device=x.device)
            _dev(g[n], torch.float32, shp, "grad " + n)
        w = lmoe_weights()
        for n in ("rms_gain", "w_down", "w_router", "router_bias", "w1", "w3", "w2", "w_up", "ws1", "ws3", "ws2"):
            t = weights.get(n)
            if t is not None:
                setattr(w, n, _dev(t, None, None, n).data_ptr())
        gs = lmoe_grads()
        for n in shapes:
            setattr(gs, "dx" if n == "x" else n, g[n].data_ptr())
        _check(lib().lmoe_forward_backward(self.handle, ctypes.byref(w), _ptr(x), _ptr(dy), _ptr(y), T,
                                           self._fwd_flags(record_stats, False), ctypes.byref(gs), _stream(stream)),
               "lmoe_forward_backward")
        self.last_T = T
        return y, g

    def forward_host(self, x_host, y_host, record_stats=False, update_bias=False, async_output=False,
                     stream=None):
        """Host tensors (pinned for asynchronous copies); y_host is valid after the stream syncs,
        or with async_output=True after host_wait() and a sync of that stream."""
        T = x_host.shape[0]
        if x_host.is_cuda or y_host.is_cuda or x_host.dtype != self.dtype or y_host.dtype != self.dtype:
            raise LmoeError("forward_host takes host tensors of the layer dtype")
        _check(lib().lmoe_forward_host(self.handle, c_void_p(x_host.data_ptr()), c_void_p(y_host.data_ptr()), T,
                                       self._fwd_flags(record_stats, update_bias) | (ASYNC_OUTPUT if async_output else 0),
                                       _stream(stream)),
               "lmoe_forward_host")
        self.last_T = T
        return y_host

    def host_wait(self, stream=None):
        """Makes the stream wait for every async_output copy enqueued so far."""
        _check(lib().lmoe_host_wait(self.handle, _stream(stream)), "lmoe_host_wait")

    def route_scores(self, scores, record_stats=False, stream=None):
        T = scores.shape[0]
        _dev(scores, torch.float32, (T, self.cfg.E), "scores")
        _check(lib().lmoe_route_scores(self.handle, _ptr(scores), T, RECORD_STATS if record_stats else 0,
                                       _stream(stream)), "lmoe_route_scores")
        self.last_T = T

    def qb_update(self, beta, literal=False, sign_rule=False, stream=None):
        """Bias update from the recorded statistics: Quantile Balancing, or with sign_rule=True the
        aux-loss-free rule b_e += beta * sign(mean load - load_e)."""
        flags = (QB_LITERAL if literal else 0) | (BIAS_SIGN if sign_rule else 0)
        _check(lib().lmoe_qb_update(self.handle, float(beta), flags, _stream(stream)), "lmoe_qb_update")

    def set_update(self, beta, literal=False, sign_rule=False):
        """Step and rule of the update that forward(..., update_bias=True) runs after its routing."""
        flags = (QB_LITERAL if literal else 0) | (BIAS_SIGN if sign_rule else 0)
        _check(lib().lmoe_set_update(self.handle, float(beta), flags), "lmoe_set_update")

    # ---------------------------------------------------------------- introspection
    def routing(self, stream=None):
        T, k, E = self.last_T, self.cfg.k, self.cfg.E
        dev = torch.device("cuda")
        out = dict(idx=torch.empty((T, k), dtype=torch.int32, device=dev),
                   gates=torch.empty((T, k), dtype=torch.float32, device=dev),
                   scores=torch.empty((T, E), dtype=torch.float32, device=dev),
                   counts=torch.empty(E, dtype=torch.int32, device=dev),
                   offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
                   perm=torch.empty(T * k, dtype=torch.int32, device=dev),
                   inv=torch.empty(T * k, dtype=torch.int32, device=dev))
        _check(lib().lmoe_get_routing(self.handle, *(_ptr(out[n]) for n in
                                                     ("idx", "gates", "scores", "counts", "offsets", "perm", "inv")),
                                      _stream(stream)), "lmoe_get_routing")
        return out

    def bias(self, stream=None):
        b = torch.empty(self.cfg.E, dtype=torch.float32, device="cuda")
        _check(lib().lmoe_get_bias(self.handle, _ptr(b), _stream(stream)), "lmoe_get_bias")
        return b

    def set_bias(self, b, stream=None):
        _dev(b, torch.float32, (self.cfg.E,), "b")
        _check(lib().lmoe_set_bias(self.handle, _ptr(b), _stream(stream)), "lmoe_set_bias")

    def hist(self, stream=None):
        hist = torch.empty((self.cfg.E, NBINS), dtype=torch.int32, device="cuda")
        n = torch.empty(1, dtype=torch.int64, device="cuda")
        _check(lib().lmoe_get_hist(self.handle, _ptr(hist), _ptr(n), _stream(stream)), "lmoe_get_hist")
        return hist, n

    def set_hist(self, hist, ntok, stream=None):
        _dev(hist, torch.int32, (self.cfg.E, NBINS), "hist")
        _dev(ntok, torch.int64, (1,), "ntok")
        _check(lib().lmoe_set_hist(self.handle, _ptr(hist), _ptr(ntok), _stream(stream)), "lmoe_set_hist")

    def load(self, stream=None):
        load = torch.empty(self.cfg.E, dtype=torch.int64, device="cuda")
        _check(lib().lmoe_get_load(self.handle, _ptr(load), _stream(stream)), "lmoe_get_load")
        return load

    def set_load(self, load, stream=None):
        _dev(load, torch.int64, (self.cfg.E,), "load")
        _check(lib().lmoe_set_load(self.handle, _ptr(load), _stream(stream)), "lmoe_set_load")

    def profile(self, enable: bool = True):
        _check(lib().lmoe_profile_enable(self.handle, 1 if enable else 0), "lmoe_profile_enable")

    def profile_read(self):
        """(per-stage milliseconds summed over the recorded calls, number of recorded forwards)."""
        ms = (c_float * NUM_STAGES)()
        calls = c_int32(0)
        _check(lib().lmoe_profile_read(self.handle, ms, NUM_STAGES, ctypes.byref(calls)), "lmoe_profile_read")
        return {stage_name(i): ms[i] for i in range(NUM_STAGES)}, calls.value

    def launches(self) -> int:
        n = ctypes.c_int64(0)
        _check(lib().lmoe_launch_count(self.handle, ctypes.byref(n)), "lmoe_launch_count")
        return n.value

    def status(self) -> int:
        v = c_uint32(0)
        _check(lib().lmoe_get_status(self.handle, ctypes.byref(v)), "lmoe_get_status")
        return v.value

    def close(self):
        if self.handle:
            _check(lib().lmoe_destroy(self.handle), "lmoe_destroy")
            self.handle = c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def watchdog_selftest(limit_us: int = 20000, stream=None) -> int:
    """Runs the bounded-wait check (a wait on a barrier nothing completes) and returns the status word."""
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    _check(lib().lmoe_watchdog_selftest(_ptr(st), int(limit_us), _stream(stream)), "lmoe_watchdog_selftest")
    torch.cuda.synchronize()
    return int(st.item()) & 0xffffffff


def stage_name(i: int) -> str:
    return lib().lmoe_stage_name(i).decode()


def workspace_bytes(d, l, E, k, h, hs, dtype, max_tokens, rms_eps=1e-6, experts=EXPERTS_BF16) -> int:
    cfg = lmoe_config(d, l, E, k, h, hs, dtype, NBINS, rms_eps, max_tokens, experts)
    n = c_size_t(0)
    _check(lib().lmoe_workspace_bytes(ctypes.byref(cfg), ctypes.byref(n)), "lmoe_workspace_bytes")
    return n.value


def gemm_bf16(a, b, stream=None):
    """C = A B^T on the tensor-core engine (fp32 result), for checks of the engine itself."""
    M, K = a.shape
    N = b.shape[0]
    _dev(a, torch.bfloat16, (M, K), "a")
    _dev(b, torch.bfloat16, (N, K), "b")
    c = torch.empty((M, N), dtype=torch.float32, device=a.device)
    _check(lib().lmoe_gemm_bf16(_ptr(a), _ptr(b), _ptr(c), M, N, K, _stream(stream)), "lmoe_gemm_bf16")
    return c


def gemm_bf16_ex(a, b, a_mn=False, b_mn=False, k_split=1, stream=None):
    """C = op(A) op(B)^T with op(A) = A ([M, K]) or, a_mn, A^T of A stored [K, M]; likewise B
    ([N, K], or stored [K, N] with b_mn).  k_split > 1 adds K-range partial products by TMA
    reductions.  For checks of the engine's MN-major operands and split K."""
    M, K = (a.shape[1], a.shape[0]) if a_mn else a.shape
    N = b.shape[1] if b_mn else b.shape[0]
    _dev(a, torch.bfloat16, None, "a")
    _dev(b, torch.bfloat16, None, "b")
    if (b.shape[0] if b_mn else b.shape[1]) != K:
        raise LmoeError("A and B disagree on K")
    c = torch.empty((M, N), dtype=torch.float32, device=a.device)
    _check(lib().lmoe_gemm_bf16_ex(_ptr(a), int(a_mn), _ptr(b), int(b_mn), _ptr(c), M, N, K, k_split,
                                   _stream(stream)), "lmoe_gemm_bf16_ex")
    return c


def sum_qb_statistics(hist, ntok, load=None, group=None):
    """The data-parallel exchange step of the bias update: sums the integer histograms [E, 4096],
    token counts and (for the sign rule) expert loads [E] of all ranks in place (torch.distributed
    all-reduce), so every rank then applies the same bias update as one device that saw every
    token."""
    import torch.distributed as dist
    dist.all_reduce(hist, group=group)
    dist.all_reduce(ntok, group=group)
    if load is not None:
        dist.all_reduce(load, group=group)
    return hist, ntok, load


def dp_qb_update(layer, beta, literal=False, sign_rule=False, group=None, stream=None):
    """The data-parallel bias update, on every rank of `group`: read this rank's statistics
    recorded since the last update (histogram, token count and, for the sign rule, expert loads),
    sum them over the ranks with sum_qb_statistics, set the sums back, and run the update.  Every
    rank then applies the update one device would apply after seeing every rank's tokens, and all
    ranks keep the same bias ("Pretraining a Mini Kimi K3", capsule 27, Bug 2: the all-reduce
    comes before the update)."""
    hist, n = layer.hist(stream)
    load = layer.load(stream) if sign_rule else None
    sum_qb_statistics(hist, n, load, group)
    layer.set_hist(hist, n, stream)
    if load is not None:
        layer.set_load(load, stream)
    layer.qb_update(beta, literal=literal, sign_rule=sign_rule, stream=stream)


def dp_train_step(layer, x, dy, weights, beta=None, literal=False, sign_rule=False, group=None, grads=None,
                  stream=None):
    """One data-parallel training step's layer work on every rank of `group`: forward_backward of
    this rank's tokens (QB statistics recorded), then the exchange: every weight gradient summed
    over the ranks with one all-reduce each (the loss is the sum over all ranks' tokens, so its
    gradient is the sum of the ranks' own; dL/dx stays per rank), and, when beta is given, the
    ranks' QB statistics summed and the bias updated (dp_qb_update).  Returns (y, grads)."""
    import torch.distributed as dist
    y, g = layer.forward_backward(x, dy, weights, record_stats=True, grads=grads, stream=stream)
    for name, t in g.items():
        if name != "x":
            dist.all_reduce(t, group=group)
    if beta is not None:
        dp_qb_update(layer, beta, literal=literal, sign_rule=sign_rule, group=group, stream=stream)
    return y, g


def route_noalloc(scores, bias, k, out=None, stream=None):
    """Routing of fp32 scores [T, E] with bias [E] through lmoe_route_noalloc, which allocates no
    device memory (its scratch is a static array in the library).  `out` may pass preallocated
    buffers (idx, gates, counts, offsets, perm, inv, status); missing ones are allocated here by
    torch.  out["status"] (one int32 word) holds the call's fault bits once the stream syncs."""
    T, E = scores.shape
    _dev(scores, torch.float32, (T, E), "scores")
    _dev(bias, torch.float32, (E,), "bias")
    dev = scores.device
    shapes = dict(idx=((T, k), torch.int32), gates=((T, k), torch.float32), counts=((E,), torch.int32),
                  offsets=((E + 1,), torch.int32), perm=((T * k,), torch.int32), inv=((T * k,), torch.int32),
                  status=((1,), torch.int32))
    out = dict(out or {})
    for n, (shp, dt) in shapes.items():
        if n not in out:
            out[n] = torch.empty(shp, dtype=dt, device=dev)
        _dev(out[n], dt, shp, n)
    _check(lib().lmoe_route_noalloc(_ptr(scores), _ptr(bias), T, E, k,
                                    *(_ptr(out[n]) for n in ("idx", "gates", "counts", "offsets", "perm", "inv",
                                                             "status")),
                                    _stream(stream)), "lmoe_route_noalloc")
    return out


def layer_from_weights(shape, weights_cpu: dict, max_tokens=None, device="cuda", stream=None,
                       experts=EXPERTS_BF16) -> Layer:
    """Creates a Layer from the CPU weight dict of the seeded generator (copied to the device)."""
    w = {n: t.to(device) for n, t in weights_cpu.items()}
    return Layer(shape.d, shape.l, shape.E, shape.k, shape.h, shape.hs,
                 F32 if shape.dtype == "f32" else BF16, max_tokens or shape.T, w,
                 rms_eps=shape.rms_eps, stream=stream, experts=experts)
