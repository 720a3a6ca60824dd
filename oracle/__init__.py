"""CPU oracle for the Stable-LatentMoE layer forward and Quantile Balancing.

TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and the CPU
baseline / reference leg of bench.py may import this package.  The CUDA
library never imports, links or calls it, and this package imports nothing
from the library: the two share only the seeded input generator (datagen).

What it is: the layer's definition written out in float64 numpy, one step
per function, in the order the layer applies them, with no blocking, fusion
or reordering beyond what each definition states.  A numpy matmul, sort or
cumulative sum serves as a library step.

Sources, cited by page title and section:
  [demo]  "KimiK3MoE架构轻量化复刻演示上线,12个交互模块详解StableLatentMoE设计逻辑"
          (tech.news18a.com/article/17573): Tab 1 data flow (width
          separation, shared/routed dual path), Tab 2 / Figure 2(a)(b)
          (QB load balance 3.7 -> 1.5, histogram-vs-exact quantile error
          0.0027), Tab 3 forward contract, Tab 5 RMSNorm, Tab 8-11 QB
          (bias only reroutes, weight normalisation, delayed update, mean
          centring, frozen at inference, single-step convergence),
          Tab 12 SiTU-GLU.
  [course] "Attention→K3 三十天课 · Day 28" (ai.air7.fun): design survival
          table (Stable LatentMoE 896 choose 16, QB, RMSNorm).
  [ebook] "免费电子书:Pretraining a Mini Kimi K3" (g.15386.cn): capsule 16
          (aux-loss-free sign rule for the bias, gamma 1e-2), capsule 20 and 25 (batched experts,
          dispatch buffer without silent fallback), capsule 27 Bug 2
          (all-reduce of load statistics before the bias update).
  [blog]  "Kimi K3登顶开源第一，靠的是把浪费逼到墙角" (cge.wang): latent
          experts compress first; QB raises the bar for hot experts.

The pages give no formula for SiTU-GLU, the router or RMSNorm.  The layer
contract this library implements fixes them: RMSNorm with eps 1e-6, a sigmoid
router in fp32, SwiGLU as a marked stand-in for SiTU-GLU, a 4096-bin
histogram over [0, 1] for the QB quantile.

Readings where the pages are silent:
  * QB quantile is the type-1 (inverse empirical CDF) quantile at rank
    m = ceil((E - k) * N / E), computed in exact integer arithmetic.
  * Bin rule min(floor(s * 4096), 4095) on the fp32 score (the layer keeps s in
    fp32, so the bin is decided in that precision); the estimate interpolates linearly
    inside the bin where the cumulative count first reaches m, so
    |estimate - exact| <= 1/4096.
  * The update uses the quantile of the biased column s + b, which is
    q_e + b_e because b_e is constant over the column (set literal=True for
    the un-biased reading).
  * Top-k order: larger s + b first, then lower expert index.
  * No capacity limit, no token dropping.

Parity unpinned: swiglu() is the stand-in for SiTU-GLU, whose formula the
pages do not give; it is pinned only as SwiGLU (a textbook form), not as
SiTU-GLU.
"""
from __future__ import annotations

import numpy as np

NBINS = 4096


def f64(a) -> np.ndarray:
    """Widen an input (numpy array or CPU torch tensor, fp32 or bf16) exactly to float64."""
    if hasattr(a, "detach"):  # torch tensor
        import torch
        return a.detach().to(torch.float64).numpy()
    return np.asarray(a, dtype=np.float64)


# --------------------------------------------------------------------------
# Forward steps.  [demo] Tab 1: tokens go to routed experts in the latent
# width l and to a shared expert in the backbone width d; RMSNorm (Tab 5)
# comes first ([course] survival table lists RMSNorm in the block).
# --------------------------------------------------------------------------

def rms_reciprocal(x: np.ndarray, eps: float) -> np.ndarray:
    """r_t = 1 / sqrt(mean_j x_tj^2 + eps), one value per token ([demo] Tab 5)."""
    return 1.0 / np.sqrt(np.mean(x * x, axis=1) + eps)


def rmsnorm(x: np.ndarray, gain: np.ndarray, eps: float) -> np.ndarray:
    """x_hat = gain * x * r_t ([demo] Tab 5; no compensation term, it is never formulated)."""
    return gain[None, :] * x * rms_reciprocal(x, eps)[:, None]


def latent_down(x_hat: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    """h = x_hat W_down^T, width d -> l ([demo] Tab 1 width separation; [blog] compress first)."""
    return x_hat @ w_down.T


def sigmoid(z: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-z))


def router_scores(h: np.ndarray, w_router: np.ndarray, c: np.ndarray) -> np.ndarray:
    """s = sigmoid(h W_router^T + c), one affinity per (token, expert)."""
    return sigmoid(h @ w_router.T + c[None, :])


def biased_topk(s: np.ndarray, b: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest u = s + b per token, larger u first, ties to the lower index.

    [demo] Tab 8-10: the bias b only reroutes tokens.  A stable sort of -u
    keeps equal keys in ascending expert order.
    """
    u = s + b[None, :]
    return np.argsort(-u, axis=1, kind="stable")[:, :k]


def topk_gap(s: np.ndarray, b: np.ndarray, k: int) -> np.ndarray:
    """Per token, u_(k) - u_(k+1): the margin between the last chosen and first unchosen biased score."""
    E = s.shape[1]
    if k >= E:
        return np.full(s.shape[0], np.inf)
    u = np.sort(s + b[None, :], axis=1)[:, ::-1]
    return u[:, k - 1] - u[:, k]


def topk_order_gap(s: np.ndarray, b: np.ndarray, k: int) -> np.ndarray:
    """Per token, the smallest margin between consecutive biased scores among the top k+1
    (the top k when k == E): how close the rank order of the chosen experts is to a tie."""
    E = s.shape[1]
    u = np.sort(s + b[None, :], axis=1)[:, ::-1][:, :min(k + 1, E)]
    if u.shape[1] < 2:
        return np.full(s.shape[0], np.inf)
    return np.min(u[:, :-1] - u[:, 1:], axis=1)


def gate_weights(s: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """g_i = s_{sel_i} / sum_j s_{sel_j}: unbiased scores of the chosen experts, renormalised.

    [demo] Tab 8-10: the bias does not change weight magnitudes, and the
    weights are normalised.
    """
    chosen = np.take_along_axis(s, idx, axis=1)
    return chosen / chosen.sum(axis=1, keepdims=True)


def silu(v: np.ndarray) -> np.ndarray:
    return v / (1.0 + np.exp(-v))


def swiglu(a: np.ndarray, w1: np.ndarray, w3: np.ndarray, w2: np.ndarray) -> np.ndarray:
    """(silu(a W1^T) * (a W3^T)) W2^T -- SwiGLU, the stand-in for SiTU-GLU ([demo] Tab 12)."""
    return (silu(a @ w1.T) * (a @ w3.T)) @ w2.T


def routed_outputs(h: np.ndarray, idx: np.ndarray, w1, w3, w2) -> np.ndarray:
    """o[t, i] = SwiGLU_{idx[t,i]}(h[t]) in latent width l, for every chosen (token, slot).

    Every pair is processed: there is no capacity limit ([ebook] capsule 25,
    the overflowing dispatch buffer was a bug).  w1/w3/w2 are indexable per
    expert (numpy or torch); each expert is widened to float64 when used.
    """
    T, k = idx.shape
    o = np.zeros((T, k, w2.shape[1]), dtype=np.float64)
    for e in np.unique(idx):
        t, i = np.nonzero(idx == e)
        o[t, i] = swiglu(h[t], f64(w1[e]), f64(w3[e]), f64(w2[e]))
    return o


def combine(g: np.ndarray, o: np.ndarray) -> np.ndarray:
    """z_t = sum_i g_ti o_ti, summed in rank order, still in latent width l."""
    z = g[:, 0, None] * o[:, 0]
    for i in range(1, g.shape[1]):
        z = z + g[:, i, None] * o[:, i]
    return z


def up_projection(z: np.ndarray, w_up: np.ndarray) -> np.ndarray:
    """z W_up^T, latent l -> backbone d ([demo] Tab 1)."""
    return z @ w_up.T


def shared_expert(x_hat: np.ndarray, ws1, ws3, ws2) -> np.ndarray:
    """One SwiGLU expert on x_hat at full width d, used by every token ([demo] Tab 1)."""
    return swiglu(x_hat, ws1, ws3, ws2)


def layer_forward(x, w: dict, b, k: int, eps: float = 1e-6) -> dict:
    """The whole layer for the given tokens; returns every intermediate in float64.

    x: [T, d]; w: the weight dict of datagen.layer_weights; b: [E] QB bias.
    y = W_up(sum_i g_i SwiGLU_{sel_i}(h)) + SharedSwiGLU(x_hat); no residual.
    """
    x = f64(x)
    b = f64(b)
    x_hat = rmsnorm(x, f64(w["rms_gain"]), eps)
    h = latent_down(x_hat, f64(w["w_down"]))
    s = router_scores(h, f64(w["w_router"]), f64(w["router_bias"]))
    idx = biased_topk(s, b, k)
    g = gate_weights(s, idx)
    o = routed_outputs(h, idx, w["w1"], w["w3"], w["w2"])
    z = combine(g, o)
    y = up_projection(z, f64(w["w_up"]))
    if "ws1" in w:
        y = y + shared_expert(x_hat, f64(w["ws1"]), f64(w["ws3"]), f64(w["ws2"]))
    return dict(r=rms_reciprocal(x, eps), h=h, s=s, idx=idx, gates=g, gap=topk_gap(s, b, k),
                order_gap=topk_order_gap(s, b, k), o=o, z=z, y=y)


def layer_routing(x, w: dict, b, k: int, eps: float = 1e-6) -> dict:
    """Only the routing half of layer_forward (RMSNorm, W_down, router, top-k, gates)."""
    x = f64(x)
    b = f64(b)
    x_hat = rmsnorm(x, f64(w["rms_gain"]), eps)
    h = latent_down(x_hat, f64(w["w_down"]))
    s = router_scores(h, f64(w["w_router"]), f64(w["router_bias"]))
    idx = biased_topk(s, b, k)
    return dict(h=h, s=s, idx=idx, gates=gate_weights(s, idx), gap=topk_gap(s, b, k),
                order_gap=topk_order_gap(s, b, k))


# --------------------------------------------------------------------------
# Dispatch bookkeeping: per-expert counts, offsets and a stable permutation
# ([ebook] capsule 20: experts run as grouped matmuls over their tokens).
# --------------------------------------------------------------------------

def expert_counts(idx: np.ndarray, E: int) -> np.ndarray:
    """cnt_e = number of (token, slot) pairs routed to expert e."""
    return np.bincount(idx.ravel(), minlength=E).astype(np.int64)


def expert_offsets(counts: np.ndarray) -> np.ndarray:
    """Exclusive prefix sum, E+1 entries: expert e owns permuted rows [off_e, off_{e+1})."""
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)


def stable_permutation(idx: np.ndarray, E: int):
    """Permuted order of the (token, slot) pairs: expert ascending, then token ascending.

    Returns (perm_token [T*k], perm_slot [T*k], inv [T, k]) with
    perm_token[inv[t, i]] == t and perm_slot[inv[t, i]] == i.
    """
    T, k = idx.shape
    perm_token, perm_slot = [], []
    for e in range(E):
        t, i = np.nonzero(idx == e)  # row-major: token ascending
        perm_token.append(t)
        perm_slot.append(i)
    perm_token = np.concatenate(perm_token).astype(np.int64)
    perm_slot = np.concatenate(perm_slot).astype(np.int64)
    inv = np.empty((T, k), dtype=np.int64)
    inv[perm_token, perm_slot] = np.arange(T * k)
    return perm_token, perm_slot, inv


# --------------------------------------------------------------------------
# Quantile Balancing ([demo] Tab 2 Figure 2(b), Tab 8-11; [blog] raise the
# bar for hot experts, lower it for cold ones).
# --------------------------------------------------------------------------

def score_bins(s: np.ndarray, nbins: int = NBINS) -> np.ndarray:
    """Bin of each score on [0, 1]: min(floor(s * nbins), nbins - 1).

    The layer keeps its router scores in fp32, so the bin (an integer decided by a float) is
    taken on the score rounded to fp32, the precision the layer fixes for s.
    """
    s32 = np.asarray(s, dtype=np.float32).astype(np.float64)
    return np.minimum(np.floor(s32 * nbins), nbins - 1).astype(np.int64)


def score_histogram(s: np.ndarray, nbins: int = NBINS) -> np.ndarray:
    """hist[e, j] = number of tokens whose score for expert e falls in bin j."""
    bins = score_bins(s, nbins)
    E = s.shape[1]
    hist = np.zeros((E, nbins), dtype=np.int64)
    for e in range(E):
        hist[e] = np.bincount(bins[:, e], minlength=nbins)
    return hist


def quantile_rank(N: int, k: int, E: int) -> int:
    """m = ceil((1 - k/E) N) in exact integer arithmetic, clamped to [1, N]."""
    m = ((E - k) * N + E - 1) // E
    return int(min(max(m, 1), N))


def exact_quantile(column: np.ndarray, m: int) -> float:
    """The m-th smallest value (type-1 quantile)."""
    return float(np.sort(column)[m - 1])


def histogram_quantile(hist_e: np.ndarray, m: int, nbins: int = NBINS) -> float:
    """Quantile estimate from one expert's histogram.

    j* = first bin whose cumulative count reaches m; the estimate places the
    m-th value linearly inside bin j*: (j* + (m - cum_{j*-1}) / cnt_{j*}) / nbins.
    """
    cum = np.cumsum(hist_e)
    j = int(np.argmax(cum >= m))
    below = int(cum[j] - hist_e[j])
    return (j + (m - below) / hist_e[j]) / nbins


def qb_update(b, hist: np.ndarray, N: int, k: int, beta: float, literal: bool = False,
              nbins: int = NBINS) -> np.ndarray:
    """One delayed, mean-centred bias step from the accumulated histogram.

    b_e <- b_e - beta (u_e - mean_e u) with u_e = q_e + b_e, the quantile of
    the biased column (literal=True: u_e = q_e).  Mean centring keeps mean(b)
    fixed ([demo] Tab 8-10); the statistics come from earlier forwards, so
    the update is delayed.
    """
    b = f64(b)
    E = hist.shape[0]
    m = quantile_rank(N, k, E)
    q = np.array([histogram_quantile(hist[e], m, nbins) for e in range(E)])
    u = q if literal else q + b
    return b - beta * (u - u.mean())


def sign_rule_update(b, load: np.ndarray, gamma: float) -> np.ndarray:
    """The aux-loss-free bias rule: b_e <- b_e + gamma * sign(mean load - load_e).

    [ebook] capsule 16 gives the rule with gamma = 1e-2 as the fix for expert
    collapse; load_e is the number of (token, slot) pairs routed to expert e
    since the previous update (expert_counts summed over those forwards), and
    with data-parallel ranks it is the sum over all ranks (capsule 27, Bug 2).
    The sign is taken exactly: mean load - load_e has the sign of
    sum(load) - E * load_e, an integer.
    """
    b = f64(b)
    load = np.asarray(load, dtype=np.int64)
    E = load.shape[0]
    direction = np.sign(load.sum() - E * load).astype(np.float64)
    return b + float(gamma) * direction


def load_ratio(counts: np.ndarray) -> float:
    """max/min expert load (inf if an expert got no token)."""
    lo = counts.min()
    return float("inf") if lo == 0 else float(counts.max() / lo)
