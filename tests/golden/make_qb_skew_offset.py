"""Writes qb_skew_offset.json: the router column offset of the skewed-router QB workload.

The workload (T=4096, d=1024, l=256, E=128, k=8, hidden 256, bf16, seed 3)
asks for a router whose expert 0 takes about 3.7x the mean load with a
max/min load ratio of at least 3.5, which is the starting point of the QB
demo's Figure 2(a) ("KimiK3MoE架构轻量化复刻演示上线...", Tab 2: expert 0 near
3500 tokens, max/min 3.7 before QB).  The reading used: only expert 0 gets a
column offset c_0 = a, every other c_e = 0, and a is found by bisection on
the step-0 tokens (seed 3 + 0) so that load_0 / mean load = 3.7.

Uses only the oracle and the seeded input generator.  Run from the repo root:
    python tests/golden/make_qb_skew_offset.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import datagen  # noqa: E402
import oracle  # noqa: E402

TARGET = 3.7


def main():
    shape = datagen.WORKLOADS["qb_skewed"]
    E, k, T = shape.E, shape.k, shape.T
    w = datagen.layer_weights(shape)
    x = datagen.tokens(shape, seed=shape.seed + 0)
    b = np.zeros(E)
    # h does not depend on c, so compute it once; the offset moves only column 0.
    x_hat = oracle.rmsnorm(oracle.f64(x), oracle.f64(w["rms_gain"]), shape.rms_eps)
    h = oracle.latent_down(x_hat, oracle.f64(w["w_down"]))
    wr = oracle.f64(w["w_router"])
    mean_load = T * k / E

    def ratio0(a):
        c = np.zeros(E)
        c[0] = a
        s = oracle.router_scores(h, wr, c)
        cnt = oracle.expert_counts(oracle.biased_topk(s, b, k), E)
        return cnt[0] / mean_load, cnt

    lo, hi = 0.0, 8.0
    for _ in range(60):
        mid = 0.5 * (lo + hi)
        if ratio0(mid)[0] < TARGET:
            lo = mid
        else:
            hi = mid
    a = float(np.float32(hi))  # stored as the fp32 value both sides receive
    r0, cnt = ratio0(a)
    out = {
        "a": a,
        "expert0_load_over_mean": float(r0),
        "initial_max_min": oracle.load_ratio(cnt),
        "note": "c_0 = a, c_e = 0 otherwise; step-0 tokens; written by make_qb_skew_offset.py",
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "qb_skew_offset.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out))


if __name__ == "__main__":
    main()
