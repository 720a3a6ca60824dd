"""The seeded input generator: reproducible, subset-consistent, and shaped as the five workloads."""
import dataclasses

import numpy as np
import torch

import datagen


def test_row_subsets_regenerate_the_full_matrix():
    """Sampled parity checks draw only some rows; they must be the same rows the GPU sees."""
    shape = dataclasses.replace(datagen.WORKLOADS["mini_replica"], T=3000)
    full = datagen.tokens(shape)
    rows = np.array([0, 1, 1023, 1024, 2047, 2999, 5, 1500])
    assert torch.equal(datagen.tokens(shape, rows=rows), full[torch.from_numpy(rows)])
    assert torch.equal(datagen.tokens(shape), full)                      # same seed, same values
    assert not torch.equal(datagen.tokens(shape, seed=shape.seed + 1), full)
    assert full.dtype == torch.bfloat16 and full.shape == (3000, shape.d)


def test_workload_table():
    w = datagen.WORKLOADS
    sizes = {n: (s.T, s.d, s.l, s.E, s.k, s.h, s.hs, s.dtype, s.seed) for n, s in w.items()}
    assert sizes["tiny_fp32"] == (256, 256, 64, 32, 4, 128, 512, "f32", 0)
    assert sizes["mini_replica"] == (8192, 1024, 256, 256, 6, 256, 2048, "bf16", 1)
    assert sizes["wide_stress"] == (16384, 7168, 2048, 896, 16, 512, 4096, "bf16", 2)
    assert sizes["qb_skewed"][1:] == (1024, 256, 128, 8, 256, 2048, "bf16", 3) and w["qb_skewed"].T == 4096
    assert sizes["sweep"][1:] == (1024, 256, 256, 6, 256, 2048, "bf16", 4)
    assert w["mini_replica"].offset_var == 0.5 and w["sweep"].offset_var == 0.5
    assert w["tiny_fp32"].beta == 0.01 and w["qb_skewed"].beta == 0.05 and w["qb_skewed"].steps == 50


def test_weight_scales_follow_fan_in():
    shape = datagen.LayerShape("scales", 8, 512, 128, 16, 2, 256, 384, "f32", seed=9, offset_var=0.5)
    w = datagen.layer_weights(shape)
    fan_in = {"w_down": 512, "w_router": 128, "w1": 128, "w3": 128, "w2": 256, "w_up": 128,
              "ws1": 512, "ws3": 512, "ws2": 384}
    for name, fi in fan_in.items():
        var = float(w[name].double().var())
        assert abs(var * fi - 1.0) < 0.05, (name, var * fi)
    assert torch.equal(w["rms_gain"], torch.ones(512))
    c = w["router_bias"].double()
    assert abs(float(c.var()) - 0.5) < 0.35 and w["router_bias"].dtype == torch.float32  # 16 draws of N(0, 0.5)
