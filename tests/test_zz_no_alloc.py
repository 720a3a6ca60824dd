"""lmoe_route_noalloc: the routing stage for callers that cannot allocate device memory.

Such callers (code running under CUDA-graph stream capture, hosts that own all device memory,
loops that must not enter the allocator) get routing whose scratch is a static device array in
the library.  This file checks, through the C ABI, that two calls in a row match the handle-based
routing (lmoe_route_scores + lmoe_get_routing) exactly, and that a size beyond the array is
refused.  It runs last so that a stop at the first failure has already run every other test; it
builds the library itself, so it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import datagen
import latent_routing_quantile_b200 as lq

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from latent_routing_quantile_b200 import build
    build.build()
    yield


def handle_routing(scores, bias, k):
    """The existing entry point: a layer handle routes the same scores."""
    T, E = scores.shape
    shape = datagen.LayerShape("noalloc_ref", T, 64, 64, E, k, 64, 0, "bf16", seed=1)
    layer = lq.layer_from_weights(shape, datagen.layer_weights(shape))
    layer.set_bias(bias)
    layer.route_scores(scores)
    r = layer.routing()
    torch.cuda.synchronize()
    layer.close()
    return r


@pytest.mark.parametrize("T,E,k,quant", [(1000, 256, 6, 0), (333, 64, 8, 16)])
def test_noalloc_routing_matches_handle_routing_twice(T, E, k, quant):
    outs = {}
    for call in range(2):
        s = torch.from_numpy(datagen.uniform_scores(T, E, seed=100 * call + T, quantise=quant)).cuda()
        b = torch.from_numpy(datagen.normal_bias(E, seed=call + 7, std=0.02)).cuda()
        got = lq.route_noalloc(s, b, k)
        torch.cuda.synchronize()
        ref = handle_routing(s, b, k)
        for name in ("idx", "counts", "offsets", "perm", "inv"):
            assert torch.equal(got[name], ref[name]), (call, name)
        np.testing.assert_allclose(got["gates"].cpu().numpy(), ref["gates"].cpu().numpy(), rtol=0, atol=0)
        outs[call] = got
    # the second call saw different scores, so the shared scratch did not leak the first result
    assert not torch.equal(outs[0]["idx"], outs[1]["idx"])


def test_noalloc_rejects_sizes_beyond_its_scratch():
    T, E, k = 200000, 256, 6
    s = torch.zeros((T, E), dtype=torch.float32, device="cuda")
    b = torch.zeros(E, dtype=torch.float32, device="cuda")
    with pytest.raises(lq.LmoeError, match="unsupported"):
        lq.route_noalloc(s, b, k)
