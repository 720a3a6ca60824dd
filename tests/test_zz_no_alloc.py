"""lmoe_route_noalloc: the routing stage for callers that cannot allocate device memory.

Such callers (plug-ins whose host application owns every byte of device memory, code running
inside another memory manager, real-time loops that must not enter the driver's allocator) get
routing whose scratch is a static device array in the library.  This file checks, through the C
ABI, that two calls in a row give the oracle's routing on the fp32 scores they are given and the
same routing as the handle-based entry point (lmoe_route_scores + lmoe_get_routing), that the
caller's status word reports a NaN score, and that sizes beyond the array are refused.  It runs
last so that a stop at the first failure has already run every other test; it builds the library
itself, so it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import datagen
import oracle
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
def test_noalloc_routing_matches_oracle_and_handle_routing_twice(T, E, k, quant):
    outs = {}
    for call in range(2):
        s_np = datagen.uniform_scores(T, E, seed=100 * call + T, quantise=quant)
        b_np = datagen.normal_bias(E, seed=call + 7, std=0.02)
        s, b = torch.from_numpy(s_np).cuda(), torch.from_numpy(b_np).cuda()
        got = lq.route_noalloc(s, b, k)
        torch.cuda.synchronize()
        assert int(got["status"].item()) == 0
        # the oracle, deciding on the same fp32 biased scores the kernels rank
        u32 = (s_np + b_np[None, :]).astype(np.float32).astype(np.float64)
        idx = oracle.biased_topk(u32, np.zeros(E), k)
        cnt = oracle.expert_counts(idx, E)
        pt, ps, inv = oracle.stable_permutation(idx, E)
        assert np.array_equal(got["idx"].cpu().numpy(), idx), call
        np.testing.assert_allclose(got["gates"].cpu().numpy(), oracle.gate_weights(s_np.astype(np.float64), idx),
                                   rtol=2e-6)
        assert np.array_equal(got["counts"].cpu().numpy(), cnt)
        assert np.array_equal(got["offsets"].cpu().numpy(), oracle.expert_offsets(cnt))
        assert np.array_equal(got["perm"].cpu().numpy(), pt)
        assert np.array_equal(got["inv"].cpu().numpy(), inv.ravel())
        # and exactly what the handle-based entry point returns
        ref = handle_routing(s, b, k)
        for name in ("idx", "gates", "counts", "offsets", "perm", "inv"):
            assert torch.equal(got[name], ref[name]), (call, name)
        outs[call] = got
    # the second call saw different scores, so the shared scratch did not leak the first result
    assert not torch.equal(outs[0]["idx"], outs[1]["idx"])


def test_noalloc_reports_a_nan_score_in_the_callers_status_word():
    T, E, k = 64, 64, 4
    s_np = datagen.uniform_scores(T, E, seed=3)
    s_np[5, 7] = np.nan
    got = lq.route_noalloc(torch.from_numpy(s_np).cuda(), torch.zeros(E, device="cuda"), k)
    torch.cuda.synchronize()
    assert int(got["status"].item()) & lq.STATUS_NAN_SCORE
    assert 7 not in got["idx"][5].cpu().tolist()
    # the next call clears the word and reports only its own faults
    got = lq.route_noalloc(torch.from_numpy(datagen.uniform_scores(T, E, seed=4)).cuda(),
                           torch.zeros(E, device="cuda"), k, out={"status": got["status"]})
    torch.cuda.synchronize()
    assert int(got["status"].item()) == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    T, E, k = 94497, 256, 6  # one token past the largest size the 8 MiB array holds
    s = torch.zeros((T, E), dtype=torch.float32, device="cuda")
    b = torch.zeros(E, dtype=torch.float32, device="cuda")
    with pytest.raises(lq.LmoeError, match="unsupported"):
        lq.route_noalloc(s, b, k)
    got = lq.route_noalloc(s[:T - 1], b, k)  # the largest size runs
    torch.cuda.synchronize()
    assert int(got["status"].item()) == 0 and int(got["offsets"][-1].item()) == (T - 1) * k
    with pytest.raises(lq.LmoeError, match="unsupported"):
        lq.route_noalloc(torch.zeros((8, 1088), device="cuda"), torch.zeros(1088, device="cuda"), 4)
