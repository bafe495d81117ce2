"""h2o_attend_noalloc against the handle API, through the C ABI (needs a GPU).

The allocation-free entry point serves callers that cannot call cudaMalloc
(an engine whose own pool holds nearly all device memory, or code that cannot
afford cudaMalloc's device synchronisation); its scratch is a fixed array in
the library's static device memory, shared by every call.  Two calls in a row
-- a prefill chunk against an empty cache, then a step chunk against the
filled cache -- must give the outputs and summed weights that h2o_prefill and
h2o_step give, within the parity tolerances.  The second call also shows that
the shared scratch left by the first does not leak into its results.
"""
import numpy as np
import pytest
import torch

from tests.parity_util import SCORE_RTOL, check_outputs, to64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.bfloat16, 128)])
def test_noalloc_matches_handle_api_on_two_calls(cuda_ok, dtype, d):
    import dataclasses

    import h2o_kv_cache_b200 as h2o
    from h2o_kv_cache_b200.workload import CONFIGS, gen_batch, split_chunks

    cfg = dataclasses.replace(CONFIGS[0], B=2, d=d, dtype=dtype, M=300, R=20, P=200, S=150,
                              T=350, planted=0.01, name="noalloc")
    Q, K, V = gen_batch(cfg, 0, device="cuda")
    (q0, k0, v0), (q1, k1, v1) = split_chunks(Q, K, V, cfg.bounds())
    cache = h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype)
    out0 = cache.prefill(q0, k0, v0)
    _, sc0, pos0 = cache.read_state()
    kc, vc = cache.read_kv()
    n_valid0 = cache.info()["n_valid"]
    out1 = cache.step(q1, k1, v1)
    slots1, sc1, pos1 = cache.read_state()
    torch.cuda.synchronize()

    # call 1: the prefill chunk against an empty cache
    oa, ca = h2o.attend_noalloc(q0, k0, v0, None, None, n_valid=0, M=cfg.M)
    # call 2: the step chunk against the cache the prefill left
    ob, cb = h2o.attend_noalloc(q1, k1, v1, kc, vc, n_valid=n_valid0, M=cfg.M)
    torch.cuda.synchronize()

    check_outputs(to64(oa), to64(out0), dtype, "noalloc call 1")
    check_outputs(to64(ob), to64(out1), dtype, "noalloc call 2")
    P, S, M = cfg.P, cfg.S, cfg.M
    ca, cb = to64(ca), to64(cb)
    sc0, sc1, slots1 = to64(sc0), to64(sc1), slots1.cpu().numpy()
    # call 1: the prefill's scores are the chunk keys' summed weights, no cache mass
    assert np.all(ca[:, :, :M] == 0)
    np.testing.assert_allclose(ca[:, :, M:M + P], sc0[:, :, :P], rtol=SCORE_RTOL, atol=0)
    # call 2: kept slots gained the cache columns, filled slots hold the chunk keys'
    for b in range(cfg.B):
        for h in range(cfg.Hkv):
            filled = set(slots1[b, h].tolist())
            kept = np.array([s for s in range(n_valid0) if s not in filled])
            np.testing.assert_allclose(sc1[b, h, kept], sc0[b, h, kept] + cb[b, h, kept],
                                       rtol=SCORE_RTOL, atol=0)
            np.testing.assert_allclose(sc1[b, h, slots1[b, h]], cb[b, h, M:M + S],
                                       rtol=SCORE_RTOL, atol=0)
    cache.close()


def test_noalloc_rejects_sizes_above_its_scratch(cuda_ok):
    import h2o_kv_cache_b200 as h2o
    # 4 * 8 * (65536 + 1024) accumulator words: above the 2 Mi-word array
    q = torch.zeros(4, 32, 1024, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(4, 8, 1024, 128, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(4, 8, 65536, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(h2o.H2OError) as ei:
        h2o.attend_noalloc(q, k, k, kc, kc, n_valid=65536, M=65536)
    assert ei.value.status == -2 and "fixed maximum" in str(ei.value)
