"""The same-budget counterexample of the HeadQ summary (section 4) on the CUDA path.

Two side codes of exactly the same size (rank r, 4-bit levels, one fp32 scale
per token) differ only in their basis: HeadQ's query-PCA basis, and the basis
fitted to the key residuals, which is best for key storage.  Both caches are
written by the CUDA cache-write kernel (every plane bit-exact with the oracle,
so both have the oracle's key-storage error) and read by the CUDA diagnostic
kernel: the residual basis has the lower storage error and a far higher
attention KL, with each KL within the diagnostic tolerance of the oracle's.
"""

import numpy as np
import pytest

import oracle
from parity_helpers import (assert_diag_close, assert_planes_equal, gpu_cache, gpu_query, layer,
                            planes_to_numpy)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("i", [2, 3, 4])
def test_same_budget_counterexample_through_the_gpu_path(i):
    import torch
    from bit_decode_attention_sm_b200 import headq as hq
    w, L = layer(i, T=512, B=min(2, configs_B(i)))
    T = L.keys.shape[2]
    Uq, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    Ue = oracle.residual_basis(L.keys, w.r)
    dt = torch.bfloat16 if w.kv_dtype == "bf16" else torch.float32
    k_all = torch.from_numpy(L.keys).cuda().to(dt)
    v_all = torch.from_numpy(L.values).cuda().to(dt)
    res = {}
    for tag, U in (("query", Uq), ("residual", Ue)):
        ref = oracle.cache_write(L.keys, U, v=L.values, vmode=w.vmode)
        kl_ref, fv_ref, _, _ = oracle.attn_kl(L.queries, ref, U, L.keys, L.values, v=L.values,
                                              vmode=w.vmode)
        cache, Ut = gpu_cache(w, L, U)
        assert_planes_equal(planes_to_numpy(cache, 0, T), ref, w.r, w.vmode, w.kv_dtype,
                            values=L.values)
        kl, fv, _, _ = hq.headq_attn_kl(cache, gpu_query(w, L), Ut, k_all, v_all)
        kl, fv = kl.cpu().numpy(), fv.cpu().numpy()
        assert_diag_close(kl, kl_ref, "kl " + tag)
        assert_diag_close(fv, fv_ref, "fisher variance " + tag)
        res[tag] = (oracle.key_mse(L.keys, ref, U), float(kl.mean()),
                    sum(t.numel() * t.element_size() for t in cache.planes().values()))
    assert res["residual"][2] == res["query"][2]         # the same cache size
    assert res["residual"][0] < 0.8 * res["query"][0]    # lower key-storage error
    assert res["residual"][1] > 5.0 * res["query"][1]    # far higher attention KL


def configs_B(i):
    from bit_decode_attention_sm_b200 import configs
    return configs.workload(i).B
