"""The decode kernel for 5-8 query heads per KV head (query heads on the MMA M
side, codes unpacked as exact fp16 subnormals) against the oracle, over every
shape it takes: G = 5, 6, 8 (the workloads have G = 7), head dim 64 and 128,
side-code rank 0, 8 and 16, dense and 2-bit values; then ragged lengths with
the fused append.  2-bit values without a side code are not the kernel's
(the generic kernel takes them) and are checked here as well.

Decode: max relative error per output row <= 2e-3 of the row maximum, lse to
1e-5 relative; the appended token's planes bit-exact.
"""

import numpy as np
import pytest

import oracle
from bit_decode_attention_sm_b200 import configs, synth
from parity_helpers import (DECODE_RTOL, assert_planes_equal, gpu_cache, gpu_query, oracle_side,
                            planes_to_numpy, row_rel_err, torch_dtype)

pytestmark = pytest.mark.gpu

SHAPES = [(G, d, r, vmode) for G in (5, 6, 8) for d in (64, 128) for r in (0, 8, 16)
          for vmode in ("dense", "2bit")]


def _workload(G, d, r, vmode, B, T):
    base = configs.workload(2)
    return base.with_(d=d, r=r, r_s=max(2, min(8, d // 2)), Hq=2 * G, Hkv=2, B=B, T=T,
                      n_cal=64, kv_dtype="bf16", vmode=vmode)


def _basis(w, L):
    if w.r > 0:
        U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
        return U
    return np.zeros((w.Hkv, w.d, 0), np.float32)


@pytest.mark.parametrize("G,d,r,vmode", SHAPES,
                         ids=["G%d-d%d-r%d-%s" % s for s in SHAPES])
def test_gqa_decode_matches_oracle(G, d, r, vmode):
    """T = 333: five full 64-token tiles and a ragged one; 2 sequences x 2 KV heads."""
    from bit_decode_attention_sm_b200 import headq as hq
    w = _workload(G, d, r, vmode, B=2, T=333)
    L = synth.make_layer(w)
    U = _basis(w, L)
    _, out_ref, lse_ref = oracle_side(w, L, U)
    cache, Ut = gpu_cache(w, L, U)
    out, lse = hq.headq_decode_attn(cache, gpu_query(w, L), Ut, T=w.T)
    assert row_rel_err(out.cpu().numpy(), out_ref) <= DECODE_RTOL
    np.testing.assert_allclose(lse.cpu().numpy(), lse_ref, rtol=1e-5, atol=1e-4)


APPEND = [(5, 128, 16, "dense"), (8, 128, 16, "2bit"), (6, 64, 8, "2bit"), (8, 64, 0, "dense")]


@pytest.mark.parametrize("G,d,r,vmode", APPEND, ids=["G%d-d%d-r%d-%s" % s for s in APPEND])
def test_gqa_decode_append_ragged(G, d, r, vmode):
    """headq_decode_append with per-sequence lengths 0, 1, 65 and T: the new token
    of each sequence written at T_b - 1 (planes bit-exact) and the attention over
    tokens < T_b."""
    import torch
    from bit_decode_attention_sm_b200 import headq as hq
    T = 300
    w = _workload(G, d, r, vmode, B=4, T=T)
    L = synth.make_layer(w)
    B, Hkv = w.B, w.Hkv
    sl = np.array([0, 1, 65, T], np.int32)
    U = _basis(w, L)
    planes, out_ref, lse_ref = oracle_side(w, L, U, seq_lens=sl)
    # the cache holds other data where the new tokens go
    stale = synth.LayerInputs(L.keys.copy(), L.values.copy(), L.queries, L.q_cal, {})
    rng = np.random.default_rng(3)
    for b in range(B):
        if sl[b] > 0:
            stale.keys[b, :, sl[b] - 1] = rng.standard_normal((Hkv, d)).astype(np.float32)
            stale.values[b, :, sl[b] - 1] = rng.standard_normal((Hkv, d)).astype(np.float32)
    stale.keys = synth.round_bf16(stale.keys)
    stale.values = synth.round_bf16(stale.values)
    cache, Ut = gpu_cache(w, stale, U)
    dt = torch_dtype(w)
    pos = np.maximum(sl - 1, 0)
    k_new = torch.from_numpy(np.ascontiguousarray(L.keys[np.arange(B), :, pos])).cuda().to(dt)
    v_new = torch.from_numpy(np.ascontiguousarray(L.values[np.arange(B), :, pos])).cuda().to(dt)
    ws = hq.decode_workspace(cache, w.Hq, T)
    out, lse = hq.headq_decode_append(cache, k_new, v_new, gpu_query(w, L), Ut, T=T,
                                      seq_lens=torch.from_numpy(sl).cuda(), ws=ws)
    hq.headq_workspace_status(ws)
    o, l_ = out.cpu().numpy(), lse.cpu().numpy()
    assert (o[0] == 0).all() and np.isneginf(l_[0]).all()
    assert row_rel_err(o[1:], out_ref[1:]) <= DECODE_RTOL
    np.testing.assert_allclose(l_[1:], lse_ref[1:], rtol=1e-5, atol=1e-4)
    got = planes_to_numpy(cache, 0, T)
    for b in range(1, B):
        p_ = sl[b] - 1
        one = {k: a[b:b + 1, :, p_:p_ + 1] for k, a in got.items()}
        ref1 = {k: a[b:b + 1, :, p_:p_ + 1] for k, a in planes.items() if k != "y"}
        assert_planes_equal(one, ref1, w.r, w.vmode, w.kv_dtype,
                            values=L.values[b:b + 1, :, p_:p_ + 1])
