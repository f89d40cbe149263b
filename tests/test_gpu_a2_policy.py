"""A^2 value policy (full-KV composition) on the GPU against the oracle.

Scores: fp32 kernels vs the fp64 oracle, elementwise within 1e-3 relative (of
the per-(b, kv) maximum).  Selection is integer work: fed the same fp32 scores,
the kernel's kept set equals the oracle's exactly (ties included) and the
copied values are bit-identical; on its own scores, the GPU's kept set is
checked to be a valid top-K of the oracle's scores up to near-ties.  The
value fixup after a decode is compared with the oracle's decode over the
mixed values, with the kept set the oracle chose.
"""

import numpy as np
import pytest

import oracle
from bit_decode_attention_sm_b200 import configs, synth
from parity_helpers import (DECODE_RTOL, gpu_cache, gpu_query, layer, row_rel_err,
                            torch_dtype)

pytestmark = pytest.mark.gpu

SCORE_RTOL = 1e-3


def _headq():
    from bit_decode_attention_sm_b200 import headq
    return headq


def _setup(i, n_obs=4, **kw):
    w, L = layer(i, **kw)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    planes = oracle.cache_write(L.keys, U, v=L.values, vmode=w.vmode)
    vh = oracle.cached_values(planes, w.vmode, L.values)
    qo = synth.make_observation_queries(w, L, n_obs)
    return w, L, U, planes, vh, qo


def _to(w, a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda().to(torch_dtype(w))


CASES = [(4, dict(T=700, B=3), [700, 300, 64]), (4, dict(T=333, B=2), None),
         (2, dict(T=500, B=2), [500, 1]), (0, {}, [300])]


@pytest.mark.parametrize("i,kw,sl", CASES,
                         ids=["cfg4-ragged", "cfg4", "cfg2-dense", "cfg0-fp32-2bit"])
def test_a2_scores_match_oracle(i, kw, sl):
    """bf16 workloads take the tensor-core passes, fp32 the CUDA-core ones."""
    import torch
    hq = _headq()
    w, L, U, planes, vh, qo = _setup(i, **kw)
    if w.kv_dtype == "f32":  # give the fp32 workload 2-bit values, so a_j is not 0
        w = w.with_(vmode="2bit")
        planes = oracle.cache_write(L.keys, U, v=L.values, vmode="2bit")
        vh = oracle.cached_values(planes, "2bit")
    sl = None if sl is None else np.array(sl, np.int32)
    ref = oracle.a2_scores(qo, L.keys, L.values, vh, seq_lens=sl)
    cache, Ut = gpu_cache(w, L, U)
    slt = None if sl is None else torch.from_numpy(sl).cuda()
    ws = hq.a2_workspace(cache, qo.shape[1], w.Hq, L.keys.shape[2])
    got = hq.headq_a2_scores(cache, _to(w, qo), _to(w, L.keys), _to(w, L.values),
                             seq_lens=slt, ws=ws).cpu().numpy()
    hq.headq_workspace_status(ws)
    scale = np.maximum(ref.max(axis=2, keepdims=True), 1e-30)
    assert np.abs(got - ref).max() <= SCORE_RTOL * scale.max()
    assert (np.abs(got - ref) <= SCORE_RTOL * scale + 1e-30).all()
    if sl is not None:
        for b in range(len(sl)):
            assert (got[b, :, sl[b]:] == 0).all()


@pytest.mark.parametrize("K", [0, 1, 37, 64, 400, 1000])
def test_a2_select_bit_exact_on_shared_scores(K):
    """Same fp32 scores in: same kept positions (ties to the lower position),
    -1 padding, and the exact value rows copied."""
    import torch
    hq = _headq()
    w, L = layer(4, T=700, B=3)
    rng = np.random.default_rng(K)
    sc = rng.gamma(0.5, size=(3, w.Hkv, 700)).astype(np.float32)
    sc[0, 0] = np.round(sc[0, 0] * 4) / 4            # heavy ties
    sc[1, 1, :] = 0.0                                 # all equal
    sl = np.array([700, 250, 0], np.int32)
    ref = oracle.a2_select(sc.astype(np.float64), K, seq_lens=sl)
    vt = _to(w, L.values)
    idx, kv_ = hq.headq_a2_select(torch.from_numpy(sc).cuda(), K, vt,
                                  seq_lens=torch.from_numpy(sl).cuda())
    got = idx.cpu().numpy()
    np.testing.assert_array_equal(got, ref)
    kvh = kv_.float().cpu().numpy()
    for b in range(3):
        for h in range(w.Hkv):
            for k, j in enumerate(ref[b, h]):
                want = L.values[b, h, j] if j >= 0 else np.zeros(w.d, np.float32)
                np.testing.assert_array_equal(kvh[b, h, k], want)


def test_a2_gpu_pipeline_keeps_a_valid_top_k():
    """Scores and selection both on the GPU: every kept token's oracle score is
    at least every dropped token's, up to the score tolerance."""
    import torch
    hq = _headq()
    w, L, U, planes, vh, qo = _setup(4, T=700, B=2, n_obs=8)
    sl = np.array([700, 333], np.int32)
    ref = oracle.a2_scores(qo, L.keys, L.values, vh, seq_lens=sl)
    cache, Ut = gpu_cache(w, L, U)
    slt = torch.from_numpy(sl).cuda()
    sc = hq.headq_a2_scores(cache, _to(w, qo), _to(w, L.keys), _to(w, L.values), seq_lens=slt)
    K = 70
    idx, _ = hq.headq_a2_select(sc, K, _to(w, L.values), seq_lens=slt)
    got = idx.cpu().numpy()
    for b in range(2):
        for h in range(w.Hkv):
            kept = got[b, h][got[b, h] >= 0]
            assert len(kept) == min(K, sl[b]) and (np.diff(kept) > 0).all()
            dropped = np.setdiff1d(np.arange(sl[b]), kept)
            tol = SCORE_RTOL * ref[b, h].max()
            assert ref[b, h, kept].min() >= ref[b, h, dropped].max() - 2 * tol


@pytest.mark.parametrize("i,kw,sl,K", [
    (4, dict(T=700, B=3), [700, 300, 1], 90),
    (4, dict(T=257, B=2), None, 257),
    (0, {}, None, 40),
], ids=["cfg4-ragged", "cfg4-all-kept", "cfg0-fp32"])
def test_a2_value_fixup_matches_mixed_value_decode(i, kw, sl, K):
    import torch
    hq = _headq()
    w, L, U, planes, vh, qo = _setup(i, **kw)
    if w.vmode != "2bit":  # the fp32 workload with 2-bit values
        w = w.with_(vmode="2bit")
        planes = oracle.cache_write(L.keys, U, v=L.values, vmode="2bit")
        vh = oracle.cached_values(planes, "2bit")
    sl = None if sl is None else np.array(sl, np.int32)
    ref_sc = oracle.a2_scores(qo, L.keys, L.values, vh, seq_lens=sl)
    keep = oracle.a2_select(ref_sc, K, seq_lens=sl)
    mixed = oracle.a2_mixed_values(vh, L.values, keep)
    out_ref, lse_ref = oracle.decode(L.queries, planes, U, v=mixed, seq_lens=sl)
    base_ref, _ = oracle.decode(L.queries, planes, U, vmode="2bit", seq_lens=sl)
    cache, Ut = gpu_cache(w, L, U)
    B, Hkv, T, d = L.keys.shape
    keep_v = np.zeros((B, Hkv, K, d), np.float32)
    for b in range(B):
        for h in range(Hkv):
            for k, j in enumerate(keep[b, h]):
                if j >= 0:
                    keep_v[b, h, k] = L.values[b, h, j]
    slt = None if sl is None else torch.from_numpy(sl).cuda()
    q = gpu_query(w, L)
    out, lse = hq.headq_decode_attn(cache, q, Ut, T=T, seq_lens=slt)
    assert row_rel_err(out.cpu().numpy(), base_ref) <= DECODE_RTOL
    hq.headq_a2_value_fixup(cache, q, Ut, torch.from_numpy(keep).cuda(), _to(w, keep_v), out,
                            lse, T=T, seq_lens=slt)
    o = out.cpu().numpy()
    fin = np.isfinite(lse_ref)
    assert row_rel_err(o[fin], out_ref[fin]) <= DECODE_RTOL
    assert (o[~fin] == 0).all()
    # the policy moved the output towards the exact-value attention
    exact, _ = oracle.decode(L.queries, planes, U, v=L.values, seq_lens=sl)
    e_mixed = np.abs(o[fin] - exact[fin]).max()
    e_base = np.abs(base_ref[fin] - exact[fin]).max()
    assert e_mixed < e_base


def test_a2_scores_on_a_paged_cache():
    import torch
    from test_gpu_paged import paged_cache
    hq = _headq()
    w, L, U, planes, vh, qo = _setup(4, T=300, B=2)
    ref = oracle.a2_scores(qo, L.keys, L.values, vh)
    cache, _ = paged_cache(w, L, U, 64)
    got = hq.headq_a2_scores(cache, _to(w, qo), _to(w, L.keys), _to(w, L.values)).cpu().numpy()
    assert np.abs(got - ref).max() <= SCORE_RTOL * ref.max()
