"""Decode parity away from unit scale (gist.science summary of HeadQ, section 3,
step 3: the corrected logit and the attention readout hold for any query, key
and value magnitude).

The tensor-core decode feeds fp16 operands to the MMAs: the query split into
fp16 high and low parts (and sigma U_h^T q likewise), and with 2-bit values the
product p * scale of each token and value group.  These tests scale queries,
keys and values far from the generator's unit scale, and spread the value
scale over six decades token by token, and check every output row against the
oracle with the same tolerance as the unit-scale tests.  The per-channel key
code (a scale per channel and 64-token block, folded into the fp16 query parts
tile by tile) is checked the same way, with the key channels also spread over
four decades.  Inputs stay
representable in the workload's dtype (bf16 rounding after scaling), so both
sides see the same numbers.
"""

import numpy as np
import pytest

import oracle
from bit_decode_attention_sm_b200 import synth
from parity_helpers import (DECODE_RTOL, gpu_cache, gpu_query, layer, oracle_side,
                            row_rel_err)

pytestmark = pytest.mark.gpu


def _scaled(w, L, q=1.0, k=1.0, v=1.0, v_token_decades=0.0, k_channel_decades=0.0, seed=0):
    """A copy of the layer with queries, keys and values scaled (values also by
    10^u per token and KV head, u uniform in +-v_token_decades/2; keys by 10^u
    per KV head and channel, u uniform in +-k_channel_decades/2)."""
    rnd = synth.round_bf16 if w.kv_dtype == "bf16" else (lambda a: a.astype(np.float32))
    rng = np.random.default_rng(seed)
    vals = L.values * np.float32(v)
    if v_token_decades:
        u = rng.uniform(-0.5, 0.5, size=vals.shape[:3] + (1,)) * v_token_decades
        vals = vals * (10.0 ** u).astype(np.float32)
    keys = L.keys * np.float32(k)
    if k_channel_decades:
        B, Hkv, T, d = keys.shape
        u = rng.uniform(-0.5, 0.5, size=(1, Hkv, 1, d)) * k_channel_decades
        keys = keys * (10.0 ** u).astype(np.float32)
    return synth.LayerInputs(rnd(keys), rnd(vals), rnd(L.queries * np.float32(q)), L.q_cal, L.meta)


CASES = [  # (id, workload, reduced sizes, scaling)
    ("fullkv2bit-v1e-4", 4, dict(T=700, B=2), dict(v=1e-4)),
    ("fullkv2bit-v1e3", 4, dict(T=700, B=2), dict(v=1e3)),
    ("fullkv2bit-v-spread-6-decades", 4, dict(T=700, B=2), dict(v_token_decades=6.0)),
    ("fullkv2bit-q300", 4, dict(T=700, B=2), dict(q=300.0)),
    ("fullkv2bit-q1e-3", 4, dict(T=700, B=2), dict(q=1e-3)),
    ("gqa7-q1e-3", 2, dict(T=1000, B=2), dict(q=1e-3)),
    ("gqa7-q300", 2, dict(T=1000, B=2), dict(q=300.0)),
    ("longctx-q1e-3", 3, dict(T=2500), dict(q=1e-3)),
    ("longctx-q300", 3, dict(T=2500), dict(q=300.0)),
    ("longctx-k1e3", 3, dict(T=2500), dict(k=1e3)),
    ("longctx-q1e4-k1e-2", 3, dict(T=2500), dict(q=1e4, k=1e-2)),
    ("mha-d64-q1e-3-v1e3", 1, dict(T=300), dict(q=1e-3, v=1e3)),
]


@pytest.mark.parametrize("name,i,kw,sc", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("sigma", [1, -1])
def test_decode_far_from_unit_scale(name, i, kw, sc, sigma):
    _check(i, kw, sc, sigma, "token")


CHANNEL_CASES = [
    ("longctx-q1e-3", 3, dict(T=2500), dict(q=1e-3)),
    ("longctx-q1e4-k1e-2", 3, dict(T=2500), dict(q=1e4, k=1e-2)),
    ("longctx-k-channels-4-decades", 3, dict(T=2500), dict(k_channel_decades=4.0)),
    ("gqa7-q300-k-channels-4-decades", 2, dict(T=1000, B=2), dict(q=300.0, k_channel_decades=4.0)),
    ("fullkv2bit-v-spread-6-decades", 4, dict(T=700, B=2), dict(v_token_decades=6.0)),
    ("mha-d64-q1e-3-v1e3", 1, dict(T=300), dict(q=1e-3, v=1e3)),
]


@pytest.mark.parametrize("name,i,kw,sc", CHANNEL_CASES, ids=[c[0] for c in CHANNEL_CASES])
@pytest.mark.parametrize("sigma", [1, -1])
def test_channel_keys_far_from_unit_scale(name, i, kw, sc, sigma):
    _check(i, kw, sc, sigma, "channel")


def _check(i, kw, sc, sigma, kmode):
    from bit_decode_attention_sm_b200 import headq as hq
    w, L0 = layer(i, **kw)
    U, _ = oracle.calibrate(L0.q_cal, w.Hkv, w.r)
    L = _scaled(w, L0, **sc)
    _, out_ref, lse_ref = oracle_side(w, L, U, sigma=float(sigma), kmode=kmode)
    assert np.isfinite(out_ref).all()
    cache, Ut = gpu_cache(w, L, U, kmode=kmode)
    T = L.keys.shape[2]
    ws = hq.decode_workspace(cache, w.Hq, T)
    out, lse = hq.headq_decode_attn(cache, gpu_query(w, L), Ut, T=T, corr_sign=sigma, ws=ws)
    hq.headq_workspace_status(ws)
    out = out.cpu().numpy()
    assert np.isfinite(out).all()
    err = row_rel_err(out, out_ref)
    assert err <= DECODE_RTOL, err
    np.testing.assert_allclose(lse.cpu().numpy(), lse_ref, rtol=1e-5,
                               atol=1e-4 * max(1.0, float(np.abs(lse_ref).max()) * 1e-2))
