"""The alternative base code (per-channel keys over 64-token blocks) on the GPU
against the oracle: every plane bit-exact, decode and diagnostics within the
usual tolerances, on the contiguous and the paged layout; and the null-space
intervention of the pages run through the CUDA path end to end."""

import numpy as np
import pytest

import oracle
from bit_decode_attention_sm_b200 import configs, synth
from parity_helpers import (DECODE_RTOL, assert_diag_close, gpu_query, layer, row_rel_err,
                            torch_dtype)

pytestmark = pytest.mark.gpu


def _headq():
    from bit_decode_attention_sm_b200 import headq
    return headq


def channel_cache(w, L, U, T_cap=None, t0=0, chunks=None):
    """A per-channel-key cache holding L's tokens at [t0, t0 + T), written in
    `chunks` (lengths) or one call."""
    import torch
    hq = _headq()
    dt = torch_dtype(w)
    B, Hkv, T, d = L.keys.shape
    T_cap = -(-(t0 + T) // 64) * 64 if T_cap is None else T_cap
    cache = hq.HeadQCache(B, Hkv, T_cap, d, w.r, vmode=w.vmode, v_dtype=dt, kmode="channel")
    Ut = torch.from_numpy(np.ascontiguousarray(U)).cuda()
    pos = 0
    for n in (chunks or [T]):
        k = torch.from_numpy(np.ascontiguousarray(L.keys[:, :, pos:pos + n])).cuda().to(dt)
        v = torch.from_numpy(np.ascontiguousarray(L.values[:, :, pos:pos + n])).cuda().to(dt)
        hq.headq_cache_write(cache, k, v, Ut, t0=t0 + pos)
        pos += n
    return cache, Ut


def assert_channel_planes(cache, ref, w, T, values, t0=0):
    import torch

    def np_(t):
        t = t.cpu()
        return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()
    nb = -(-T // 64)
    b0 = t0 // 64
    np.testing.assert_array_equal(np_(cache.k_codes)[:, :, t0:t0 + T], ref["kc"])
    np.testing.assert_array_equal(np_(cache.k_scale)[:, :, b0:b0 + nb].view(np.uint32),
                                  ref["ks"].view(np.uint32))
    np.testing.assert_array_equal(np_(cache.k_min)[:, :, b0:b0 + nb].view(np.uint32),
                                  ref["km"].view(np.uint32))
    if w.r > 0:
        np.testing.assert_array_equal(np_(cache.z_codes)[:, :, t0:t0 + T, :w.r // 2], ref["zc"])
        np.testing.assert_array_equal(np_(cache.z_scale)[:, :, t0:t0 + T].view(np.uint32),
                                      ref["zs"].view(np.uint32))
    if w.vmode == "2bit":
        np.testing.assert_array_equal(np_(cache.v_codes)[:, :, t0:t0 + T], ref["vc"])
    elif w.kv_dtype == "bf16":
        np.testing.assert_array_equal(np_(cache.v)[:, :, t0:t0 + T], synth.f32_to_bf16_bits(values))


CASES = [(2, dict(T=1000, B=2)), (3, dict(T=2500)), (4, dict(T=700, B=2)), (1, dict(T=300)),
         (0, {})]
IDS = ["cfg%d" % c[0] for c in CASES]


@pytest.mark.parametrize("i,kw", CASES, ids=IDS)
def test_channel_write_and_decode(i, kw):
    hq = _headq()
    w, L = layer(i, **kw)
    B, Hkv, T, d = L.keys.shape
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    ref = oracle.cache_write(L.keys, U, v=L.values, vmode=w.vmode, kmode="channel")
    out_ref, lse_ref = oracle.decode(L.queries, ref, U, v=L.values, vmode=w.vmode,
                                     kmode="channel")
    cache, Ut = channel_cache(w, L, U)
    assert_channel_planes(cache, ref, w, T, L.values)
    out, lse = hq.headq_decode_attn(cache, gpu_query(w, L), Ut, T=T)
    assert row_rel_err(out.cpu().numpy(), out_ref) <= DECODE_RTOL
    np.testing.assert_allclose(lse.cpu().numpy(), lse_ref, rtol=1e-5, atol=1e-4)


def test_channel_write_in_chunks_at_a_block_offset():
    """Three writes (64 + 192 + 44 tokens) starting at block 2 give the planes of
    one write of the 300 tokens."""
    w, L = layer(2, T=300, B=2)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    ref = oracle.cache_write(L.keys, U, v=L.values, vmode=w.vmode, kmode="channel")
    cache, _ = channel_cache(w, L, U, T_cap=512, t0=128, chunks=[64, 192, 44])
    assert_channel_planes(cache, ref, w, 300, L.values, t0=128)


def test_channel_diagnostics_and_ragged():
    import torch
    hq = _headq()
    w, L = layer(2, T=700, B=3)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    ref = oracle.cache_write(L.keys, U, v=L.values, vmode=w.vmode, kmode="channel")
    sl = np.array([700, 65, 0], np.int32)
    cache, Ut = channel_cache(w, L, U)
    out_ref, _ = oracle.decode(L.queries, ref, U, v=L.values, seq_lens=sl, kmode="channel")
    out, lse = hq.headq_decode_attn(cache, gpu_query(w, L), Ut, T=700,
                                    seq_lens=torch.from_numpy(sl).cuda())
    o = out.cpu().numpy()
    assert (o[2] == 0).all()
    assert row_rel_err(o[:2], out_ref[:2]) <= DECODE_RTOL
    diag = oracle.attn_kl(L.queries, ref, U, L.keys, L.values, v=L.values, kmode="channel")
    dt = torch_dtype(w)
    got = hq.headq_attn_kl(cache, gpu_query(w, L), Ut, torch.from_numpy(L.keys).cuda().to(dt),
                           torch.from_numpy(L.values).cuda().to(dt))
    for g, r_, name in zip(got, diag, ("kl", "fisher_var", "a2_vdist", "dout2")):
        assert_diag_close(g.cpu().numpy(), r_, name)


def test_channel_keys_on_a_paged_cache():
    import torch
    hq = _headq()
    w, L = layer(2, T=400, B=2)
    B, Hkv, T, d = L.keys.shape
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    ref = oracle.cache_write(L.keys, U, v=L.values, kmode="channel")
    out_ref, _ = oracle.decode(L.queries, ref, U, v=L.values, kmode="channel")
    table = np.random.default_rng(5).permutation(9)[:8].reshape(2, 4).astype(np.int32)
    dt = torch_dtype(w)
    cache = hq.PagedHeadQCache(B, Hkv, d, w.r, 128, 9, 4, v_dtype=dt, kmode="channel",
                               block_table=torch.from_numpy(table))
    Ut = torch.from_numpy(U).cuda()
    hq.headq_cache_write(cache, torch.from_numpy(L.keys).cuda().to(dt),
                         torch.from_numpy(L.values).cuda().to(dt), Ut)
    # block rows in logical order: page table[b][t // 128], block (t % 128) // 64
    ks = cache.k_scale.cpu().numpy()                      # [pages, Hkv, 2, d]
    got = np.stack([np.concatenate([ks[table[b, i // 2], :, i % 2][:, None] for i in range(7)],
                                   axis=1) for b in range(B)])
    np.testing.assert_array_equal(got.view(np.uint32), ref["ks"].view(np.uint32))
    out, _ = hq.headq_decode_attn(cache, gpu_query(w, L), Ut, T=T)
    assert row_rel_err(out.cpu().numpy(), out_ref) <= DECODE_RTOL


def test_null_space_intervention_through_the_gpu_path():
    """The pages' null-space intervention on the CUDA path: a softmax-null mean
    added to every key multiplies the Fisher damage of the per-token code and
    leaves the per-channel code's unchanged (cache write and diagnostic kernels)."""
    import torch
    hq = _headq()
    w = configs.workload(2).with_(B=2, T=512, n_cal=256)
    L = synth.make_layer(w)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    Ut = torch.from_numpy(U).cuda()
    mu = (16.0 * np.random.default_rng(35).standard_normal(w.d)).astype(np.float32)
    fv = {}
    for mode in ("token", "channel"):
        for tag, k in (("plain", L.keys), ("mean", L.keys + mu)):
            cache = hq.HeadQCache(2, w.Hkv, 512, w.d, w.r, kmode=mode)
            kt = torch.from_numpy(np.ascontiguousarray(k)).cuda()      # fp32 keys
            vt = torch.from_numpy(L.values).cuda()
            hq.headq_cache_write(cache, kt, vt, Ut)
            _, f, _, _ = hq.headq_attn_kl(cache, gpu_query(w, L), Ut, kt, vt)
            fv[mode, tag] = float(f.mean())
    assert fv["token", "mean"] > 2.5 * fv["token", "plain"]
    assert abs(fv["channel", "mean"] / fv["channel", "plain"] - 1) < 0.05
