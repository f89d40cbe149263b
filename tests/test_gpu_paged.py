"""Paged cache layout vs the CPU oracle, through the C ABI.

A paged cache keeps each plane as a pool of fixed-size pages and maps every
sequence's logical pages to pool pages with a block table.  The placement is
pure data movement, so the oracle (which knows only the contiguous layout) is
still the reference: the GPU planes are gathered back into logical order with
the block table and compared bit-exactly; decode, decode-and-append and the
diagnostics are compared with the same tolerances as the contiguous layout.
Block tables here are random permutations of a pool larger than needed, so
neighbouring logical pages are never neighbours in memory.
"""

import numpy as np
import pytest

import oracle
from bit_decode_attention_sm_b200 import configs, synth
from parity_helpers import (DECODE_RTOL, assert_diag_close, assert_planes_equal, gpu_query,
                            layer, oracle_side, row_rel_err, torch_dtype)

pytestmark = pytest.mark.gpu


def _headq():
    from bit_decode_attention_sm_b200 import headq
    return headq


def paged_cache(w, L, U, page_size, seed=0, spare=5, write=True, T_cap=None):
    """A paged cache holding L's keys/values at logical positions [0, T), its
    block table a random injection into a pool with `spare` unused pages."""
    import torch
    hq = _headq()
    B, Hkv, T, d = L.keys.shape
    max_pages = -(-(T if T_cap is None else T_cap) // page_size)
    num_pages = B * max_pages + spare
    rng = np.random.default_rng(seed)
    table = rng.permutation(num_pages)[:B * max_pages].reshape(B, max_pages).astype(np.int32)
    dt = torch_dtype(w)
    cache = hq.PagedHeadQCache(B, Hkv, d, w.r, page_size, num_pages, max_pages, vmode=w.vmode,
                               v_dtype=dt, block_table=torch.from_numpy(table))
    Ut = torch.from_numpy(np.ascontiguousarray(U)).cuda()
    if write:
        k = torch.from_numpy(L.keys).cuda().to(dt)
        v = torch.from_numpy(L.values).cuda().to(dt)
        hq.headq_cache_write(cache, k, v, Ut, t0=0)
    return cache, Ut


def gathered(cache, T):
    """Every plane in logical order [B, Hkv, T, ...] as numpy (bf16 as uint16)."""
    import torch
    bt = cache.block_table.long()
    B, P = bt.shape
    out = {}
    for name, t in cache.planes().items():
        g = t[bt.reshape(-1)]                              # [B*P, Hkv, ps, ...]
        g = g.reshape((B, P) + tuple(t.shape[1:])).transpose(1, 2)
        g = g.reshape((B, t.shape[1], P * t.shape[2]) + tuple(t.shape[3:]))[:, :, :T]
        g = g.contiguous().cpu()
        out[name] = (g.view(torch.int16).numpy().view(np.uint16) if g.dtype == torch.bfloat16
                     else g.numpy())
    return out


CASES = [  # (workload, reduced sizes, page size)
    (2, dict(T=1000, B=3), 64),      # tensor-core decode, G = 7
    (3, dict(T=2500), 256),          # G = 4, long pages
    (1, dict(T=300), 128),           # d = 64
    (4, dict(T=700, B=2), 64),       # 2-bit values
    (0, {}, 128),                    # fp32 keys and values
]
IDS = ["cfg%d-p%d" % (c[0], c[2]) for c in CASES]


@pytest.mark.parametrize("i,kw,ps", CASES, ids=IDS)
def test_paged_write_and_decode(i, kw, ps):
    import torch
    hq = _headq()
    w, L = layer(i, **kw)
    B, Hkv, T, d = L.keys.shape
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    planes, out_ref, lse_ref = oracle_side(w, L, U)
    cache, Ut = paged_cache(w, L, U, ps)
    assert_planes_equal(gathered(cache, T), planes, w.r, w.vmode, w.kv_dtype, values=L.values)
    ws = hq.decode_workspace(cache, w.Hq, T)
    out, lse = hq.headq_decode_attn(cache, gpu_query(w, L), Ut, T=T, ws=ws)
    hq.headq_workspace_status(ws)
    assert row_rel_err(out.cpu().numpy(), out_ref) <= DECODE_RTOL
    np.testing.assert_allclose(lse.cpu().numpy(), lse_ref, rtol=1e-5, atol=1e-4)


def test_paged_matches_contiguous_write_at_offset():
    """A write starting mid-page (t0 not a multiple of the page size) lands in
    the right pages: planes for [t0, t0 + n) equal the oracle's."""
    import torch
    hq = _headq()
    w, L = layer(2, T=300, B=2)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    planes = oracle.cache_write(L.keys, U, v=L.values, vmode=w.vmode)
    t0 = 37
    cache, Ut = paged_cache(w, L, U, 64, write=False, T_cap=t0 + 300)
    dt = torch_dtype(w)
    k = torch.from_numpy(L.keys).cuda().to(dt)
    v = torch.from_numpy(L.values).cuda().to(dt)
    hq.headq_cache_write(cache, k, v, Ut, t0=t0)
    got = {n: a[:, :, t0:] for n, a in gathered(cache, t0 + 300).items()}
    assert_planes_equal(got, planes, w.r, w.vmode, w.kv_dtype, values=L.values)


def test_paged_ragged_sequences():
    """Lengths 0, 1, 65 and T; the pages past each length are never touched."""
    import torch
    hq = _headq()
    w, L = layer(2, T=777, B=4)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    sl = np.array([0, 1, 65, 777], np.int32)
    _, out_ref, lse_ref = oracle_side(w, L, U, seq_lens=sl)
    cache, Ut = paged_cache(w, L, U, 128, T_cap=1024)
    out, lse = hq.headq_decode_attn(cache, gpu_query(w, L), Ut, T=777,
                                    seq_lens=torch.from_numpy(sl).cuda())
    o, l_ = out.cpu().numpy(), lse.cpu().numpy()
    assert (o[0] == 0).all() and np.isneginf(l_[0]).all()
    assert row_rel_err(o[1:], out_ref[1:]) <= DECODE_RTOL
    np.testing.assert_allclose(l_[1:], lse_ref[1:], rtol=1e-5, atol=1e-4)


@pytest.mark.parametrize("d,r,Hq,Hkv,T,B", [(32, 8, 8, 1, 300, 2), (256, 16, 8, 2, 200, 1)])
def test_paged_generic_kernel(d, r, Hq, Hkv, T, B):
    """Head dims outside the tensor-core kernel use the generic split kernel."""
    hq = _headq()
    w = configs.workload(1).with_(d=d, r=r, r_s=8, Hq=Hq, Hkv=Hkv, B=B, T=T, n_cal=64)
    L = synth.make_layer(w)
    U, _ = oracle.calibrate(L.q_cal, Hkv, r)
    planes, out_ref, _ = oracle_side(w, L, U)
    cache, Ut = paged_cache(w, L, U, 64)
    assert_planes_equal(gathered(cache, T), planes, r, w.vmode, w.kv_dtype, values=L.values)
    out, _ = hq.headq_decode_attn(cache, gpu_query(w, L), Ut, T=T)
    assert row_rel_err(out.cpu().numpy(), out_ref) <= DECODE_RTOL


@pytest.mark.parametrize("i,kw,sl", [(2, dict(T=640, B=3), [640, 64, 1]),
                                     (4, dict(T=300, B=2), None)], ids=["cfg2", "cfg4"])
def test_paged_decode_append(i, kw, sl):
    """One serving step on a paged cache: the new token lands at T_b - 1 of the
    right page (bit-exact) and the attention includes it."""
    import torch
    hq = _headq()
    w, L = layer(i, **kw)
    B, Hkv, T, d = L.keys.shape
    sl = None if sl is None else np.array(sl, np.int32)
    lens = np.full(B, T, np.int32) if sl is None else sl
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    planes, out_ref, lse_ref = oracle_side(w, L, U, seq_lens=sl)
    stale = synth.LayerInputs(L.keys.copy(), L.values.copy(), L.queries, L.q_cal, {})
    rng = np.random.default_rng(3)
    for b in range(B):
        stale.keys[b, :, lens[b] - 1] = rng.standard_normal((Hkv, d)).astype(np.float32)
        stale.values[b, :, lens[b] - 1] = rng.standard_normal((Hkv, d)).astype(np.float32)
    if w.kv_dtype == "bf16":
        stale.keys = synth.round_bf16(stale.keys)
        stale.values = synth.round_bf16(stale.values)
    cache, Ut = paged_cache(w, stale, U, 64)
    dt = torch_dtype(w)
    pos = lens - 1
    k_new = torch.from_numpy(np.ascontiguousarray(L.keys[np.arange(B), :, pos])).cuda().to(dt)
    v_new = torch.from_numpy(np.ascontiguousarray(L.values[np.arange(B), :, pos])).cuda().to(dt)
    slt = None if sl is None else torch.from_numpy(sl).cuda()
    ws = hq.decode_workspace(cache, w.Hq, T)
    out, lse = hq.headq_decode_append(cache, k_new, v_new, gpu_query(w, L), Ut, T=T,
                                      seq_lens=slt, ws=ws)
    hq.headq_workspace_status(ws)
    assert row_rel_err(out.cpu().numpy(), out_ref) <= DECODE_RTOL
    np.testing.assert_allclose(lse.cpu().numpy(), lse_ref, rtol=1e-5, atol=1e-4)
    got = gathered(cache, T)
    for b in range(B):
        p_ = lens[b] - 1
        one = {k: a[b:b + 1, :, p_:p_ + 1] for k, a in got.items()}
        ref1 = {k: a[b:b + 1, :, p_:p_ + 1] for k, a in planes.items() if k != "y"}
        assert_planes_equal(one, ref1, w.r, w.vmode, w.kv_dtype,
                            values=L.values[b:b + 1, :, p_:p_ + 1])


def test_paged_attn_kl():
    import torch
    hq = _headq()
    w, L = layer(2, T=500, B=2)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    planes = oracle.cache_write(L.keys, U, v=L.values, vmode=w.vmode)
    ref = oracle.attn_kl(L.queries, planes, U, L.keys, L.values, v=L.values, vmode=w.vmode)
    cache, Ut = paged_cache(w, L, U, 128)
    dt = torch_dtype(w)
    kf = torch.from_numpy(L.keys).cuda().to(dt)
    vf = torch.from_numpy(L.values).cuda().to(dt)
    got = hq.headq_attn_kl(cache, gpu_query(w, L), Ut, kf, vf)
    for g, r_, name in zip(got, ref, ("kl", "fisher_var", "a2_vdist", "dout2")):
        assert_diag_close(g.cpu().numpy(), r_, name)


def test_block_table_entry_outside_pool_is_reported():
    """An entry outside [0, num_pages) is caught by the kernels' own range check:
    the read is redirected to page 0 and the workspace error word is raised;
    the other sequences are unaffected."""
    import torch
    hq = _headq()
    w, L = layer(2, T=256, B=2)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    _, out_ref, _ = oracle_side(w, L, U)
    cache, Ut = paged_cache(w, L, U, 64)
    cache.block_table[0, 1] = cache.num_pages + 7
    ws = hq.decode_workspace(cache, w.Hq, 256)
    out, _ = hq.headq_decode_attn(cache, gpu_query(w, L), Ut, T=256, ws=ws)
    with pytest.raises(hq.HeadQError):
        hq.headq_workspace_status(ws)
    hq.headq_workspace_status(ws)  # the word was cleared
    assert row_rel_err(out[1:].cpu().numpy(), out_ref[1:]) <= DECODE_RTOL
