"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Cache write: every plane bit-exact (fp32 planes compared as bit patterns).
Decode: max relative error per output row <= 2e-3 of the row maximum.
Diagnostics: relative 1e-2 or absolute 1e-6, whichever is looser.
Calibration: projector distance |U U^T - U_ref U_ref^T|_F <= 1e-3, eigenvalues
to relative 1e-4.

Reduced sizes keep each workload's distribution and head layout and still span
several tiles, several T-splits and a ragged tail; the full-size cases run the
exact launch configuration of the benchmark and check sampled rows the oracle
recomputes from scratch.
"""

import numpy as np
import pytest

import oracle
from bit_decode_attention_sm_b200 import configs, synth
from parity_helpers import (DECODE_RTOL, assert_diag_close, assert_planes_equal, gpu_cache,
                            gpu_query, layer, oracle_side, planes_to_numpy, roundup,
                            row_rel_err, torch_dtype)

pytestmark = pytest.mark.gpu

CASES = [(0, {}), (1, dict(T=300)), (2, dict(T=1000, B=2)), (3, dict(T=2500)),
         (4, dict(T=700, B=3))]
IDS = ["cfg%d" % c[0] for c in CASES]


def _headq():
    from bit_decode_attention_sm_b200 import headq
    return headq


@pytest.mark.parametrize("i,kw", CASES, ids=IDS)
def test_cache_write_bit_exact(i, kw):
    w, L = layer(i, **kw)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    ref = oracle.cache_write(L.keys, U, v=L.values, vmode=w.vmode)
    cache, _ = gpu_cache(w, L, U)
    got = planes_to_numpy(cache, 0, L.keys.shape[2])
    assert_planes_equal(got, ref, w.r, w.vmode, w.kv_dtype, values=L.values)


def test_cache_write_chunks_and_offset():
    """A prefill chunk followed by one-token appends at an odd offset writes the
    same planes as the oracle on the whole sequence."""
    import torch
    hq = _headq()
    w, L = layer(2, T=203, B=2)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    ref = oracle.cache_write(L.keys, U, v=L.values)
    dt = torch_dtype(w)
    t0 = 5
    cache = hq.HeadQCache(2, w.Hkv, roundup(t0 + 203, 16), w.d, w.r, v_dtype=dt)
    Ut = torch.from_numpy(U).cuda()
    k = torch.from_numpy(L.keys).cuda().to(dt)
    v = torch.from_numpy(L.values).cuda().to(dt)
    hq.headq_cache_write(cache, k[:, :, :190].contiguous(), v[:, :, :190].contiguous(), Ut,
                         t0=t0)
    for t in range(190, 203):
        hq.headq_cache_write(cache, k[:, :, t:t + 1].contiguous(), v[:, :, t:t + 1].contiguous(),
                             Ut, t0=t0 + t)
    got = planes_to_numpy(cache, t0, 203)
    assert_planes_equal(got, ref, w.r, w.vmode, w.kv_dtype, values=L.values)


@pytest.mark.parametrize("sigma", [1, 0, -1])
@pytest.mark.parametrize("i,kw", CASES, ids=IDS)
def test_decode_matches_oracle(i, kw, sigma):
    hq = _headq()
    w, L = layer(i, **kw)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    _, out_ref, lse_ref = oracle_side(w, L, U, sigma=float(sigma))
    cache, Ut = gpu_cache(w, L, U)
    T = L.keys.shape[2]
    ws = hq.decode_workspace(cache, w.Hq, T)
    out, lse = hq.headq_decode_attn(cache, gpu_query(w, L), Ut, T=T, corr_sign=sigma, ws=ws)
    hq.headq_workspace_status(ws)
    err = row_rel_err(out.cpu().numpy(), out_ref)
    assert err <= DECODE_RTOL, err
    np.testing.assert_allclose(lse.cpu().numpy(), lse_ref, rtol=1e-5, atol=1e-4)


def test_decode_from_oracle_planes():
    """The decode kernel alone: planes written by the oracle, uploaded as they are."""
    import torch
    hq = _headq()
    w, L = layer(3, T=1500)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    planes, out_ref, _ = oracle_side(w, L, U)
    T = L.keys.shape[2]
    cache = hq.HeadQCache(1, w.Hkv, roundup(T, 16), w.d, w.r, v_dtype=torch.bfloat16)
    for name, t in cache.planes().items():
        src = planes[name] if name != "v" else None
        if name == "v":
            t[:, :, :T] = torch.from_numpy(L.values).to(torch.bfloat16).cuda()
        else:
            t[:, :, :T] = torch.from_numpy(np.ascontiguousarray(src)).cuda()
    out, _ = hq.headq_decode_attn(cache, gpu_query(w, L), torch.from_numpy(U).cuda(), T=T)
    assert row_rel_err(out.cpu().numpy(), out_ref) <= DECODE_RTOL


def test_decode_ragged_sequences():
    """Per-sequence lengths 0, 1, 33 and T with capacity beyond T."""
    import torch
    hq = _headq()
    w, L = layer(2, T=777, B=4)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    sl = np.array([0, 1, 33, 777], np.int32)
    _, out_ref, lse_ref = oracle_side(w, L, U, seq_lens=sl)
    cache, Ut = gpu_cache(w, L, U, T_cap=1024)
    out, lse = hq.headq_decode_attn(cache, gpu_query(w, L), Ut, T=777,
                                    seq_lens=torch.from_numpy(sl).cuda())
    o, l = out.cpu().numpy(), lse.cpu().numpy()
    assert (o[0] == 0).all() and np.isneginf(l[0]).all()
    assert row_rel_err(o[1:], out_ref[1:]) <= DECODE_RTOL
    np.testing.assert_allclose(l[1:], lse_ref[1:], rtol=1e-5, atol=1e-4)


SMALL = [  # (d, r, Hq, Hkv, T, B) beyond the five workloads: every head dim, GQA groups
    (8, 4, 2, 1, 16, 2), (16, 2, 4, 2, 45, 1), (32, 8, 8, 1, 130, 2),
    (64, 16, 14, 2, 129, 1), (128, 32, 8, 8, 70, 1), (256, 16, 8, 2, 300, 1),
    (128, 0, 4, 4, 90, 1),
    (64, 16, 24, 2, 100, 1),   # G = 12: the generic kernel's 16-head batch
    (32, 8, 40, 2, 75, 1),     # G = 20: two head passes in the generic kernel
]


@pytest.mark.parametrize("d,r,Hq,Hkv,T,B", SMALL)
@pytest.mark.parametrize("kv_dtype,vmode", [("bf16", "dense"), ("f32", "dense"),
                                            ("bf16", "2bit")])
def test_small_shapes(d, r, Hq, Hkv, T, B, kv_dtype, vmode):
    hq = _headq()
    base = configs.workload(1)
    w = base.with_(d=d, r=r, r_s=max(2, min(8, d // 2)), Hq=Hq, Hkv=Hkv, B=B, T=T,
                   n_cal=64, kv_dtype=kv_dtype, vmode=vmode)
    L = synth.make_layer(w)
    if r > 0:
        U, _ = oracle.calibrate(L.q_cal, Hkv, r)
    else:
        U = np.zeros((Hkv, d, 0), np.float32)
    planes, out_ref, lse_ref = oracle_side(w, L, U)
    cache, Ut = gpu_cache(w, L, U)
    got = planes_to_numpy(cache, 0, T)
    assert_planes_equal(got, planes, r, vmode, kv_dtype, values=L.values)
    out, lse = hq.headq_decode_attn(cache, gpu_query(w, L), Ut, T=T)
    assert row_rel_err(out.cpu().numpy(), out_ref) <= DECODE_RTOL
    np.testing.assert_allclose(lse.cpu().numpy(), lse_ref, rtol=1e-5, atol=1e-4)


@pytest.mark.parametrize("sigma", [1, -1])
@pytest.mark.parametrize("i,kw", CASES, ids=IDS)
def test_attn_kl_matches_oracle(i, kw, sigma):
    import torch
    hq = _headq()
    w, L = layer(i, **kw)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    planes = oracle.cache_write(L.keys, U, v=L.values, vmode=w.vmode)
    ref = oracle.attn_kl(L.queries, planes, U, L.keys, L.values, v=L.values, vmode=w.vmode,
                         sigma=float(sigma))
    cache, Ut = gpu_cache(w, L, U)
    dt = torch_dtype(w)
    kf = torch.from_numpy(L.keys).cuda().to(dt)
    vf = torch.from_numpy(L.values).cuda().to(dt)
    got = hq.headq_attn_kl(cache, gpu_query(w, L), Ut, kf, vf, corr_sign=sigma)
    for g, r_, name in zip(got, ref, ("kl", "fisher_var", "a2_vdist", "dout2")):
        assert_diag_close(g.cpu().numpy(), r_, name)


@pytest.mark.parametrize("i", [0, 1, 2, 3, 4])
@pytest.mark.parametrize("center", [False, True])
def test_calibrate_matches_oracle(i, center):
    import torch
    hq = _headq()
    w, L = layer(i, T=16, B=1)
    U_ref, eig_ref = oracle.calibrate(L.q_cal, w.Hkv, w.r, center=center)
    q = torch.from_numpy(L.q_cal).cuda().to(torch_dtype(w))
    U, eig = hq.headq_calibrate(q, w.Hkv, w.r, center=center)
    U, eig = U.cpu().numpy().astype(np.float64), eig.cpu().numpy()
    for kv in range(w.Hkv):
        P = U[kv] @ U[kv].T
        Pr = U_ref[kv].astype(np.float64) @ U_ref[kv].T.astype(np.float64)
        assert np.linalg.norm(P - Pr) <= 1e-3
        np.testing.assert_allclose(eig[kv], eig_ref[kv], rtol=1e-4)
        # same sign rule: columns agree, not just the subspace
        assert np.abs(U[kv] - U_ref[kv]).max() <= 1e-3


def test_wrong_sign_and_base_only_through_the_abi():
    """Section 4 control on the GPU: sigma=-1 gives larger KL than sigma=0 and +1."""
    import torch
    hq = _headq()
    w, L = layer(2, T=512, B=2)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    cache, Ut = gpu_cache(w, L, U)
    dt = torch_dtype(w)
    kf = torch.from_numpy(L.keys).cuda().to(dt)
    vf = torch.from_numpy(L.values).cuda().to(dt)
    q = gpu_query(w, L)
    kl = {s: hq.headq_attn_kl(cache, q, Ut, kf, vf, corr_sign=s)[0].mean().item()
          for s in (1, 0, -1)}
    assert kl[1] < kl[0] < kl[-1], kl


FULL = [1, 2, 3, 4]


@pytest.mark.parametrize("i", FULL, ids=["cfg%d-full" % i for i in FULL])
def test_full_size_sampled_rows(i):
    """Full workload size, the benchmark's launch configuration; the oracle
    re-encodes two sampled (b, kv) sequences from the inputs and decodes their
    query heads."""
    import torch
    hq = _headq()
    w = configs.workload(i)
    L = synth.make_layer(w)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    cache, Ut = gpu_cache(w, L, U)
    out, lse = hq.headq_decode_attn(cache, gpu_query(w, L), Ut, T=w.T)
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    rng = np.random.default_rng(100 + i)
    picks = {(int(rng.integers(w.B)), int(rng.integers(w.Hkv))) for _ in range(2)}
    for b, kv in sorted(picks):
        sub = synth.LayerInputs(L.keys[b:b + 1, kv:kv + 1], L.values[b:b + 1, kv:kv + 1],
                                L.queries[b:b + 1, kv * w.G:(kv + 1) * w.G], None, {})
        w1 = w.with_(B=1, Hkv=1, Hq=w.G)
        planes, out_ref, lse_ref = oracle_side(w1, sub, U[kv:kv + 1])
        got = planes_to_numpy(cache, 0, w.T, b=b, kv=kv)
        assert_planes_equal(got, planes, w.r, w.vmode, w.kv_dtype, values=sub.values)
        o = out[b:b + 1, kv * w.G:(kv + 1) * w.G]
        assert row_rel_err(o, out_ref) <= DECODE_RTOL
        np.testing.assert_allclose(lse[b:b + 1, kv * w.G:(kv + 1) * w.G], lse_ref,
                                   rtol=1e-5, atol=1e-4)
    del cache
    torch.cuda.empty_cache()


APPEND_FULL = [2, 3, 4]


@pytest.mark.parametrize("i", APPEND_FULL, ids=["cfg%d-full-append" % i for i in APPEND_FULL])
def test_full_size_decode_append(i):
    """The benchmarked call at full size in the benchmark's launch plan:
    headq_decode_append writes every sequence's token T-1 into a cache whose
    position T-1 held other data, then attends over all T tokens.  The new
    token's planes are bit-exact for every (b, kv); the outputs of every query
    head are compared with the oracle on the long-context layer (one sequence,
    8 KV heads, T = 131072), and on four sampled (b, kv) sequences of the
    batched layers."""
    import torch
    hq = _headq()
    w = configs.workload(i)
    L = synth.make_layer(w)
    B, Hkv, T, d = L.keys.shape
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    stale = synth.LayerInputs(L.keys.copy(), L.values.copy(), L.queries, L.q_cal, {})
    rng = np.random.default_rng(7)
    stale.keys[:, :, T - 1] = synth.round_bf16(rng.standard_normal((B, Hkv, d)).astype(np.float32))
    stale.values[:, :, T - 1] = synth.round_bf16(rng.standard_normal((B, Hkv, d)).astype(np.float32))
    cache, Ut = gpu_cache(w, stale, U)
    del stale
    dt = torch_dtype(w)
    k_new = torch.from_numpy(np.ascontiguousarray(L.keys[:, :, T - 1])).cuda().to(dt)
    v_new = torch.from_numpy(np.ascontiguousarray(L.values[:, :, T - 1])).cuda().to(dt)
    splits, chunk, _, _ = hq.decode_plan(cache, w.Hq, T)
    assert splits >= 1
    ws = hq.decode_workspace(cache, w.Hq, T)
    out, lse = hq.headq_decode_append(cache, k_new, v_new, gpu_query(w, L), Ut, T=T, ws=ws)
    hq.headq_workspace_status(ws)
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    # the appended token of every (b, kv), bit-exact
    new_planes = oracle.cache_write(L.keys[:, :, T - 1:T], U, v=L.values[:, :, T - 1:T],
                                    vmode=w.vmode)
    got = planes_to_numpy(cache, T - 1, 1)
    new_planes.pop("y", None)
    assert_planes_equal(got, new_planes, w.r, w.vmode, w.kv_dtype,
                        values=L.values[:, :, T - 1:T])
    if B * Hkv <= 8:
        pairs = [(b, kv) for b in range(B) for kv in range(Hkv)]
    else:
        r2 = np.random.default_rng(200 + i)
        pairs = sorted({(int(r2.integers(B)), int(r2.integers(Hkv))) for _ in range(4)})
    for b, kv in pairs:
        sub = synth.LayerInputs(L.keys[b:b + 1, kv:kv + 1], L.values[b:b + 1, kv:kv + 1],
                                L.queries[b:b + 1, kv * w.G:(kv + 1) * w.G], None, {})
        w1 = w.with_(B=1, Hkv=1, Hq=w.G)
        _, out_ref, lse_ref = oracle_side(w1, sub, U[kv:kv + 1])
        o = out[b:b + 1, kv * w.G:(kv + 1) * w.G]
        assert row_rel_err(o, out_ref) <= DECODE_RTOL, (b, kv)
        np.testing.assert_allclose(lse[b:b + 1, kv * w.G:(kv + 1) * w.G], lse_ref,
                                   rtol=1e-5, atol=1e-4)
    del cache
    torch.cuda.empty_cache()


def test_one_workspace_reused_across_shapes():
    """A decode workspace sized for the largest call serves calls of different
    shapes in any order: partials of one call never disturb the next."""
    import ctypes
    hq = _headq()
    cases = []
    for i, kw in ((2, dict(T=1000, B=2)), (1, dict(T=300)), (3, dict(T=2500)), (1, dict(T=700))):
        w, L = layer(i, **kw)
        U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
        _, out_ref, lse_ref = oracle_side(w, L, U)
        cache, Ut = gpu_cache(w, L, U)
        cases.append((w, L, cache, Ut, out_ref, lse_ref))
    need = max(hq.lib().headq_decode_workspace_bytes(ctypes.byref(c[2].struct()), c[0].Hq,
                                                     c[1].keys.shape[2]) for c in cases)
    import torch
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for rep in range(2):
        for w, L, cache, Ut, out_ref, lse_ref in cases:
            out, lse = hq.headq_decode_attn(cache, gpu_query(w, L), Ut, T=L.keys.shape[2], ws=ws)
            assert row_rel_err(out.cpu().numpy(), out_ref) <= DECODE_RTOL
            np.testing.assert_allclose(lse.cpu().numpy(), lse_ref, rtol=1e-5, atol=1e-4)
    hq.headq_workspace_status(ws)


def _edge_keys(d, T, seed):
    """Keys built to stress the codec's rounding: exact ties (x - min)/scale =
    k + 1/2, near-ties a few ulp away, constant, signed-zero, subnormal, tiny
    normal and huge groups, and side-code inputs on a coarse dyadic grid."""
    rng = np.random.default_rng(seed)
    gs = min(32, d)
    k = np.zeros((1, 1, T, d), np.float32)
    for t in range(T):
        for g in range(d // gs):
            kind = t % 8
            if kind == 0:     # integer levels 0..6 over span 6 -> scale 2, ties at 1, 3, 5
                x = rng.integers(0, 7, gs).astype(np.float32)
                x[0], x[1] = 0, 6
            elif kind == 1:   # near-ties: tie values nudged by -4..4 ulp
                x = rng.integers(0, 7, gs).astype(np.float32)
                x[0], x[1] = 0, 6
                nudge = rng.integers(-4, 5, gs)
                for j in range(2, gs):
                    for _ in range(abs(int(nudge[j]))):
                        x[j] = np.nextafter(x[j], np.float32(np.inf if nudge[j] > 0 else -np.inf))
            elif kind == 2:   # constant group: scale 0, all codes 0
                x = np.full(gs, rng.standard_normal(), np.float32)
            elif kind == 3:   # signed zeros and zeros
                x = np.where(rng.random(gs) < 0.5, np.float32(-0.0), np.float32(0.0))
            elif kind == 4:   # subnormal group
                x = (rng.integers(0, 9, gs) * np.float32(2.0 ** -149)).astype(np.float32)
            elif kind == 5:   # tiny normals around 1e-37
                x = (rng.standard_normal(gs) * 1e-37).astype(np.float32)
            elif kind == 6:   # huge values
                x = (rng.standard_normal(gs) * 1e30).astype(np.float32)
            else:             # dyadic grid: residuals and side codes hit exact ratios
                x = (rng.integers(-64, 65, gs) / 16.0).astype(np.float32)
            k[0, 0, t, g * gs:(g + 1) * gs] = x
    return k


@pytest.mark.parametrize("d,r", [(32, 8), (128, 16), (64, 2), (8, 4)])
def test_cache_write_rounding_edges_bit_exact(d, r):
    import torch
    hq = _headq()
    T = 96
    k = _edge_keys(d, T, seed=d + r)
    v = _edge_keys(d, T, seed=d + r + 1)
    rng = np.random.default_rng(5)
    # a dyadic basis (entries k/8): projections of dyadic residuals are exact, so
    # side-code quotients land on ties too; plus a random orthonormal basis
    for U in (np.stack([np.round(synth.random_orthonormal(rng, d, r) * 8) / 8]).astype(np.float32),
              np.stack([synth.random_orthonormal(rng, d, r)])):
        for vmode in ("dense", "2bit"):
            ref = oracle.cache_write(k, U, v=v, vmode=vmode)
            cache = hq.HeadQCache(1, 1, T, d, r, vmode=vmode, v_dtype=torch.float32)
            hq.headq_cache_write(cache, torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(),
                                 torch.from_numpy(np.ascontiguousarray(U)).cuda())
            got = planes_to_numpy(cache, 0, T)
            assert_planes_equal(got, ref, r, vmode, "f32", values=v)


APPEND_CASES = [
    (3, dict(T=2500), None),
    (2, dict(T=700, B=4), np.array([700, 1, 0, 333], np.int32)),
    (1, dict(T=300), np.array([300, 17, 1, 64, 299, 150, 0, 65], np.int32)),
    (4, dict(T=500, B=2), np.array([500, 250], np.int32)),    # 2-bit V: generic path
    (0, {}, None),                                             # fp32 V: generic path
]


@pytest.mark.parametrize("i,kw,sl", APPEND_CASES, ids=["cfg%d" % c[0] for c in APPEND_CASES])
def test_decode_append_matches_oracle(i, kw, sl):
    """headq_decode_append: each sequence's new token written at T_b - 1 (planes
    bit-exact) and the attention over tokens < T_b, in one call."""
    import torch
    hq = _headq()
    w, L = layer(i, **kw)
    B, Hkv, T, d = L.keys.shape
    lens = np.full(B, T, np.int32) if sl is None else sl
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    planes, out_ref, lse_ref = oracle_side(w, L, U, seq_lens=sl)
    # cache holding every token except the new ones (those positions hold other data)
    stale = synth.LayerInputs(L.keys.copy(), L.values.copy(), L.queries, L.q_cal, {})
    rng = np.random.default_rng(1)
    for b in range(B):
        if lens[b] > 0:
            stale.keys[b, :, lens[b] - 1] = rng.standard_normal((Hkv, d)).astype(np.float32)
            stale.values[b, :, lens[b] - 1] = rng.standard_normal((Hkv, d)).astype(np.float32)
    if w.kv_dtype == "bf16":
        stale.keys = synth.round_bf16(stale.keys)
        stale.values = synth.round_bf16(stale.values)
    cache, Ut = gpu_cache(w, stale, U)
    dt = torch_dtype(w)
    pos = np.maximum(lens - 1, 0)
    k_new = torch.from_numpy(np.ascontiguousarray(L.keys[np.arange(B), :, pos])).cuda().to(dt)
    v_new = torch.from_numpy(np.ascontiguousarray(L.values[np.arange(B), :, pos])).cuda().to(dt)
    slt = None if sl is None else torch.from_numpy(sl).cuda()
    ws = hq.decode_workspace(cache, w.Hq, T)
    out, lse = hq.headq_decode_append(cache, k_new, v_new, gpu_query(w, L), Ut, T=T,
                                      seq_lens=slt, ws=ws)
    hq.headq_workspace_status(ws)
    o, l_ = out.cpu().numpy(), lse.cpu().numpy()
    assert row_rel_err(o, out_ref) <= DECODE_RTOL
    np.testing.assert_allclose(l_, lse_ref, rtol=1e-5, atol=1e-4)
    got = planes_to_numpy(cache, 0, T)
    for b in range(B):
        if lens[b] == 0:
            continue
        p_ = lens[b] - 1
        one = {k: a[b:b + 1, :, p_:p_ + 1] for k, a in got.items()}
        ref1 = {k: a[b:b + 1, :, p_:p_ + 1] for k, a in planes.items() if k != "y"}
        assert_planes_equal(one, ref1, w.r, w.vmode, w.kv_dtype,
                            values=L.values[b:b + 1, :, p_:p_ + 1])


def test_decode_append_without_values_keeps_v():
    """v_new = NULL writes the key planes only; the cached value stays."""
    import torch
    hq = _headq()
    w, L = layer(2, T=300, B=2)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    cache, Ut = gpu_cache(w, L, U)
    before = cache.v.clone()
    k_new = torch.from_numpy(np.ascontiguousarray(L.keys[:, :, -1])).cuda().to(torch.bfloat16)
    out, _ = hq.headq_decode_append(cache, k_new, None, gpu_query(w, L), Ut, T=300)
    assert torch.equal(cache.v, before)
    _, out_ref, _ = oracle_side(w, L, U)
    assert row_rel_err(out.cpu().numpy(), out_ref) <= DECODE_RTOL
