"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test ties one oracle function to something fixed independently: a value
derived by hand from the definition, an exhaustive search on a tiny input,
exact rational arithmetic, a closed form, an invariant the HeadQ pages state
(gist.science technical summary of "HeadQ: Model-Visible Distortion and
Score-Space Correction for KV-Cache Quantization", sections 2-4), or a library
routine (torch scaled_dot_product_attention, scipy entropy, numpy eigh/cov).
A plausible slip in the oracle (a dropped term, a wrong sign, a transposed U,
a wrong packing position, a reversed KL) fails at least one of them; the
mutation tests in test_oracle_mutants.py check that claim.
"""

from fractions import Fraction

import numpy as np
import pytest

import oracle
from bit_decode_attention_sm_b200 import configs, synth


def _codes2(packed, d):
    c = np.arange(d)
    return (packed[..., c // 4] >> (2 * (c % 4))) & 3


def _nibbles(zc, r):
    i = np.arange(r)
    v = (zc[..., i // 2] >> (4 * (i % 2))) & 0xF
    return np.where(v >= 8, v.astype(np.int32) - 16, v.astype(np.int32))


def _round_f32(x: Fraction) -> np.float32:
    """Correctly rounded (nearest, ties to even) fp32 of an exact rational."""
    f = np.float32(float(x))
    cands = {float(f), float(np.nextafter(f, np.float32(-np.inf))),
             float(np.nextafter(f, np.float32(np.inf)))}

    def key(c):
        return (abs(Fraction(c) - x), int(np.float32(c).view(np.uint32)) & 1)

    return np.float32(min(cands, key=key))


def _rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------------------
# Codec: values derived by hand from the definitions.
# ---------------------------------------------------------------------------

def test_base_code_hand_example():
    # d = 8 (one group of 8).  min 0, max 3 -> scale 1, codes = rint(x):
    # 0.25 -> 0, 0.5 -> 0 (tie to even), 0.75 -> 1, 1.5 -> 2 (tie to even),
    # 2.9 -> 3.  Packing puts channel c at bit 2*(c%4) of byte c/4:
    # byte0 = 0 | 0<<2 | 0<<4 | 1<<6 = 0x40, byte1 = 2 | 3<<2 | 3<<4 | 1<<6 = 0x7E.
    x = np.array([[0.0, 0.25, 0.5, 0.75, 1.5, 3.0, 2.9, 1.0]], np.float32)
    codes, sc, mn = oracle.base_quantize(x)
    assert codes.tolist() == [[0x40, 0x7E]]
    assert sc.tolist() == [[1.0]] and mn.tolist() == [[0.0]]
    # dequantised: min + code*scale
    assert oracle.base_dequantize(codes, sc, mn).tolist() == \
        [[0.0, 0.0, 0.0, 1.0, 2.0, 3.0, 3.0, 1.0]]


def test_base_code_two_groups_hand_example():
    # d = 64: group 0 spans [-6, 0] -> scale 2; group 1 is constant 5 -> scale 0,
    # every code 0 and the dequantised value is the minimum.
    x = np.zeros((1, 64), np.float32)
    x[0, :32] = -3.0
    x[0, 0] = -6.0
    x[0, 1] = 0.0
    x[0, 2] = -1.0   # (-1 + 6)/2 = 2.5 -> 2 (tie to even)
    x[0, 3] = -5.0   # 0.5 -> 0 (tie to even)
    x[0, 32:] = 5.0
    codes, sc, mn = oracle.base_quantize(x)
    assert sc.tolist() == [[2.0, 0.0]] and mn.tolist() == [[-6.0, 5.0]]
    c = _codes2(codes, 64)[0]
    assert c[:4].tolist() == [0, 3, 2, 0]
    assert (c[4:32] == 2).all()       # -3 -> (3/2) = 1.5 -> 2
    assert (c[32:] == 0).all()
    assert codes[0, 0] == (0 | 3 << 2 | 2 << 4 | 0 << 6)


def test_negative_zero_extremes_store_positive_zero():
    x = np.array([[-0.0, 0.0, 0.0, -0.0, 0.0, -0.0, -0.0, 0.0]], np.float32)
    codes, sc, mn = oracle.base_quantize(x)
    assert mn.view(np.uint32).tolist() == [[0]] and sc.view(np.uint32).tolist() == [[0]]
    assert codes.tolist() == [[0, 0]]


def test_side_code_hand_example():
    # max|y| = 7 -> s = 1; w = rint(y): 3.5 -> 4 (tie to even), -7, 1.75 -> 2, 0.
    # Nibbles (two's complement): 4 -> 0x4, -7 -> 0x9, 2 -> 0x2, 0 -> 0x0;
    # even index in the low nibble: bytes 0x94, 0x02.
    zc, zs = oracle.side_quantize(np.array([[3.5, -7.0, 1.75, 0.0]], np.float32))
    assert zc.tolist() == [[0x94, 0x02]] and zs.tolist() == [1.0]
    assert oracle.side_dequantize(zc, zs).tolist() == [[4.0, -7.0, 2.0, 0.0]]
    # all-zero projection: s = 0, every code 0
    zc, zs = oracle.side_quantize(np.zeros((1, 4), np.float32))
    assert zc.tolist() == [[0, 0]] and zs.tolist() == [0.0]


# ---------------------------------------------------------------------------
# Codec: exhaustive search and exact arithmetic on tiny inputs (d = 8, T = 16).
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d", [8, 32, 64])
def test_base_code_is_nearest_level(d):
    rng = _rng(d)
    x = (rng.standard_normal((16, d)) * rng.uniform(0.1, 10)).astype(np.float32)
    x = synth.round_bf16(x)
    # a subnormal token: the scale rounds so coarsely that the clamp to 3 acts
    tiny = np.float32(2.0 ** -149)
    # (span 4 ulp -> scale rounds to 1 ulp -> the top value reads 4, clamped to 3)
    x[15] = tiny * rng.integers(0, 5, size=d).astype(np.float32)
    x[15, ::min(32, d)] = 0
    x[15, 1::min(32, d)] = tiny * 4
    codes, sc, mn = oracle.base_quantize(x)
    gs = min(32, d)
    c = _codes2(codes, d)
    for t in range(16):
        for g in range(d // gs):
            xg = x[t, g * gs:(g + 1) * gs]
            assert mn[t, g] == np.min(xg)
            assert sc[t, g] == np.float32((np.max(xg) - np.min(xg))) / np.float32(3)
            for k in range(gs):
                u = np.float32(xg[k] - mn[t, g]) / sc[t, g]   # fp32 quotient
                dist = [abs(float(u) - lvl) for lvl in range(4)]
                best = min(dist)
                cands = [lvl for lvl in range(4) if dist[lvl] == best]
                want = cands[0] if len(cands) == 1 else [v for v in cands if v % 2 == 0][0]
                assert c[t, g * gs + k] == want


# ---------------------------------------------------------------------------
# The alternative base code: per-channel keys over 64-token blocks.
# ---------------------------------------------------------------------------

def test_channel_code_hand_example():
    # d = 8, three tokens.  Channel 0 holds 1, 4, 2.5 -> min 1, scale 1, codes
    # 0, 3, 2 (1.5 ties to even); channel 1 is constant -> scale 0, codes 0;
    # every other channel holds 0, 3, 1.5 -> codes 0, 3, 2.
    # Token 0 byte0 = 0|0<<2|0<<4|0<<6 = 0x00; token 1: 3|0<<2|3<<4|3<<6 = 0xF3;
    # token 2: 2|0<<2|2<<4|2<<6 = 0xA2 (bytes 1 repeat channels 4..7: 0x00, 0xFF, 0xAA).
    x = np.zeros((1, 1, 3, 8), np.float32)
    x[0, 0, :, 0] = [1.0, 4.0, 2.5]
    x[0, 0, :, 1] = 7.0
    for c in range(2, 8):
        x[0, 0, :, c] = [0.0, 3.0, 1.5]
    U = np.zeros((1, 8, 2), np.float32)
    pl = oracle.cache_write(x, U, kmode="channel")
    assert pl["ks"].shape == (1, 1, 1, 8)
    np.testing.assert_array_equal(pl["km"][0, 0, 0], [1, 7, 0, 0, 0, 0, 0, 0])
    np.testing.assert_array_equal(pl["ks"][0, 0, 0], [1, 0, 1, 1, 1, 1, 1, 1])
    np.testing.assert_array_equal(pl["kc"][0, 0], [[0x00, 0x00], [0xF3, 0xFF], [0xA2, 0xAA]])
    khat = oracle.base_dequantize_channel(pl["kc"], pl["ks"], pl["km"])
    np.testing.assert_array_equal(khat[0, 0, :, 0], [1.0, 4.0, 3.0])


def test_channel_code_is_the_token_code_of_the_transpose():
    """A block of 32 tokens quantised per channel is, arithmetic for arithmetic,
    the per-token group-32 code of the transposed block (pinned above by hand
    and by exhaustive search); with n = 70 the blocks are 64 + 6 tokens."""
    rng = _rng(31)
    for n in (32, 70):
        x = synth.round_bf16((rng.standard_normal((2, 1, n, 64)) * 3 + 1).astype(np.float32))
        pl = oracle.cache_write(x, np.zeros((1, 64, 2), np.float32), kmode="channel")
        assert pl["ks"].shape == (2, 1, -(-n // 64), 64)
        for b in range(2):
            for blk, (t0, t1) in enumerate([(0, min(n, 64)), (64, n)][:-(-n // 64)]):
                xt = np.ascontiguousarray(x[b, 0, t0:t1].T)          # [64 channels, nt]
                if xt.shape[1] not in (32,):
                    # not a group size: check min / scale and nearest levels directly
                    mn = xt.min(axis=1) + np.float32(0)
                    sc = (xt.max(axis=1) - xt.min(axis=1)) / np.float32(3)
                    np.testing.assert_array_equal(pl["km"][b, 0, blk], mn)
                    np.testing.assert_array_equal(pl["ks"][b, 0, blk], sc)
                    c = _codes2(pl["kc"][b, 0, t0:t1], 64)           # [nt, 64]
                    for ch in range(64):
                        for t in range(t1 - t0):
                            u = float(np.float32(xt[ch, t] - mn[ch]) / sc[ch])
                            dist = [abs(u - lvl) for lvl in range(4)]
                            best = [lvl for lvl in range(4) if dist[lvl] == min(dist)]
                            want = best[0] if len(best) == 1 else [v for v in best if v % 2 == 0][0]
                            assert c[t, ch] == want
                    continue
                codes_t, sc_t, mn_t = oracle.base_quantize(xt)           # per channel row
                np.testing.assert_array_equal(pl["km"][b, 0, blk], mn_t[:, 0])
                np.testing.assert_array_equal(pl["ks"][b, 0, blk], sc_t[:, 0])
                np.testing.assert_array_equal(_codes2(pl["kc"][b, 0, t0:t1], 64).T,
                                              _codes2(codes_t, t1 - t0))


def test_channel_code_is_equivariant_to_a_shared_translation():
    """Adding the same vector mu to every key (a softmax-null component, summary
    section 2.1) leaves the per-channel codes, scales and residuals unchanged
    and shifts the minima by mu, so the HeadQ attention is unchanged; the
    per-token group code is not equivariant and its attention moves.  Values on
    a dyadic grid keep every sum exact."""
    rng = _rng(33)
    B, Hkv, T, d, r = 1, 2, 128, 32, 8
    # every channel of every 64-token block spans exactly 0.75 (scale 0.25):
    # x = m + 0.25 j + delta, with the block's first two tokens at the ends
    m = (rng.integers(-64, 64, size=(B, Hkv, 2, 1, d)) / 16).astype(np.float32)
    j = rng.integers(0, 4, size=(B, Hkv, 2, 64, d))
    delta = rng.integers(-3, 4, size=(B, Hkv, 2, 64, d)) / 64
    delta = np.where(j == 0, np.abs(delta), np.where(j == 3, -np.abs(delta), delta))
    j[..., 0, :], j[..., 1, :] = 0, 3
    delta[..., 0:2, :] = 0
    k = (m + 0.25 * j + delta).astype(np.float32).reshape(B, Hkv, T, d)
    mu = (rng.integers(-256, 256, size=d) / 8).astype(np.float32)
    v = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    q = rng.standard_normal((B, 4, d)).astype(np.float32)
    U = np.stack([synth.random_orthonormal(rng, d, r) for _ in range(Hkv)])
    outs = {}
    for mode in ("channel", "token"):
        p0 = oracle.cache_write(k, U, kmode=mode)
        p1 = oracle.cache_write(k + mu, U, kmode=mode)
        o0, _ = oracle.decode(q, p0, U, v=v, kmode=mode)
        o1, _ = oracle.decode(q, p1, U, v=v, kmode=mode)
        outs[mode] = (p0, p1, o0, o1)
    p0, p1, o0, o1 = outs["channel"]
    for name in ("kc", "ks", "zc", "zs", "y"):
        np.testing.assert_array_equal(p1[name], p0[name])
    np.testing.assert_array_equal(p1["km"], p0["km"] + mu)
    np.testing.assert_allclose(o1, o0, rtol=1e-11, atol=1e-12)
    p0, p1, o0, o1 = outs["token"]
    assert not np.array_equal(p1["kc"], p0["kc"])
    assert np.abs(o1 - o0).max() > 1e-3


def test_null_space_intervention_hurts_only_the_non_equivariant_code():
    """Summary section 4 (null-space interventions): restoring a softmax-null
    mean component raises the Fisher damage sharply for a non-equivariant code
    and leaves an equivariant one alone.  Synthetic keys of the 28q/4kv layer
    (reduced), with and without a shared mean of scale 4 added after RoPE."""
    w = configs.workload(2).with_(B=2, T=512, n_cal=256)
    L = synth.make_layer(w)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    mu = (16.0 * _rng(35).standard_normal(w.d)).astype(np.float32)
    for sigma in (0.0, 1.0):       # the base code alone, and with the HeadQ correction
        fv = {}
        for mode in ("token", "channel"):
            for tag, k in (("plain", L.keys), ("mean", L.keys + mu)):
                pl = oracle.cache_write(k, U, kmode=mode)
                _, f, _, _ = oracle.attn_kl(L.queries, pl, U, k, L.values, v=L.values,
                                            kmode=mode, sigma=sigma)
                fv[mode, tag] = float(np.mean(f))
        assert fv["token", "mean"] > 2.5 * fv["token", "plain"]
        assert abs(fv["channel", "mean"] / fv["channel", "plain"] - 1) < 0.05


def test_projection_exact_rational_sequential():
    """y_i = fl(y_i + fl(U_ci e_c)) for c = 0..d-1 in order (d=8, r=4): every
    product rounded to fp32, then every sum rounded (a multiply, then an add)."""
    rng = _rng(3)
    d, r, T = 8, 4, 16
    k = synth.round_bf16(rng.standard_normal((1, 1, T, d)).astype(np.float32) * 3)
    U = synth.random_orthonormal(rng, d, r)[None]
    planes = oracle.cache_write(k, U)
    codes, sc, mn = planes["kc"][0, 0], planes["ks"][0, 0], planes["km"][0, 0]
    c = _codes2(codes, d)
    for t in range(T):
        # residual with the dequantised base key, each fp32 op rounded
        khat = [np.float32(mn[t, 0] + np.float32(np.float32(c[t, j]) * sc[t, 0]))
                for j in range(d)]
        e = [np.float32(k[0, 0, t, j] - khat[j]) for j in range(d)]
        for i in range(r):
            y = np.float32(0.0)
            for j in range(d):
                term = _round_f32(Fraction(float(U[0, j, i])) * Fraction(float(e[j])))
                y = _round_f32(Fraction(float(y)) + Fraction(float(term)))
            assert planes["y"][0, 0, t, i].view(np.uint32) == np.float32(y).view(np.uint32)


@pytest.mark.parametrize("r", [2, 8, 16])
def test_side_code_is_nearest_level(r):
    rng = _rng(r)
    y = (rng.standard_normal((32, r)) * rng.uniform(0.01, 5, size=(32, 1))).astype(np.float32)
    # subnormal rows: max|y|/7 rounds coarsely and the clamp to +-7 acts
    tiny = np.float32(2.0 ** -149)
    y[30] = tiny * rng.integers(-10, 11, size=r).astype(np.float32)
    y[30, 0] = tiny * 10
    y[31] = tiny * rng.integers(-3, 4, size=r).astype(np.float32)
    zc, zs = oracle.side_quantize(y)
    w = _nibbles(zc, r)
    for t in range(32):
        assert zs[t] == np.float32(np.max(np.abs(y[t]))) / np.float32(7)
        if zs[t] == 0:          # max|y|/7 underflows to 0: every code is 0
            assert (w[t] == 0).all()
            continue
        for i in range(r):
            u = float(np.float32(y[t, i]) / zs[t])
            dist = {lvl: abs(u - lvl) for lvl in range(-7, 8)}
            best = min(dist.values())
            cands = [lvl for lvl, v in dist.items() if v == best]
            want = cands[0] if len(cands) == 1 else [v for v in cands if v % 2 == 0][0]
            assert w[t, i] == want


# ---------------------------------------------------------------------------
# Cache read: brute force, special cases, closed forms.
# ---------------------------------------------------------------------------

def _tiny_layer(d=8, T=16, Hkv=1, G=2, B=2, r=4, seed=0):
    rng = _rng(seed)
    k = synth.round_bf16((rng.standard_normal((B, Hkv, T, d)) * 2 + 1).astype(np.float32))
    v = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    q = rng.standard_normal((B, Hkv * G, d)).astype(np.float32)
    U = np.stack([synth.random_orthonormal(rng, d, r) for _ in range(Hkv)])
    return k, v, q, U


def test_decode_brute_force_d8_T16():
    """Direct formula: exp without the max trick, explicit loops, fp64."""
    k, v, q, U = _tiny_layer()
    B, Hkv, T, d = k.shape
    Hq, r = q.shape[1], U.shape[-1]
    G = Hq // Hkv
    planes = oracle.cache_write(k, U)
    out, lse = oracle.decode(q, planes, U, v=v)
    c = _codes2(planes["kc"], d)
    w = _nibbles(planes["zc"], r)
    sm = 1.0 / np.sqrt(d)
    for b in range(B):
        for h in range(Hq):
            kv = h // G
            s = []
            for j in range(T):
                base = 0.0
                for ch in range(d):
                    kh = np.float32(planes["km"][b, kv, j, 0]
                                    + np.float32(np.float32(c[b, kv, j, ch])
                                                 * planes["ks"][b, kv, j, 0]))
                    base += float(q[b, h, ch]) * float(kh)
                corr = 0.0
                for ch in range(d):
                    uz = 0.0
                    for i in range(r):
                        zh = np.float32(np.float32(w[b, kv, j, i]) * planes["zs"][b, kv, j])
                        uz += float(U[kv, ch, i]) * float(zh)
                    corr += float(q[b, h, ch]) * uz
                s.append(sm * (base + corr))
            ex = [np.exp(x) for x in s]
            Z = sum(ex)
            o = [sum(ex[j] / Z * float(v[b, kv, j, ch]) for j in range(T)) for ch in range(d)]
            np.testing.assert_allclose(out[b, h], o, rtol=1e-12, atol=1e-13)
            assert abs(lse[b, h] - np.log(Z)) < 1e-12


def _sdpa(q, k, v, sm, seq_lens=None):
    import torch
    import torch.nn.functional as F
    B = q.shape[0]
    outs, lses = [], []
    for b in range(B):
        Tb = k.shape[2] if seq_lens is None else int(seq_lens[b])
        qt = torch.from_numpy(q[b:b + 1].astype(np.float64))[:, :, None, :]
        kt = torch.from_numpy(k[b:b + 1, :, :Tb].astype(np.float64))
        vt = torch.from_numpy(v[b:b + 1, :, :Tb].astype(np.float64))
        o = F.scaled_dot_product_attention(qt, kt, vt, scale=sm, enable_gqa=True)
        rep = q.shape[1] // k.shape[1]
        lg = torch.einsum("bhd,bhtd->bht", qt[:, :, 0], kt.repeat_interleave(rep, 1)) * sm
        outs.append(o[0, :, 0].numpy())
        lses.append(torch.logsumexp(lg, -1)[0].numpy())
    return np.stack(outs), np.stack(lses)


def test_sigma_zero_is_plain_base_code_attention():
    """sigma = 0 drops the correction: softmax(q k^base / sqrt d) V (library SDPA)."""
    k, v, q, U = _tiny_layer(d=32, T=40, Hkv=2, G=3, B=3, r=8, seed=5)
    planes = oracle.cache_write(k, U)
    khat = oracle.base_dequantize(planes["kc"], planes["ks"], planes["km"])
    seq_lens = np.array([40, 17, 1], np.int32)
    out, lse = oracle.decode(q, planes, U, v=v, sigma=0.0, seq_lens=seq_lens)
    ref, ref_lse = _sdpa(q, khat, v, 1 / np.sqrt(32), seq_lens)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_exact_attention_matches_sdpa():
    k, v, q, _ = _tiny_layer(d=64, T=33, Hkv=2, G=2, B=2, seed=6)
    out, lse = oracle.exact_attention(q, k, v)
    ref, ref_lse = _sdpa(q, k, v, 1 / 8.0)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12)


def test_unquantised_side_code_recovers_span_component():
    """With z^ = U_h^T e (no Q_q), q^T k^base + (U_h^T q)^T z^ = q^T k - ((I - U U^T) q)^T e;
    for q in span(U_h) the HeadQ logit equals the full-precision logit."""
    w = configs.workload(0)
    L = synth.make_layer(w, T=64)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    planes = oracle.cache_write(L.keys, U)
    khat = oracle.base_dequantize(planes["kc"], planes["ks"], planes["km"])
    y = planes["y"].astype(np.float64)
    e = L.keys.astype(np.float64) - khat.astype(np.float64)
    Ud = U[0].astype(np.float64)
    # a general query and one projected into span(U_h)
    q = L.queries.astype(np.float64)[0]                  # [Hq, d]
    q_in = (q @ Ud) @ Ud.T
    sm = 1 / np.sqrt(w.d)
    for qq in (q, q_in):
        qq32 = qq.astype(np.float32)[None]
        _, _, s_hat = oracle.attend(qq32, khat, L.values, U=U, zhat=y, want_logits=True)
        _, _, s_full = oracle.attend(qq32, L.keys, L.values, sigma=0.0, want_logits=True)
        qd = qq32[0].astype(np.float64)
        P = np.eye(w.d) - Ud @ Ud.T
        # closed form of the gap, per head and token
        gap = -np.einsum("hd,td->ht", qd @ P.T, e[0, 0]) * sm
        np.testing.assert_allclose(s_hat[0] - s_full[0], gap, atol=2e-4 * np.abs(s_full).max())
    # in span: the gap is ~ fp32 rounding of y only
    _, _, s_hat = oracle.attend(q_in.astype(np.float32)[None], khat, L.values, U=U, zhat=y,
                                want_logits=True)
    _, _, s_full = oracle.attend(q_in.astype(np.float32)[None], L.keys, L.values, sigma=0.0,
                                 want_logits=True)
    assert np.abs(s_hat - s_full).max() < 1e-5 * np.abs(s_full).max()


def test_u_column_sign_flip():
    """Flipping a column of U_h negates that side code and leaves every logit unchanged."""
    k, v, q, U = _tiny_layer(d=64, T=50, Hkv=2, G=2, B=2, r=8, seed=9)
    U2 = U.copy()
    U2[:, :, [1, 4]] *= -1
    p1 = oracle.cache_write(k, U)
    p2 = oracle.cache_write(k, U2)
    w1, w2 = _nibbles(p1["zc"], 8), _nibbles(p2["zc"], 8)
    assert np.array_equal(w1[..., [1, 4]], -w2[..., [1, 4]])
    assert np.array_equal(np.delete(w1, [1, 4], -1), np.delete(w2, [1, 4], -1))
    assert np.array_equal(p1["zs"], p2["zs"])
    o1, l1 = oracle.decode(q, p1, U, v=v)
    o2, l2 = oracle.decode(q, p2, U2, v=v)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_softmax_null_translation():
    """A token-shared translation mu of all keys leaves attention unchanged."""
    k, v, q, _ = _tiny_layer(d=64, T=64, Hkv=2, G=2, B=2, seed=11)
    mu = (np.random.default_rng(1).standard_normal(64) * 3).astype(np.float64)
    k64 = k.astype(np.float64)
    o1, l1 = oracle.exact_attention(q, k64.astype(np.float32), v)
    o2, l2 = oracle.exact_attention(q, (k64 + mu).astype(np.float32), v)
    # translation changes every logit by the same constant q.mu/sqrt(d)
    shift = np.einsum("bhd,d->bh", q.astype(np.float64), mu) / 8.0
    np.testing.assert_allclose(o1, o2, rtol=1e-5, atol=1e-6)   # fp32 rounding of k + mu
    np.testing.assert_allclose(l2 - l1, shift, atol=1e-4)


def test_empty_and_single_token_sequences():
    k, v, q, U = _tiny_layer(d=32, T=8, Hkv=1, G=2, B=3, r=4, seed=2)
    planes = oracle.cache_write(k, U)
    out, lse = oracle.decode(q, planes, U, v=v, seq_lens=np.array([0, 1, 8], np.int32))
    assert (out[0] == 0).all() and np.isneginf(lse[0]).all()
    # one token: p = 1, out = v_0
    np.testing.assert_array_equal(out[1], np.repeat(v[1, :, 0], 2, axis=0).astype(np.float64))


def test_merge_of_token_shards_equals_whole():
    """Split-T: decoding disjoint token ranges separately and merging the
    partials by their log-sum-exps equals one decode over all tokens (softmax
    over a union of token sets); ranges a sequence never reaches contribute
    nothing, and a sequence of length 0 stays out = 0, lse = -inf."""
    k, v, q, U = _tiny_layer(d=32, T=100, Hkv=2, G=2, B=3, r=8, seed=21)
    planes = oracle.cache_write(k, U)
    seq_lens = np.array([100, 30, 0], np.int32)
    whole, whole_lse = oracle.decode(q, planes, U, v=v, seq_lens=seq_lens)
    bounds = [0, 17, 64, 100]
    outs, lses = [], []
    for lo, hi in zip(bounds[:-1], bounds[1:]):
        sub = {n: a[:, :, lo:hi] for n, a in planes.items()}
        loc = np.clip(seq_lens - lo, 0, hi - lo).astype(np.int32)
        o, l_ = oracle.decode(q, sub, U, v=v[:, :, lo:hi], seq_lens=loc)
        outs.append(o)
        lses.append(l_)
    assert np.isneginf(lses[2][1]).all() and all(np.isneginf(l_[2]).all() for l_ in lses)
    out, lse = oracle.merge_partials(outs, lses)
    np.testing.assert_allclose(out, whole, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse[:2], whole_lse[:2], rtol=1e-13)
    assert (out[2] == 0).all() and np.isneginf(lse[2]).all()
    # the order of the parts does not matter; one part is returned unchanged
    out_r, lse_r = oracle.merge_partials(outs[::-1], lses[::-1])
    np.testing.assert_allclose(out_r, out, rtol=1e-13, atol=1e-15)
    o1, l1 = oracle.merge_partials(outs[:1], lses[:1])
    np.testing.assert_allclose(o1, outs[0], rtol=1e-15, atol=0)
    # library check: per-range SDPA merged equals SDPA over all tokens
    khat = oracle.base_dequantize(planes["kc"], planes["ks"], planes["km"])
    ref, ref_lse = _sdpa(q, khat, v, 1 / np.sqrt(32))
    po, pl = zip(*[_sdpa(q, khat[:, :, lo:hi], v[:, :, lo:hi], 1 / np.sqrt(32))
                   for lo, hi in zip(bounds[:-1], bounds[1:])])
    mo, ml = oracle.merge_partials(np.stack(po), np.stack(pl))
    np.testing.assert_allclose(mo, ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(ml, ref_lse, rtol=1e-12)


def test_a2_scores_sum_to_the_a2_diagnostic():
    """With the decode query as the only observation query, the A^2 policy
    scores of a KV head sum to the A^2 value distortion the diagnostic reports
    for its G heads (an independent implementation in the C oracle)."""
    k, v, q, U = _tiny_layer(d=32, T=60, Hkv=2, G=3, B=2, r=8, seed=17)
    planes = oracle.cache_write(k, U, v=v, vmode="2bit")
    vh = oracle.cached_values(planes, "2bit")
    seq_lens = np.array([60, 23], np.int32)
    sc = oracle.a2_scores(q[:, None], k, v, vh, seq_lens=seq_lens)
    _, _, a2v, _ = oracle.attn_kl(q, planes, U, k, v, vmode="2bit", seq_lens=seq_lens)
    np.testing.assert_allclose(sc.sum(axis=2), a2v.reshape(2, 2, 3).sum(axis=2), rtol=1e-10)
    assert (sc[1, :, 23:] == 0).all() and (sc >= 0).all()


def test_a2_scores_uniform_attention_closed_form():
    """Zero observation queries attend uniformly: a_j = n_obs G |dv_j|^2 / T_b^2."""
    k, v, q, U = _tiny_layer(d=16, T=40, Hkv=1, G=2, B=1, r=4, seed=18)
    planes = oracle.cache_write(k, U, v=v, vmode="2bit")
    vh = oracle.cached_values(planes, "2bit")
    sc = oracle.a2_scores(np.zeros((1, 3, 2, 16), np.float32), k, v, vh)
    dv2 = ((vh.astype(np.float64) - v) ** 2).sum(-1)
    np.testing.assert_allclose(sc, 3 * 2 * dv2 / 40 ** 2, rtol=1e-12)


def test_a2_selection_minimises_the_surrogate_brute_force():
    """For every budget K the kept set leaves the smallest surrogate sum over
    the dropped tokens of all subsets of that size (exhaustive search), and
    among equally good sets it takes the lower positions."""
    import itertools
    rng = _rng(19)
    T = 9
    scores = rng.integers(0, 4, size=(2, 1, T)).astype(np.float64)  # many ties
    seq_lens = np.array([9, 6], np.int32)
    for K in range(0, T + 2):
        kept = oracle.a2_select(scores, K, seq_lens=seq_lens)
        for b in range(2):
            Tb = int(seq_lens[b])
            m = min(K, Tb)
            got = tuple(int(j) for j in kept[b, 0] if j >= 0)
            assert len(got) == m and list(got) == sorted(got)
            assert (kept[b, 0, m:] == -1).all()
            best = min((sum(scores[b, 0, j] for j in range(Tb) if j not in S), S)
                       for S in itertools.combinations(range(Tb), m))
            assert best[1] == got


def test_a2_mixed_values_limits():
    """K = 0 is plain 2-bit value attention; keeping every token is attention
    over the exact values (same HeadQ logits in both)."""
    k, v, q, U = _tiny_layer(d=32, T=50, Hkv=2, G=2, B=2, r=8, seed=20)
    planes = oracle.cache_write(k, U, v=v, vmode="2bit")
    vh = oracle.cached_values(planes, "2bit")
    none = oracle.a2_select(np.ones((2, 2, 50)), 0)
    every = oracle.a2_select(np.ones((2, 2, 50)), 50)
    o2, _ = oracle.decode(q, planes, U, vmode="2bit")
    o0, _ = oracle.decode(q, planes, U, v=oracle.a2_mixed_values(vh, v, none))
    np.testing.assert_array_equal(o0, o2)
    oe, _ = oracle.decode(q, planes, U, v=v)
    om, _ = oracle.decode(q, planes, U, v=oracle.a2_mixed_values(vh, v, every))
    np.testing.assert_array_equal(om, oe)


def test_output_inside_value_bounding_box():
    k, v, q, U = _tiny_layer(d=64, T=100, Hkv=2, G=3, B=2, r=8, seed=13)
    planes = oracle.cache_write(k, U)
    out, _ = oracle.decode(q, planes, U, v=v)
    for b in range(2):
        for h in range(6):
            vv = v[b, h // 3].astype(np.float64)
            assert (out[b, h] <= vv.max(0) + 1e-12).all()
            assert (out[b, h] >= vv.min(0) - 1e-12).all()


# ---------------------------------------------------------------------------
# Diagnostics (summary section 2): KL, Fisher variance, A^2 value distortion.
# ---------------------------------------------------------------------------

def _kl_case(d=32, T=24, seed=21, eps=1.0, vmode="dense"):
    """Planes from keys, and a full-precision key set chosen so s^ - s is known."""
    rng = _rng(seed)
    k, v, q, U = _tiny_layer(d=d, T=T, Hkv=1, G=2, B=1, r=4, seed=seed)
    planes = oracle.cache_write(k, U, v=v, vmode=vmode)
    khat = oracle.base_dequantize(planes["kc"], planes["ks"], planes["km"])
    wdir = rng.standard_normal(khat.shape).astype(np.float32)
    k_full = (khat.astype(np.float64) - eps * wdir).astype(np.float32)
    return q, planes, U, k_full, v, khat


def test_kl_and_variance_against_library():
    """sigma = 0: KL(p||p~) via scipy.stats.entropy, Var_p via numpy.cov(aweights)."""
    from scipy.stats import entropy
    from scipy.special import softmax
    q, planes, U, k_full, v, khat = _kl_case(eps=0.3)
    kl, fv, a2, do2 = oracle.attn_kl(q, planes, U, k_full, v, v=v, sigma=0.0)
    sm = 1 / np.sqrt(q.shape[-1])
    for h in range(q.shape[1]):
        s = (k_full[0, 0].astype(np.float64) @ q[0, h].astype(np.float64)) * sm
        sh = (khat[0, 0].astype(np.float64) @ q[0, h].astype(np.float64)) * sm
        p, ph = softmax(s), softmax(sh)
        assert abs(kl[0, h] - entropy(p, ph)) < 1e-12 * max(1, kl[0, h])
        var = np.cov(sh - s, aweights=p, bias=True)
        assert abs(fv[0, h] - var) < 1e-10 * max(1.0, var)
    assert (a2 == 0).all() and (do2 == 0).all()     # dense V: no value distortion


def test_kl_local_second_order_form():
    """KL(p || softmax(s + eps*delta)) / (eps^2/2 Var_p(delta)) -> 1, error O(eps)."""
    errs = []
    for eps in (1e-1, 1e-2, 1e-3):
        q, planes, U, k_full, v, _ = _kl_case(eps=eps, seed=23)
        kl, fv, _, _ = oracle.attn_kl(q, planes, U, k_full, v, v=v, sigma=0.0)
        errs.append(np.abs(kl / (0.5 * fv) - 1).max())
    assert errs[2] < 1e-2
    assert errs[1] < errs[0] * 0.3 and errs[2] < errs[1] * 0.3


def test_kl_direction_two_tokens():
    """Two tokens, s = (0, 0), s^ = (0, t): KL(p||p~) = log((1+e^t)/2) - t/2."""
    d = 8
    k = np.zeros((1, 1, 2, d), np.float32)
    k[0, 0, 0] = [0, 1, 2, 3, 0, 1, 2, 3]           # on the grid: lossless
    k[0, 0, 1] = [0, 3, 3, 0, 0, 3, 3, 0]
    U = np.zeros((1, d, 2), np.float32)
    planes = oracle.cache_write(k, U)
    q = np.zeros((1, 1, d), np.float32)
    q[0, 0, 0] = 1.0
    k_full = k.copy()
    tval = 0.7
    k_full[0, 0, 1, 0] = -tval * np.sqrt(d)         # s_1 = -t, s^_1 = 0
    tval = -float(k_full[0, 0, 1, 0]) / np.sqrt(d)  # the fp32-stored value
    kl, fv, _, _ = oracle.attn_kl(q, planes, U, k_full, k, v=k, sigma=0.0)
    # shift logits by +t: s = (t, 0) ~ (0, -t); p = (e^t, 1)/(1+e^t), p~ uniform
    p = np.array([np.exp(tval), 1.0]) / (1 + np.exp(tval))
    want = float(np.sum(p * np.log(p / 0.5)))
    assert abs(kl[0, 0] - want) < 1e-12
    assert abs(fv[0, 0] - p[0] * p[1] * tval ** 2) < 1e-12


def test_lossless_limit_and_one_hot_value_distortion():
    """Keys on the quantisation grid: e = 0, z = 0, KL = 0, Var = 0.  With a
    one-hot attention the A^2 distortion and the readout error are |dv_j*|^2."""
    rng = _rng(31)
    d, T = 64, 20
    codes = rng.integers(0, 4, size=(1, 1, T, d))
    codes[..., ::32] = 0
    codes[..., 1::32] = 3
    scale = np.float32(0.25)
    mn = np.float32(-1.5)
    k = (mn + codes.astype(np.float32) * scale).astype(np.float32)
    U = np.stack([synth.random_orthonormal(rng, d, 8)])
    v = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    planes = oracle.cache_write(k, U, v=v, vmode="2bit")
    assert (planes["zs"] == 0).all() and (planes["zc"] == 0).all()
    assert (planes["y"] == 0).all()
    q = rng.standard_normal((1, 2, d)).astype(np.float32)
    kl, fv, a2, do2 = oracle.attn_kl(q, planes, U, k, v, vmode="2bit")
    assert (kl == 0).all() and (np.abs(fv) < 1e-15).all()
    # one-hot attention: a single key hugely aligned with the query
    k1 = k.copy()
    k1[0, 0, 7] = np.float32(60.0) * np.sign(q[0, 0]).astype(np.float32)
    p1 = oracle.cache_write(k1, U, v=v, vmode="2bit")
    q1 = q[:, :1]
    _, _, a2, do2 = oracle.attn_kl(q1, p1, U, k1, v, vmode="2bit")
    vhat = oracle.base_dequantize(p1["vc"], p1["vs"], p1["vm"]).astype(np.float64)
    dv = vhat[0, 0, 7] - v[0, 0, 7].astype(np.float64)
    assert abs(a2[0, 0] - dv @ dv) < 1e-9 and abs(do2[0, 0] - dv @ dv) < 1e-9


def test_uniform_attention_value_distortion():
    """q = 0: p_j = 1/T, so A2V = (1/T^2) sum |dv_j|^2 and dout2 = |mean dv|^2."""
    rng = _rng(33)
    d, T = 32, 40
    k = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    v = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    U = np.stack([synth.random_orthonormal(rng, d, 4)])
    planes = oracle.cache_write(k, U, v=v, vmode="2bit")
    q = np.zeros((1, 1, d), np.float32)
    kl, fv, a2, do2 = oracle.attn_kl(q, planes, U, k, v, vmode="2bit")
    vhat = oracle.base_dequantize(planes["vc"], planes["vs"], planes["vm"]).astype(np.float64)
    dv = vhat[0, 0] - v[0, 0].astype(np.float64)
    assert abs(a2[0, 0] - (dv * dv).sum() / T ** 2) < 1e-12
    m = dv.mean(0)
    assert abs(do2[0, 0] - m @ m) < 1e-12
    assert kl[0, 0] == 0 and fv[0, 0] == 0


# ---------------------------------------------------------------------------
# Claims of the pages, as statistical checks on the synthetic workloads.
# ---------------------------------------------------------------------------

def _workload_kl(i, T, sigma, U=None):
    w = configs.workload(i)
    L = synth.make_layer(w, T=T, B=min(w.B, 2))
    if U is None:
        U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    planes = oracle.cache_write(L.keys, U)
    kl, fv, _, _ = oracle.attn_kl(L.queries, planes, U, L.keys, L.values, v=L.values,
                                  sigma=sigma)
    return kl, fv


@pytest.mark.parametrize("i", [0, 1, 2])
def test_wrong_sign_correction_is_worse(i):
    """Section 4: flipping the sign of the HeadQ correction fails; sigma=+1 helps."""
    T = 256
    klp = _workload_kl(i, T, +1.0)[0].mean()
    kl0 = _workload_kl(i, T, 0.0)[0].mean()
    klm = _workload_kl(i, T, -1.0)[0].mean()
    assert klp < kl0 < klm, (klp, kl0, klm)


def test_query_pca_beats_random_basis():
    """Section 4: a query-PCA basis recovers the active residual; a random basis of
    the same rank does not."""
    w = configs.workload(0)
    L = synth.make_layer(w, T=256)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    R = np.stack([synth.random_orthonormal(_rng(7), w.d, w.r)])
    kl_pca = _workload_kl(0, 256, 1.0, U)[0].mean()
    kl_rand = _workload_kl(0, 256, 1.0, R)[0].mean()
    assert kl_pca < 0.5 * kl_rand, (kl_pca, kl_rand)


def test_kl_and_variance_nonnegative():
    kl, fv = _workload_kl(1, 128, 1.0)
    assert (kl >= 0).all() and (fv >= -1e-12).all()


# ---------------------------------------------------------------------------
# Calibration: numpy eigh of the pooled second moment, checked by its
# defining properties and against the generator's known query subspace.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("i", [0, 2])
def test_calibration_basis(i):
    w = configs.workload(i)
    L = synth.make_layer(w, T=16, B=1)
    U, eig = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    G = w.G
    for kv in range(w.Hkv):
        X = L.q_cal[:, kv * G:(kv + 1) * G].reshape(-1, w.d).astype(np.float64)
        C = X.T @ X / X.shape[0]
        Uk = U[kv].astype(np.float64)
        np.testing.assert_allclose(Uk.T @ Uk, np.eye(w.r), atol=1e-6)
        np.testing.assert_allclose(C @ Uk, Uk * eig[kv].astype(np.float64),
                                   rtol=0, atol=1e-5 * eig[kv].max())
        assert (np.diff(eig[kv]) <= 0).all()
        # the r largest: nothing outside span(U) carries more energy
        P = np.eye(w.d) - Uk @ Uk.T
        assert np.linalg.eigvalsh(P @ C @ P).max() <= eig[kv].min() * (1 + 1e-5)
        # sign rule: the largest-magnitude entry of each column is positive
        idx = np.argmax(np.abs(Uk), axis=0)
        assert (Uk[idx, np.arange(w.r)] > 0).all()
        # the queries live (up to 0.1 noise) in span(A): U spans it
        A = L.meta["query_basis"][kv].astype(np.float64)
        Qa, _ = np.linalg.qr(A)
        k = min(w.r, w.r_s)
        sv = np.linalg.svd(Qa.T @ Uk, compute_uv=False)
        assert sv[:k].min() > 0.99


def _exact_centred_covariance(X):
    """Covariance of the rows of an integer matrix about their mean, divided by
    the row count, in exact rational arithmetic (the plain PCA matrix)."""
    M, d = X.shape
    mean = [Fraction(int(sum(int(X[m, c]) for m in range(M))), M) for c in range(d)]
    C = np.zeros((d, d))
    for a in range(d):
        for b in range(d):
            s = sum((int(X[m, a]) - mean[a]) * (int(X[m, b]) - mean[b]) for m in range(M))
            C[a, b] = float(s / M)
    return C


def test_calibration_centred_exact_rational():
    """center=True: the basis is the top eigenspace of the covariance about the
    pooled mean of a KV head's G query heads (exact rationals on a small integer
    case with head means far from 0 and from each other)."""
    rng = _rng(41)
    N, Hkv, G, d, r = 12, 2, 3, 8, 4
    q = rng.integers(-4, 5, size=(N, Hkv * G, d)).astype(np.float32)
    q += np.arange(Hkv * G, dtype=np.float32)[None, :, None] * 3 + 5  # shifted heads
    U, eig = oracle.calibrate(q, Hkv, r, center=True)
    for kv in range(Hkv):
        X = q[:, kv * G:(kv + 1) * G].reshape(-1, d).astype(np.int64)
        C = _exact_centred_covariance(X)
        w = np.sort(np.linalg.eigvalsh(C))[::-1][:r]
        np.testing.assert_allclose(eig[kv], w, rtol=1e-6, atol=1e-6 * w[0])
        Uk = U[kv].astype(np.float64)
        np.testing.assert_allclose(Uk.T @ Uk, np.eye(r), atol=1e-6)
        np.testing.assert_allclose(C @ Uk, Uk * eig[kv].astype(np.float64), atol=1e-5 * w[0])
        idx = np.argmax(np.abs(Uk), axis=0)
        assert (Uk[idx, np.arange(r)] > 0).all()


@pytest.mark.parametrize("i", [0, 2])
def test_calibration_centred_translation_and_library(i):
    """center=True equals numpy's biased covariance of the pooled queries, is
    unchanged by a shared translation of every calibration query, and equals
    the uncentred second moment minus the outer product of the mean."""
    w = configs.workload(i)
    L = synth.make_layer(w, T=16, B=1)
    shift = (3.0 * _rng(42).standard_normal(w.d)).astype(np.float32)
    U, eig = oracle.calibrate(L.q_cal, w.Hkv, w.r, center=True)
    U2, eig2 = oracle.calibrate(L.q_cal + shift, w.Hkv, w.r, center=True)
    G = w.G
    for kv in range(w.Hkv):
        X = L.q_cal[:, kv * G:(kv + 1) * G].reshape(-1, w.d).astype(np.float64)
        C = np.cov(X, rowvar=False, bias=True)
        m = X.mean(axis=0)
        np.testing.assert_allclose(C, X.T @ X / X.shape[0] - np.outer(m, m),
                                   atol=1e-9 * np.abs(C).max())
        top = np.sort(np.linalg.eigvalsh(C))[::-1][:w.r]
        np.testing.assert_allclose(eig[kv], top, rtol=1e-5)
        Uk = U[kv].astype(np.float64)
        np.testing.assert_allclose(C @ Uk, Uk * eig[kv].astype(np.float64),
                                   atol=1e-5 * eig[kv].max())
        # the translated queries give the same subspace and eigenvalues
        np.testing.assert_allclose(eig2[kv], eig[kv], rtol=1e-4)
        P = Uk @ Uk.T
        P2 = U2[kv].astype(np.float64) @ U2[kv].astype(np.float64).T
        assert np.linalg.norm(P - P2) < 1e-3


# ---------------------------------------------------------------------------
# The same-budget counterexample (summary, section 4): lower key-storage error,
# higher attention KL.  residual_basis and key_mse are pinned first.
# ---------------------------------------------------------------------------

def test_residual_basis_is_the_residual_eigenbasis():
    """residual_basis: orthonormal, the eigen-equation of the residuals' second
    moment (residuals rebuilt here from the base code's definition, exact fp32
    steps), the r largest eigenvalues, the sign rule."""
    w = configs.workload(2)
    L = synth.make_layer(w, T=128, B=2)
    U = oracle.residual_basis(L.keys, w.r)
    codes, sc, mn = oracle.base_quantize(L.keys)
    c = _codes2(codes, w.d)
    g = np.arange(w.d) // 32
    khat = mn[..., g] + (c.astype(np.float32) * sc[..., g]).astype(np.float32)
    e = (L.keys - khat).astype(np.float64)
    for kv in range(w.Hkv):
        X = e[:, kv].reshape(-1, w.d)
        C = X.T @ X / X.shape[0]
        Uk = U[kv].astype(np.float64)
        np.testing.assert_allclose(Uk.T @ Uk, np.eye(w.r), atol=1e-6)
        lam = np.diag(Uk.T @ C @ Uk)
        np.testing.assert_allclose(C @ Uk, Uk * lam, atol=1e-5 * lam.max())
        P = np.eye(w.d) - Uk @ Uk.T
        assert np.linalg.eigvalsh(P @ C @ P).max() <= lam.min() * (1 + 1e-5)
        assert (np.diff(lam) <= 1e-9 * lam.max()).all()
        idx = np.argmax(np.abs(Uk), axis=0)
        assert (Uk[idx, np.arange(w.r)] > 0).all()


def test_key_mse_pythagoras_and_lossless_limit():
    """key_mse: with orthonormal U the key error k - k^base - U z^ splits into
    (I - U U^T) e and U (y - z^), so its squared norm is |e|^2 - |y|^2 + |y - z^|^2
    (y = U^T e, the unquantised projection); and keys on the code grid give 0."""
    rng = _rng(51)
    w = configs.workload(1)
    L = synth.make_layer(w, T=64, B=1)
    U = synth.random_orthonormal(rng, w.d, w.r)[None].repeat(w.Hkv, 0)
    pl = oracle.cache_write(L.keys, U)
    codes, sc, mn = pl["kc"], pl["ks"], pl["km"]
    c = _codes2(codes, w.d)
    g = np.arange(w.d) // 32
    khat = mn[..., g] + (c.astype(np.float32) * sc[..., g]).astype(np.float32)
    e = (L.keys - khat).astype(np.float64)
    y = pl["y"].astype(np.float64)
    zh = _nibbles(pl["zc"], w.r) * pl["zs"][..., None].astype(np.float64)
    want = np.mean(np.sum(e * e, -1) - np.sum(y * y, -1) + np.sum((y - zh) ** 2, -1))
    assert abs(oracle.key_mse(L.keys, pl, U) - want) <= 1e-9 * max(1.0, want)
    # on the grid: every group spans levels 0..3 exactly
    kg = np.tile(np.array([0.0, 0.5, 1.0, 1.5], np.float32), (1, w.Hkv, 8, w.d // 4))
    assert oracle.key_mse(kg, oracle.cache_write(kg, U), U) == 0.0


@pytest.mark.parametrize("i", [0, 1, 2, 3, 4])
def test_same_budget_counterexample(i):
    """Summary, section 4: at the same bit budget, the side code fitted to the key
    residuals (best for key storage) has the lower key-storage error but a far
    higher attention KL than HeadQ's query-PCA side code."""
    w = configs.workload(i)
    L = synth.make_layer(w, T=256, B=min(w.B, 2))
    Uq, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    Ue = oracle.residual_basis(L.keys, w.r)
    res = {}
    for tag, U in (("query", Uq), ("residual", Ue)):
        pl = oracle.cache_write(L.keys, U)
        kl, _, _, _ = oracle.attn_kl(L.queries, pl, U, L.keys, L.values, v=L.values)
        res[tag] = (oracle.key_mse(L.keys, pl, U), float(np.mean(kl)),
                    sum(pl[k].nbytes for k in ("kc", "ks", "km", "zc", "zs")))
    assert res["residual"][2] == res["query"][2]          # the same bits
    assert res["residual"][0] < 0.8 * res["query"][0]     # lower storage error
    assert res["residual"][1] > 5.0 * res["query"][1]     # higher attention KL
