"""HeadQ CPU oracle -- TEST INFRASTRUCTURE ONLY.

A plain, slow and obviously correct CPU restatement of HeadQ ("HeadQ:
Model-Visible Distortion and Score-Space Correction for KV-Cache Quantization";
the gist.science technical summary, sections 2 and 3).  Only the test-suite,
the smoke check and the benchmark's CPU-baseline leg may import it.  It shares
no code with the CUDA library and never imports it.

The codec and the attention are in ``headq_oracle.c`` (exact fp32 codec,
fp64 attention), compiled by :func:`build`; the query-PCA calibration is
``numpy.linalg.eigh`` of the pooled second-moment matrix in fp64.

All array arguments are numpy arrays; keys/values/queries are fp32 (bf16
workloads pass their bf16 values converted exactly to fp32).
"""

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "headq_oracle.c")
_LIB = os.path.join(_HERE, "libheadq_oracle.so")

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
          "-fno-unsafe-math-optimizations", "-fopenmp", "-fPIC", "-shared",
          "-fvisibility=hidden", "-Wall", "-Wno-unused-function"]


def build(force=False):
    """Compile the C oracle with gcc (no implicit FMA contraction, no fast-math)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + ".tmp.%d" % os.getpid()
    subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        L = ctypes.c_int64
        D = ctypes.c_double
        lib.hqo_set_threads.argtypes = [I]
        lib.hqo_set_threads.restype = I
        lib.hqo_base_quantize.argtypes = [P, L, I, P, P, P]
        lib.hqo_base_dequantize.argtypes = [P, P, P, L, I, P]
        lib.hqo_cache_write.argtypes = [P, I, I, I, I, I, P, P, P, P, P, P, P, I, I]
        lib.hqo_base_dequantize_channel.argtypes = [P, P, P, L, I, I, I, P]
        lib.hqo_side_dequantize.argtypes = [P, P, L, I, P]
        lib.hqo_side_quantize.argtypes = [P, L, I, P, P]
        lib.hqo_attend.argtypes = [P, I, I, I, I, I, I, P, P, P, P, P, D, D, P, P, P]
        lib.hqo_decode.argtypes = [P, I, I, I, I, I, I, P, P, P, P, P, P, P, I, P,
                                   P, P, P, D, D, P, P, I, I]
        lib.hqo_attn_kl.argtypes = [P, I, I, I, I, I, I, P, P, P, P, P, P, P, I, P,
                                    P, P, P, P, P, D, D, P, P, P, P, I, I]
        for f in ("hqo_base_quantize", "hqo_base_dequantize", "hqo_cache_write",
                  "hqo_base_dequantize_channel",
                  "hqo_side_dequantize", "hqo_side_quantize", "hqo_attend", "hqo_decode", "hqo_attn_kl"):
            getattr(lib, f).restype = I
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _check(rc, what):
    if rc != 0:
        raise ValueError("oracle %s failed with code %d" % (what, rc))


def set_threads(n):
    """Number of OpenMP threads the oracle uses (returns the effective count)."""
    return _load().hqo_set_threads(int(n))


KMODES = {"token": 0, "channel": 1}
KBLOCK = 64  # tokens per block of the per-channel base code


def group_size(d):
    return d if d < 32 else 32


# --------------------------------------------------------------------------
# Step 1: calibration (gist.science summary, section 3, step 1): a rank-r
# basis U_h per KV head from the post-RoPE calibration queries.  The basis is
# the top-r eigenvectors of the pooled uncentred second moment (1/M) Q^T Q of
# the G query heads that read KV head h, eigenvalues descending; each column is
# signed so that its entry of largest magnitude is positive (lowest index on a
# tie).  center=True subtracts the pooled mean first (plain-PCA reading).
# --------------------------------------------------------------------------
def calibrate(q_cal, Hkv, r, center=False):
    q_cal = np.asarray(q_cal, dtype=np.float64)
    N, Hq, d = q_cal.shape
    G = Hq // Hkv
    U = np.zeros((Hkv, d, r), dtype=np.float32)
    eig = np.zeros((Hkv, r), dtype=np.float32)
    for kv in range(Hkv):
        X = q_cal[:, kv * G:(kv + 1) * G, :].reshape(N * G, d)
        if center:
            X = X - X.mean(axis=0, keepdims=True)
        C = (X.T @ X) / X.shape[0]
        w, V = np.linalg.eigh(C)
        order = np.argsort(-w, kind="stable")[:r]
        Vr = V[:, order]
        for i in range(r):
            j = int(np.argmax(np.abs(Vr[:, i])))
            if Vr[j, i] < 0:
                Vr[:, i] = -Vr[:, i]
        U[kv] = Vr.astype(np.float32)
        eig[kv] = w[order].astype(np.float32)
    return U, eig


# --------------------------------------------------------------------------
# The same-budget counterexample (gist.science summary, section 4: a code with
# lower key-storage error can still do worse on the attention; section 2: the
# distortion that matters is the model-visible one, not the storage one).  The
# side code's bit budget is fixed by r and the 4-bit levels whatever basis it
# uses, so two bases give two codes of exactly the same size: HeadQ's
# query-PCA basis, and the basis that is best for key storage -- the top-r
# eigenvectors of the residuals' own second moment (1/M) E^T E, residuals
# e = k - k^base of the base code, per KV head, with the sign rule of
# calibrate().
# --------------------------------------------------------------------------
def residual_basis(k, r):
    """[Hkv, d, r] fp32: per KV head, the top-r eigenvectors of the second moment
    of the base-code residuals of keys k [B, Hkv, n, d] (all sequences pooled)."""
    k = _f32(k)
    B, Hkv, n, d = k.shape
    codes, sc, mn = base_quantize(k)
    e = k.astype(np.float64) - base_dequantize(codes, sc, mn).astype(np.float64)
    U = np.zeros((Hkv, d, r), dtype=np.float32)
    for kv in range(Hkv):
        X = e[:, kv].reshape(B * n, d)
        w, V = np.linalg.eigh((X.T @ X) / X.shape[0])
        order = np.argsort(-w, kind="stable")[:r]
        Vr = V[:, order]
        for i in range(r):
            j = int(np.argmax(np.abs(Vr[:, i])))
            if Vr[j, i] < 0:
                Vr[:, i] = -Vr[:, i]
        U[kv] = Vr.astype(np.float32)
    return U


def key_mse(k, planes, U, kmode="token"):
    """Key-storage error of a cache: the mean over tokens of the squared norm of
    k - (k^base + U_h z^), the key the corrected logit q^T k^base + q^T U_h z^
    reads.  fp64."""
    k = np.asarray(k, np.float64)
    if kmode == "token":
        kb = base_dequantize(planes["kc"], planes["ks"], planes["km"])
    else:
        kb = base_dequantize_channel(planes["kc"], planes["ks"], planes["km"])
    kh = kb.astype(np.float64)
    if U.shape[-1] > 0:
        z = side_dequantize(planes["zc"], planes["zs"]).astype(np.float64)
        kh = kh + np.einsum("hdr,bhtr->bhtd", np.asarray(U, np.float64), z)
    return float(np.mean(np.sum((k - kh) ** 2, axis=-1)))


# --------------------------------------------------------------------------
# Step 2: cache write.
# --------------------------------------------------------------------------
def base_quantize(x):
    """B_b on the last axis: returns (codes uint8 [..., d/4], scale, min [..., ng])."""
    x = _f32(x)
    d = x.shape[-1]
    lead = x.shape[:-1]
    rows = int(np.prod(lead)) if lead else 1
    ng = d // group_size(d)
    codes = np.zeros(lead + (d // 4,), np.uint8)
    sc = np.zeros(lead + (ng,), np.float32)
    mn = np.zeros(lead + (ng,), np.float32)
    _check(_load().hqo_base_quantize(_p(x), rows, d, _p(codes), _p(sc), _p(mn)),
           "base_quantize")
    return codes, sc, mn


def base_dequantize_channel(codes, sc, mn, block=KBLOCK):
    """Per-channel base code: codes [S..., T, d/4], sc/mn [S..., ceil(T/block), d]
    -> k^ [S..., T, d] fp32, k^ = min_c + code * scale_c of the token's block."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    lead, T, d = codes.shape[:-2], codes.shape[-2], codes.shape[-1] * 4
    seqs = int(np.prod(lead)) if lead else 1
    out = np.zeros(lead + (T, d), np.float32)
    _check(_load().hqo_base_dequantize_channel(_p(codes), _p(_f32(sc)), _p(_f32(mn)), seqs, T,
                                               d, block, _p(out)), "base_dequantize_channel")
    return out


def base_dequantize(codes, sc, mn):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    d = codes.shape[-1] * 4
    lead = codes.shape[:-1]
    rows = int(np.prod(lead)) if lead else 1
    out = np.zeros(lead + (d,), np.float32)
    _check(_load().hqo_base_dequantize(_p(codes), _p(_f32(sc)), _p(_f32(mn)), rows,
                                       d, _p(out)), "base_dequantize")
    return out


def cache_write(k, U, v=None, vmode="dense", kmode="token"):
    """Encode keys k [B, Hkv, n, d] (and 2-bit values when vmode == '2bit').

    kmode 'token': the per-token group-32 base code (ks, km [B, Hkv, n, ng]);
    kmode 'channel': the per-channel base code over blocks of KBLOCK tokens
    counted from the first token written (ks, km [B, Hkv, ceil(n/KBLOCK), d]).
    Returns a dict of planes kc, ks, km, zc, zs (and vc, vs, vm) plus y, the
    projection U_h^T e before the side quantiser.
    """
    k = _f32(k)
    U = _f32(U)
    B, Hkv, n, d = k.shape
    r = U.shape[-1]
    ng = d // group_size(d)
    sshape = (B, Hkv, n, ng) if kmode == "token" else (B, Hkv, -(-n // KBLOCK), d)
    out = dict(
        kc=np.zeros((B, Hkv, n, d // 4), np.uint8),
        ks=np.zeros(sshape, np.float32),
        km=np.zeros(sshape, np.float32),
        zc=np.zeros((B, Hkv, n, r // 2), np.uint8),
        zs=np.zeros((B, Hkv, n), np.float32),
        y=np.zeros((B, Hkv, n, r), np.float32),
    )
    _check(_load().hqo_cache_write(_p(k), B, Hkv, n, d, r, _p(U), _p(out["kc"]),
                                   _p(out["ks"]), _p(out["km"]), _p(out["zc"]),
                                   _p(out["zs"]), _p(out["y"]), KMODES[kmode], KBLOCK),
           "cache_write")
    if vmode == "2bit":
        out["vc"], out["vs"], out["vm"] = base_quantize(v)
    return out


def side_quantize(y):
    """Q_q on the last axis of y: returns (zc uint8 [..., r/2], zs [...])."""
    y = _f32(y)
    r = y.shape[-1]
    lead = y.shape[:-1]
    rows = int(np.prod(lead)) if lead else 1
    zc = np.zeros(lead + (r // 2,), np.uint8)
    zs = np.zeros(lead, np.float32)
    _check(_load().hqo_side_quantize(_p(y), rows, r, _p(zc), _p(zs)), "side_quantize")
    return zc, zs


def side_dequantize(zc, zs):
    zc = np.ascontiguousarray(zc, dtype=np.uint8)
    r = zc.shape[-1] * 2
    lead = zc.shape[:-1]
    rows = int(np.prod(lead)) if lead else 1
    out = np.zeros(lead + (r,), np.float32)
    _check(_load().hqo_side_dequantize(_p(zc), _p(_f32(zs)), rows, r, _p(out)),
           "side_dequantize")
    return out


# --------------------------------------------------------------------------
# Step 3: cache read (decode attention).
# --------------------------------------------------------------------------
def attend(q, khat, v, U=None, zhat=None, sm_scale=None, sigma=1.0, seq_lens=None,
           want_logits=False):
    """fp64 attention with the additive logit correction.

    q [B, Hq, d]; khat, v [B, Hkv, T, d]; zhat [B, Hkv, T, r] or None.
    Returns (out [B,Hq,d], lse [B,Hq]) or also logits [B,Hq,T].
    """
    q = _f32(q)
    khat = _f32(khat)
    v = _f32(v)
    B, Hq, d = q.shape
    _, Hkv, T, _ = khat.shape
    if zhat is not None:
        zhat = np.ascontiguousarray(zhat, dtype=np.float64)
        U = _f32(U)
        r = U.shape[-1]
    else:
        r = 0
        U = np.zeros((Hkv, d, 0), np.float32)
    sm = 1.0 / np.sqrt(d) if sm_scale is None else float(sm_scale)
    sl = None if seq_lens is None else np.ascontiguousarray(seq_lens, np.int32)
    out = np.zeros((B, Hq, d), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    lg = np.zeros((B, Hq, T), np.float64) if want_logits else None
    _check(_load().hqo_attend(_p(q), B, Hq, Hkv, T, d, r, _p(sl), _p(khat), _p(zhat),
                              _p(U), _p(v), sm, float(sigma), _p(out), _p(lse),
                              _p(lg)), "attend")
    return (out, lse, lg) if want_logits else (out, lse)


def _vplanes(planes, vmode, v):
    if vmode == "2bit":
        return 1, None, planes["vc"], _f32(planes["vs"]), _f32(planes["vm"])
    return 0, _f32(v), None, None, None


def decode(q, planes, U, v=None, vmode="dense", sm_scale=None, sigma=1.0,
           seq_lens=None, kmode="token"):
    """Cache read from stored planes ([B, Hkv, T, ...]); returns (out, lse) fp64."""
    q = _f32(q)
    U = _f32(U)
    B, Hq, d = q.shape
    _, Hkv, T, _ = planes["kc"].shape
    r = U.shape[-1]
    sm = 1.0 / np.sqrt(d) if sm_scale is None else float(sm_scale)
    vm_, vd, vc, vs, vmn = _vplanes(planes, vmode, v)
    sl = None if seq_lens is None else np.ascontiguousarray(seq_lens, np.int32)
    out = np.zeros((B, Hq, d), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    c = lambda a, t: np.ascontiguousarray(a, dtype=t)
    _check(_load().hqo_decode(
        _p(q), B, Hq, Hkv, T, d, r, _p(sl), _p(c(planes["kc"], np.uint8)),
        _p(_f32(planes["ks"])), _p(_f32(planes["km"])), _p(c(planes["zc"], np.uint8)),
        _p(_f32(planes["zs"])), _p(U), vm_, _p(vd), _p(vc), _p(vs), _p(vmn), sm,
        float(sigma), _p(out), _p(lse), KMODES[kmode], KBLOCK), "decode")
    return out, lse


def merge_partials(outs, lses):
    """Attention over the union of S disjoint token sets from the S partial
    results: o_s is the softmax-weighted readout over set s and lse_s the
    log-sum-exp of its logits, so the softmax over the union weighs part s by
    exp(lse_s) (written relative to the largest lse).  A part with no tokens has
    lse_s = -inf and weight 0; a row no part covers gets out = 0, lse = -inf.
    outs [S, ..., d], lses [S, ...]; returns (out, lse) fp64."""
    outs = np.asarray(outs, np.float64)
    lses = np.asarray(lses, np.float64)
    M = lses.max(axis=0)
    covered = np.isfinite(M)
    M0 = np.where(covered, M, 0.0)
    w = np.where(np.isfinite(lses), np.exp(lses - M0), 0.0)
    L = w.sum(axis=0)
    L1 = np.where(L > 0, L, 1.0)
    out = (w[..., None] * outs).sum(axis=0) / L1[..., None]
    out = np.where(covered[..., None], out, 0.0)
    lse = np.where(covered, M0 + np.log(L1), -np.inf)
    return out, lse


# --------------------------------------------------------------------------
# A^2 value policy (abstract; summary sections 2 and 5).  The pages name the
# policy without defining it; the reading restated here: a budget of K tokens
# per (b, kv) keeps exact values, the rest keep the 2-bit code, and the kept
# set minimises the A^2 surrogate sum_j p_j^2 |v^_j - v_j|^2 summed over the
# observation queries and the heads of the KV head.
# --------------------------------------------------------------------------
def cached_values(planes, vmode, v=None):
    """v^ [B, Hkv, T, d] fp32: the 2-bit dequantised values, or the dense cache."""
    if vmode == "2bit":
        return base_dequantize(planes["vc"], planes["vs"], planes["vm"])
    return _f32(v)


def a2_scores(q_obs, k_full, v_full, v_hat, sm_scale=None, seq_lens=None):
    """a_j = |v^_j - v_j|^2 * sum_{o, h in group(kv)} p_{o,h,j}^2, fp64 [B, Hkv, T],
    with p_{o,h,.} = softmax_j(sm_scale * q_obs[b, o, h] . k_j) over j < T_b (exact
    keys), and 0 for j >= T_b.  q_obs [B, n_obs, Hq, d]; k_full, v_full, v_hat
    [B, Hkv, T, d]."""
    q = np.asarray(q_obs, np.float64)
    k = np.asarray(k_full, np.float64)
    v = np.asarray(v_full, np.float64)
    vh = np.asarray(v_hat, np.float64)
    B, n_obs, Hq, d = q.shape
    Hkv, T = k.shape[1], k.shape[2]
    G = Hq // Hkv
    sm = 1.0 / np.sqrt(d) if sm_scale is None else float(sm_scale)
    out = np.zeros((B, Hkv, T), np.float64)
    for b in range(B):
        Tb = T if seq_lens is None else int(min(max(seq_lens[b], 0), T))
        if Tb == 0:
            continue
        for kv in range(Hkv):
            qs = q[b, :, kv * G:(kv + 1) * G].reshape(-1, d)          # [n_obs*G, d]
            s = sm * (qs @ k[b, kv, :Tb].T)                             # [n_obs*G, Tb]
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            dv2 = ((vh[b, kv, :Tb] - v[b, kv, :Tb]) ** 2).sum(axis=1)
            out[b, kv, :Tb] = (p * p).sum(axis=0) * dv2
    return out


def a2_select(scores, K, seq_lens=None):
    """Kept positions int32 [B, Hkv, K]: the min(K, T_b) largest scores among
    j < T_b (equal scores: lower position first), ascending, padded with -1."""
    scores = np.asarray(scores)
    B, Hkv, T = scores.shape
    out = np.full((B, Hkv, K), -1, np.int32)
    for b in range(B):
        Tb = T if seq_lens is None else int(min(max(seq_lens[b], 0), T))
        for kv in range(Hkv):
            order = sorted(range(Tb), key=lambda j: (-scores[b, kv, j], j))
            kept = sorted(order[:min(K, Tb)])
            out[b, kv, :len(kept)] = kept
    return out


def a2_mixed_values(v_hat, v_full, keep_idx):
    """The policy's values: v_j for every kept j, v^_j for the rest."""
    mixed = np.array(v_hat, np.float32, copy=True)
    B, Hkv, K = keep_idx.shape
    for b in range(B):
        for kv in range(Hkv):
            for j in keep_idx[b, kv]:
                if j >= 0:
                    mixed[b, kv, j] = v_full[b, kv, j]
    return mixed


# --------------------------------------------------------------------------
# Step 4: diagnostics (section 2 of the summary).
# --------------------------------------------------------------------------
def attn_kl(q, planes, U, k_full, v_full, v=None, vmode="dense", sm_scale=None,
            sigma=1.0, seq_lens=None, kmode="token"):
    """Returns (kl, fisher_var, a2_vdist, dout2), each fp64 [B, Hq]."""
    q = _f32(q)
    U = _f32(U)
    B, Hq, d = q.shape
    _, Hkv, T, _ = planes["kc"].shape
    r = U.shape[-1]
    sm = 1.0 / np.sqrt(d) if sm_scale is None else float(sm_scale)
    vm_, vd, vc, vs, vmn = _vplanes(planes, vmode, v)
    sl = None if seq_lens is None else np.ascontiguousarray(seq_lens, np.int32)
    res = [np.zeros((B, Hq), np.float64) for _ in range(4)]
    c = lambda a, t: np.ascontiguousarray(a, dtype=t)
    _check(_load().hqo_attn_kl(
        _p(q), B, Hq, Hkv, T, d, r, _p(sl), _p(c(planes["kc"], np.uint8)),
        _p(_f32(planes["ks"])), _p(_f32(planes["km"])), _p(c(planes["zc"], np.uint8)),
        _p(_f32(planes["zs"])), _p(U), vm_, _p(vd), _p(vc), _p(vs), _p(vmn),
        _p(_f32(k_full)), _p(_f32(v_full)), sm, float(sigma), *[_p(a) for a in res],
        KMODES[kmode], KBLOCK), "attn_kl")
    return tuple(res)


def exact_attention(q, k, v, sm_scale=None, seq_lens=None):
    """Full-precision attention (fp64) with no quantisation at all."""
    return attend(q, k, v, sm_scale=sm_scale, sigma=0.0, seq_lens=seq_lens)
