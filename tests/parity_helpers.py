"""Shared plumbing of the GPU parity tests.

Both sides get the same seeded inputs from ``synth``; the oracle side runs on
numpy arrays, the CUDA side through the C ABI (``headq``).  Nothing flows
from the CUDA side into the oracle.
"""

import numpy as np

import oracle
from bit_decode_attention_sm_b200 import configs, synth

DECODE_RTOL = 2e-3      # max relative error per output row (of the row maximum)
DIAG_RTOL = 1e-2        # diagnostics: relative, or DIAG_ATOL absolute if looser
DIAG_ATOL = 1e-6


def torch_dtype(w):
    import torch
    return torch.bfloat16 if w.kv_dtype == "bf16" else torch.float32


def roundup(x, m):
    return (x + m - 1) // m * m


def layer(i, **kw):
    w = configs.workload(i)
    return w, synth.make_layer(w, **kw)


def oracle_side(w, L, U, seq_lens=None, sigma=1.0, kmode="token"):
    planes = oracle.cache_write(L.keys, U, v=L.values, vmode=w.vmode, kmode=kmode)
    out, lse = oracle.decode(L.queries, planes, U, v=L.values, vmode=w.vmode,
                             sigma=sigma, seq_lens=seq_lens, kmode=kmode)
    return planes, out, lse


def gpu_cache(w, L, U, T_cap=None, t0=0, kmode="token"):
    import torch
    from bit_decode_attention_sm_b200 import headq
    dt = torch_dtype(w)
    B, Hkv, T, d = L.keys.shape
    T_cap = roundup(t0 + T, 64 if kmode == "channel" else 16) if T_cap is None else T_cap
    cache = headq.HeadQCache(B, Hkv, T_cap, d, w.r, vmode=w.vmode, v_dtype=dt, kmode=kmode)
    k = torch.from_numpy(L.keys).to("cuda").to(dt)
    v = torch.from_numpy(L.values).to("cuda").to(dt)
    Ut = torch.from_numpy(np.ascontiguousarray(U)).to("cuda")
    headq.headq_cache_write(cache, k, v, Ut, t0=t0)
    return cache, Ut


def gpu_query(w, L):
    import torch
    return torch.from_numpy(L.queries).to("cuda").to(torch_dtype(w))


def planes_to_numpy(cache, t0, T, b=None, kv=None):
    """Cache planes for tokens [t0, t0+T) as numpy (one (b, kv) row if given)."""
    sl = slice(t0, t0 + T)
    bs = slice(None) if b is None else slice(b, b + 1)
    ks = slice(None) if kv is None else slice(kv, kv + 1)
    out = {}
    for name, t in cache.planes().items():
        a = t[bs, ks, sl].cpu()
        if a.dtype == __import__("torch").bfloat16:
            a = a.view(__import__("torch").int16).numpy().view(np.uint16)
        else:
            a = a.numpy()
        out[name] = a
    return out


def assert_planes_equal(gpu, ref, r, vmode, kv_dtype, values=None):
    """Bit-exact comparison of every plane (fp32 planes compared as bit patterns)."""
    np.testing.assert_array_equal(gpu["kc"], ref["kc"])
    np.testing.assert_array_equal(gpu["ks"].view(np.uint32), ref["ks"].view(np.uint32))
    np.testing.assert_array_equal(gpu["km"].view(np.uint32), ref["km"].view(np.uint32))
    if r > 0:
        np.testing.assert_array_equal(gpu["zc"][..., :r // 2], ref["zc"])
        np.testing.assert_array_equal(gpu["zs"].view(np.uint32), ref["zs"].view(np.uint32))
    if vmode == "2bit":
        np.testing.assert_array_equal(gpu["vc"], ref["vc"])
        np.testing.assert_array_equal(gpu["vs"].view(np.uint32), ref["vs"].view(np.uint32))
        np.testing.assert_array_equal(gpu["vm"].view(np.uint32), ref["vm"].view(np.uint32))
    elif values is not None:
        if kv_dtype == "bf16":
            np.testing.assert_array_equal(gpu["v"], synth.f32_to_bf16_bits(values))
        else:
            np.testing.assert_array_equal(gpu["v"].view(np.uint32),
                                          np.ascontiguousarray(values).view(np.uint32))


def row_rel_err(out, ref):
    """max over rows of max|out - ref| / max|ref| (rows = last axis)."""
    num = np.abs(np.asarray(out, np.float64) - ref).max(-1)
    den = np.abs(ref).max(-1)
    den = np.where(den > 0, den, 1.0)
    return float((num / den).max()) if num.size else 0.0


def assert_diag_close(got, ref, name):
    got = np.asarray(got, np.float64)
    tol = np.maximum(DIAG_RTOL * np.abs(ref), DIAG_ATOL)
    bad = np.abs(got - ref) > tol
    assert not bad.any(), "%s: %d/%d outside tolerance, worst %s vs %s" % (
        name, bad.sum(), bad.size, got[bad][:4], ref[bad][:4])
