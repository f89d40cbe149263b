"""Seeded synthetic inputs for HeadQ decode layers.

This module only draws random numbers and applies the workload's own
preprocessing (rotary position embedding, bf16 rounding).  It contains none of
HeadQ's arithmetic, so the CUDA path and the CPU oracle can both be fed from
it without sharing any of the method.

Recipe (one per workload, all numpy PCG64 streams split off one SeedSequence):
  keys    x_c ~ N(mu_c, sigma_c^2), mu_c ~ N(0, 1) (the token-shared
          translation), sigma_c ~ LogNormal(0, 0.5), 4 outlier channels per
          KV head multiplied by 10, optional random-walk drift of mu along the
          position axis, then interleaved-pair RoPE with theta_i =
          10000^(-2i/d) at position t.  mu/sigma/outliers are drawn per KV
          head and shared by the batch.
  values  N(0, 1).
  queries q = A g + 0.1 eps, A ~ N(0,1)^(d x r_s) per KV head (shared by the
          G query heads on it), g ~ N(0, I), eps ~ N(0, I).  Queries are
          taken to be post-RoPE vectors already.
bf16 values are rounded to nearest-even from fp32.
"""

import numpy as np

# a name appended here leaves every earlier stream unchanged (children of a
# SeedSequence depend only on their own index)
_STREAMS = ("key_stats", "keys", "values", "query_basis", "queries", "cal", "observe")


def _streams(seed):
    ss = np.random.SeedSequence(seed)
    return {name: np.random.Generator(np.random.PCG64(s))
            for name, s in zip(_STREAMS, ss.spawn(len(_STREAMS)))}


def f32_to_bf16_bits(x):
    """Round fp32 to bf16 (nearest-even), returned as uint16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b):
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def round_bf16(x):
    """fp32 array rounded to the nearest bf16 value (still stored as fp32)."""
    return bf16_bits_to_f32(f32_to_bf16_bits(x))


def rope_inplace(x, t0=0):
    """Interleaved-pair rotary embedding on the last axis, position along axis -2."""
    T, d = x.shape[-2], x.shape[-1]
    i = np.arange(d // 2, dtype=np.float64)
    theta = 10000.0 ** (-2.0 * i / d)
    ang = (np.arange(t0, t0 + T, dtype=np.float64)[:, None] * theta[None, :])
    c = np.cos(ang).astype(np.float32)
    s = np.sin(ang).astype(np.float32)
    a = x[..., 0::2].copy()
    b = x[..., 1::2].copy()
    x[..., 0::2] = a * c - b * s
    x[..., 1::2] = a * s + b * c
    return x


class LayerInputs:
    """All inputs of one synthetic decode layer, as fp32 numpy arrays.

    keys/values are [B, Hkv, T, d]; queries [B, Hq, d]; q_cal [n_cal, Hq, d].
    When the workload is bf16 every array already holds bf16-representable
    values, so converting to bf16 loses nothing.
    """

    def __init__(self, keys, values, queries, q_cal, meta):
        self.keys = keys
        self.values = values
        self.queries = queries
        self.q_cal = q_cal
        self.meta = meta


def make_keys(rng_stats, rng, B, Hkv, T, d, drift=0.0, n_outliers=4,
              outlier_mult=10.0, t0=0):
    mu = rng_stats.standard_normal((Hkv, d), dtype=np.float32)
    sigma = np.exp(0.5 * rng_stats.standard_normal((Hkv, d))).astype(np.float32)
    mult = np.ones((Hkv, d), dtype=np.float32)
    for h in range(Hkv):
        ch = rng_stats.choice(d, size=min(n_outliers, d), replace=False)
        mult[h, ch] = outlier_mult
    x = np.empty((B, Hkv, T, d), dtype=np.float32)
    for b in range(B):
        for h in range(Hkv):
            xs = rng.standard_normal((T, d), dtype=np.float32)
            xs *= sigma[h]
            if drift > 0.0:
                walk = rng.standard_normal((T, d), dtype=np.float32)
                walk *= np.float32(drift)
                np.cumsum(walk, axis=0, out=walk)
                xs += walk
            xs += mu[h]
            xs *= mult[h]
            x[b, h] = xs
    rope_inplace(x, t0)
    return x


def make_query_basis(rng, Hkv, d, r_s):
    return rng.standard_normal((Hkv, d, r_s), dtype=np.float32)


def make_queries(rng, A, n, Hq, noise=0.1):
    """n x Hq queries; head h uses the basis of KV head h // G."""
    Hkv, d, r_s = A.shape
    G = Hq // Hkv
    g = rng.standard_normal((n, Hq, r_s), dtype=np.float32)
    eps = rng.standard_normal((n, Hq, d), dtype=np.float32)
    q = np.empty((n, Hq, d), dtype=np.float32)
    for h in range(Hq):
        q[:, h, :] = g[:, h, :] @ A[h // G].T + np.float32(noise) * eps[:, h, :]
    return q


def make_layer(w, T=None, B=None, seed=None, n_cal=None):
    """Synthetic inputs for workload ``w`` (a configs.Workload).

    T, B, seed and n_cal override the workload's values (used for reduced-size
    test cases that keep the workload's distribution).
    """
    T = w.T if T is None else T
    B = w.B if B is None else B
    seed = w.seed if seed is None else seed
    n_cal = w.n_cal if n_cal is None else n_cal
    st = _streams(seed)
    keys = make_keys(st["key_stats"], st["keys"], B, w.Hkv, T, w.d, drift=w.drift)
    values = st["values"].standard_normal((B, w.Hkv, T, w.d), dtype=np.float32)
    A = make_query_basis(st["query_basis"], w.Hkv, w.d, w.r_s)
    queries = make_queries(st["queries"], A, B, w.Hq)
    q_cal = make_queries(st["cal"], A, n_cal, w.Hq)
    if w.kv_dtype == "bf16":
        keys = round_bf16(keys)
        values = round_bf16(values)
        queries = round_bf16(queries)
        q_cal = round_bf16(q_cal)
    return LayerInputs(keys, values, queries, q_cal,
                       dict(workload=w.name, B=B, T=T, seed=seed, n_cal=n_cal,
                            query_basis=A))


def make_observation_queries(w, L, n_obs, seed=None):
    """[B, n_obs, Hq, d] observation queries of each sequence (the queries an
    A^2 value policy measures attention with), drawn like the decode queries
    from the layer's query basis; bf16-representable for bf16 workloads."""
    st = _streams(L.meta["seed"] if seed is None else seed)
    B = L.queries.shape[0]
    q = make_queries(st["observe"], L.meta["query_basis"], B * n_obs, w.Hq)
    q = q.reshape(B, n_obs, w.Hq, w.d)
    return round_bf16(q) if w.kv_dtype == "bf16" else q


def random_orthonormal(rng, d, r):
    """A d x r matrix with orthonormal columns (QR of a Gaussian)."""
    m = rng.standard_normal((d, r))
    qm, rr = np.linalg.qr(m)
    qm *= np.sign(np.diag(rr))[None, :]
    return qm.astype(np.float32)
