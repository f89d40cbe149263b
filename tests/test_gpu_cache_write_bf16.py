"""bf16 prefills through the cache write (the per-token code at d in {64, 128},
r in {8, 16}) against the oracle, every plane bit-exact (gist.science summary of
HeadQ, section 3, step 2; section 5 for the 2-bit values): many tiles per KV head
and several KV heads, partial last tiles, chunks at an offset, 2-bit values, and
the codec's rounding edges with bf16 inputs.
"""

import numpy as np
import pytest

import oracle
from bit_decode_attention_sm_b200 import synth
from parity_helpers import assert_planes_equal, layer, planes_to_numpy, roundup, torch_dtype
from test_gpu_parity import _edge_keys

pytestmark = pytest.mark.gpu


def _write(w, L, U, t0=0, T_cap=None, chunks=None):
    import torch
    from bit_decode_attention_sm_b200 import headq as hq
    dt = torch_dtype(w)
    B, Hkv, T, d = L.keys.shape
    cache = hq.HeadQCache(B, Hkv, roundup(t0 + T, 16) if T_cap is None else T_cap, d, w.r,
                          vmode=w.vmode, v_dtype=dt)
    Ut = torch.from_numpy(np.ascontiguousarray(U)).cuda()
    pos = 0
    for n in (chunks or [T]):
        k = torch.from_numpy(np.ascontiguousarray(L.keys[:, :, pos:pos + n])).cuda().to(dt)
        v = torch.from_numpy(np.ascontiguousarray(L.values[:, :, pos:pos + n])).cuda().to(dt)
        hq.headq_cache_write(cache, k, v, Ut, t0=t0 + pos)
        pos += n
    return cache


# (workload, sizes): 700, 1000 and 9000 tokens end on partial 64-token tiles
CASES = [(3, dict(T=9000)), (2, dict(T=1000, B=3)), (4, dict(T=700, B=5)), (1, dict(T=2048, B=2))]


@pytest.mark.parametrize("i,kw", CASES, ids=["cfg%d" % c[0] for c in CASES])
def test_bf16_write_bit_exact(i, kw):
    w, L = layer(i, **kw)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    ref = oracle.cache_write(L.keys, U, v=L.values, vmode=w.vmode)
    cache = _write(w, L, U)
    T = L.keys.shape[2]
    assert_planes_equal(planes_to_numpy(cache, 0, T), ref, w.r, w.vmode, w.kv_dtype,
                        values=L.values)


def test_bf16_write_in_chunks_at_an_offset():
    """Chunks of 300, 64 and 333 tokens starting at position 37 write the same
    planes as the oracle on the whole sequence (the first and last tiles of each
    chunk are partial)."""
    w, L = layer(4, T=697, B=3)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    ref = oracle.cache_write(L.keys, U, v=L.values, vmode=w.vmode)
    cache = _write(w, L, U, t0=37, chunks=[300, 64, 333])
    assert_planes_equal(planes_to_numpy(cache, 37, 697), ref, w.r, w.vmode, w.kv_dtype,
                        values=L.values)


@pytest.mark.parametrize("d,r", [(64, 8), (64, 16), (128, 8), (128, 16)])
@pytest.mark.parametrize("vmode", ["dense", "2bit"])
def test_bf16_write_rounding_edges(d, r, vmode):
    """Exact ties, constant, signed-zero, tiny, huge and dyadic groups, rounded to
    bf16 first so that both sides read the same inputs."""
    import torch
    from bit_decode_attention_sm_b200 import headq as hq
    T = 208
    k = synth.round_bf16(_edge_keys(d, T, seed=d + r))
    v = synth.round_bf16(_edge_keys(d, T, seed=d + r + 1))
    rng = np.random.default_rng(11)
    for U in (np.stack([np.round(synth.random_orthonormal(rng, d, r) * 8) / 8]).astype(np.float32),
              np.stack([synth.random_orthonormal(rng, d, r)])):
        ref = oracle.cache_write(k, U, v=v, vmode=vmode)
        cache = hq.HeadQCache(1, 1, T, d, r, vmode=vmode, v_dtype=torch.bfloat16)
        hq.headq_cache_write(cache, torch.from_numpy(k).cuda().to(torch.bfloat16),
                             torch.from_numpy(v).cuda().to(torch.bfloat16),
                             torch.from_numpy(np.ascontiguousarray(U)).cuda())
        assert_planes_equal(planes_to_numpy(cache, 0, T), ref, r, vmode, "bf16", values=v)
