"""headq_decode_attn_noalloc: decode attention for callers that cannot allocate.

Some callers hold only their input and output buffers (a plugin that a host
framework hands tensors but no allocator, code that may not call cudaMalloc
after start-up), so they cannot provide the workspace headq_decode_attn needs.
This entry point uses a fixed 4 MiB scratch array inside the library instead.
These tests call it through the C ABI and check it against headq_decode_attn
with a caller workspace, on two calls in a row of different sizes, and check
that a request too large for the built-in scratch is refused.

The file is named so that pytest collects it last; it is self-contained and
passes alone in a fresh process as well as after the other tests.
"""

import ctypes
import math

import numpy as np
import pytest

import oracle
from parity_helpers import (DECODE_RTOL, gpu_cache, gpu_query, layer, row_rel_err)

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = 4 << 20


def _call_noalloc(hq, cache, q, U, T, out, lse, seq_lens=None):
    import torch
    cs = cache.struct()
    P = ctypes.c_void_p
    return hq.lib().headq_decode_attn_noalloc(
        ctypes.byref(cs), P(q.data_ptr()), hq._dtype_code(q), q.shape[1],
        None if seq_lens is None else P(seq_lens.data_ptr()), T, P(U.data_ptr()),
        ctypes.c_float(1.0 / math.sqrt(q.shape[-1])), 1, P(out.data_ptr()),
        P(lse.data_ptr()), P(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_workspace_decode_twice():
    import torch
    from bit_decode_attention_sm_b200 import headq as hq
    cases = [(2, dict(T=1000, B=2), None), (3, dict(T=2500), None),
             (1, dict(T=300), np.array([300, 1, 0, 77, 300, 150, 299, 64], np.int32))]
    for i, kw, sl in cases:
        w, L = layer(i, **kw)
        U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
        cache, Ut = gpu_cache(w, L, U)
        q = gpu_query(w, L)
        T = L.keys.shape[2]
        slt = None if sl is None else torch.from_numpy(sl).cuda()
        need = hq.lib().headq_decode_workspace_bytes(ctypes.byref(cache.struct()), w.Hq, T)
        assert 0 < need <= SCRATCH_LIMIT
        ref, ref_lse = hq.headq_decode_attn(cache, q, Ut, T=T, seq_lens=slt)
        out = torch.full_like(ref, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        assert _call_noalloc(hq, cache, q, Ut, T, out, lse, slt) == 0
        torch.cuda.synchronize()
        r, o = ref.cpu().numpy(), out.cpu().numpy()
        assert row_rel_err(o, r.astype(np.float64)) <= DECODE_RTOL
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), rtol=1e-6,
                                   atol=1e-6)


def test_noalloc_refuses_requests_beyond_its_scratch():
    import torch
    from bit_decode_attention_sm_b200 import headq as hq
    # a cache descriptor whose partials would exceed the scratch (never launched:
    # the size check fails first, so the buffers are not touched)
    cache = hq.HeadQCache(64, 16, 1024, 128, 16, device="cuda")
    cs = cache.struct()
    cs.B = 4096   # claims far more sequences than the buffers hold
    need = hq.lib().headq_decode_workspace_bytes(ctypes.byref(cs), 64, 1024)
    assert need > SCRATCH_LIMIT
    q = torch.zeros((1, 64, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((1, 64, 128), dtype=torch.float32, device="cuda")
    lse = torch.zeros((1, 64), dtype=torch.float32, device="cuda")
    U = torch.zeros((16, 128, 16), dtype=torch.float32, device="cuda")
    P = ctypes.c_void_p
    st = hq.lib().headq_decode_attn_noalloc(
        ctypes.byref(cs), P(q.data_ptr()), 1, 64, None, 1024, P(U.data_ptr()),
        ctypes.c_float(0.1), 1, P(out.data_ptr()), P(lse.data_ptr()),
        P(torch.cuda.current_stream().cuda_stream))
    assert st == 3  # HEADQ_ERR_WORKSPACE
