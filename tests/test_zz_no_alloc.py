"""headq_decode_attn_noalloc: decode attention for callers that cannot allocate.

Some callers hold only their input and output buffers (a plugin that a host
framework hands tensors but no allocator, code that may not call cudaMalloc
after start-up), so they cannot provide the workspace headq_decode_attn needs.
This entry point uses a fixed 4 MiB scratch array inside the library instead.
These tests call it through the C ABI and check:
  - that it gives bit for bit what headq_decode_attn gives with a fresh caller
    workspace (same plan, same kernels), on calls in a row of different sizes,
    including a call with many splits followed by one with fewer over the same
    (sequence, KV head) units, so stale partials left in the shared scratch
    would show; and that it is within the decode tolerance of the oracle;
  - that a request too large for the built-in scratch is refused;
  - that a device-side error of a no-alloc call (a block-table entry outside
    the page pool, caught by the kernel's own range check, which skips the bad
    page without touching memory) is reported once by
    headq_decode_noalloc_status and then cleared.

The file is named so that pytest collects it last; it is self-contained and
passes alone in a fresh process as well as after the other tests.
"""

import ctypes
import math

import numpy as np
import pytest

import oracle
from parity_helpers import (DECODE_RTOL, gpu_cache, gpu_query, layer, oracle_side,
                            row_rel_err)

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = 4 << 20
HEADQ_ERR_DEVICE = 5


def _call_noalloc(hq, cache, q, U, T, out, lse, seq_lens=None):
    import torch
    cs = cache.struct()
    P = ctypes.c_void_p
    return hq.lib().headq_decode_attn_noalloc(
        ctypes.byref(cs), P(q.data_ptr()), hq._dtype_code(q), q.shape[1],
        None if seq_lens is None else P(seq_lens.data_ptr()), T, P(U.data_ptr()),
        ctypes.c_float(1.0 / math.sqrt(q.shape[-1])), 1, P(out.data_ptr()),
        P(lse.data_ptr()), P(torch.cuda.current_stream().cuda_stream))


def _status(hq):
    import torch
    return hq.lib().headq_decode_noalloc_status(
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _noalloc_equals_workspace_decode(hq, cache, q, Ut, T, slt):
    import torch
    ref, ref_lse = hq.headq_decode_attn(cache, q, Ut, T=T, seq_lens=slt)
    out = torch.full_like(ref, float("nan"))
    lse = torch.full_like(ref_lse, float("nan"))
    assert _call_noalloc(hq, cache, q, Ut, T, out, lse, slt) == 0
    torch.cuda.synchronize()
    assert _status(hq) == 0
    np.testing.assert_array_equal(out.cpu().numpy(), ref.cpu().numpy())
    np.testing.assert_array_equal(lse.cpu().numpy(), ref_lse.cpu().numpy())
    return out.cpu().numpy()


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
        out = _noalloc_equals_workspace_decode(hq, cache, q, Ut, T, slt)
        _, out_ref, _ = oracle_side(w, L, U, seq_lens=sl)
        assert row_rel_err(out, out_ref) <= DECODE_RTOL


def test_noalloc_more_splits_then_fewer():
    """A call with many splits, then calls with fewer over the same units: the
    later calls must not pick up partials the earlier one left in the scratch."""
    from bit_decode_attention_sm_b200 import headq as hq
    w, L = layer(3, T=4000)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    cache, Ut = gpu_cache(w, L, U)
    q = gpu_query(w, L)
    splits = []
    for T in (4000, 700, 130, 4000):
        s = ctypes.c_int(0)
        hq.lib().headq_decode_plan(ctypes.byref(cache.struct()), w.Hq, T, ctypes.byref(s),
                                   None, None)
        splits.append(s.value)
        out = _noalloc_equals_workspace_decode(hq, cache, q, Ut, T, None)
        sub = type(L)(L.keys[:, :, :T], L.values[:, :, :T], L.queries, L.q_cal, {})
        _, out_ref, _ = oracle_side(w, sub, U)
        assert row_rel_err(out, out_ref) <= DECODE_RTOL
    assert splits[0] > splits[1] > splits[2] >= 1, splits


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


def test_noalloc_reports_device_errors():
    """A block-table entry outside the pool: the kernel's range check redirects
    the read to page 0 and raises the error word of the built-in scratch;
    headq_decode_noalloc_status reports it once, then the word is clear.  The
    other sequence's result is unaffected."""
    import torch
    from bit_decode_attention_sm_b200 import headq as hq
    w, L = layer(2, T=256, B=2)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    _, out_ref, _ = oracle_side(w, L, U)
    page_size, max_pages, spare = 64, 4, 5
    num_pages = 2 * max_pages + spare
    table = np.random.default_rng(0).permutation(num_pages)[:2 * max_pages]
    table = table.reshape(2, max_pages).astype(np.int32)
    dt = torch.bfloat16
    cache = hq.PagedHeadQCache(2, w.Hkv, w.d, w.r, page_size, num_pages, max_pages,
                               vmode=w.vmode, v_dtype=dt, block_table=torch.from_numpy(table))
    Ut = torch.from_numpy(np.ascontiguousarray(U)).cuda()
    hq.headq_cache_write(cache, torch.from_numpy(L.keys).cuda().to(dt),
                         torch.from_numpy(L.values).cuda().to(dt), Ut, t0=0)
    q = gpu_query(w, L)
    out = torch.zeros((2, w.Hq, w.d), dtype=torch.float32, device="cuda")
    lse = torch.zeros((2, w.Hq), dtype=torch.float32, device="cuda")
    assert _call_noalloc(hq, cache, q, Ut, 256, out, lse) == 0   # sets up the scratch
    assert _status(hq) == 0
    cache.block_table[0, 1] = num_pages + 7
    assert _call_noalloc(hq, cache, q, Ut, 256, out, lse) == 0
    assert _status(hq) == HEADQ_ERR_DEVICE
    assert _status(hq) == 0            # the word was cleared
    assert row_rel_err(out[1:].cpu().numpy(), out_ref[1:]) <= DECODE_RTOL
    cache.block_table[0, 1] = int(table[0, 1])
    assert _call_noalloc(hq, cache, q, Ut, 256, out, lse) == 0
    assert _status(hq) == 0
    assert row_rel_err(out.cpu().numpy(), out_ref) <= DECODE_RTOL
