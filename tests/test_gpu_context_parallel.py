"""Split-T across devices (context parallel) on one GPU, against the oracle.

Each emulated rank owns a cache holding only its token range; its local decode
(headq_shard_seq_lens + headq_decode_attn) writes a partial into its block of
one exchange buffer, exactly as the all-gather would leave it on every rank,
and headq_merge_partials combines the blocks.  The result must match one
oracle decode over all tokens.  The ranks run one after another: no kernel
waits on another.  The last test drives ContextParallelDecode through a real
NCCL process group of one rank.
"""

import numpy as np
import pytest

import oracle
from bit_decode_attention_sm_b200 import context_parallel as cp
from parity_helpers import (DECODE_RTOL, gpu_cache, gpu_query, layer, oracle_side,
                            row_rel_err)

pytestmark = pytest.mark.gpu


def _headq():
    from bit_decode_attention_sm_b200 import headq
    return headq


def emulated_ranks(w, L, U, world, T_cap, T, seq_lens):
    import torch
    hq = _headq()
    B, Hq, d = L.queries.shape
    BH = B * Hq
    stride = cp.part_stride(BH, d)
    buf = torch.full((world * stride,), float("nan"), dtype=torch.float32, device="cuda")
    q = gpu_query(w, L)
    slt = None if seq_lens is None else torch.from_numpy(seq_lens).cuda()
    for r in range(world):
        t_lo, cap = cp.shard_range(T_cap, r, world)
        n = max(0, min(cap, T - t_lo))
        blk = buf[r * stride:(r + 1) * stride]
        o = blk[:BH * d].view(B, Hq, d)
        lse = blk[BH * d:BH * d + BH].view(B, Hq)
        shard = type(L)(L.keys[:, :, t_lo:t_lo + cap], L.values[:, :, t_lo:t_lo + cap],
                        L.queries, L.q_cal, {})
        cache, Ut = gpu_cache(w, shard, U, T_cap=max(16, -(-cap // 16) * 16))
        lens = hq.headq_shard_seq_lens(slt, B, T, t_lo, n)
        if seq_lens is not None:
            ref_lens = np.clip(np.clip(seq_lens, 0, T) - t_lo, 0, n)
            np.testing.assert_array_equal(lens.cpu().numpy(), ref_lens)
        hq.headq_decode_attn(cache, q, Ut, T=n, seq_lens=lens, out=o, lse=lse)
    return hq.headq_merge_partials(buf, world, BH, d, stride)


@pytest.mark.parametrize("world", [2, 3, 5])
@pytest.mark.parametrize("i,kw,T,sl", [
    (2, dict(T=1024, B=3), 1000, [1000, 300, 0]),
    (3, dict(T=2560), 2500, None),
    (4, dict(T=704, B=2), 700, [700, 64]),
], ids=["cfg2", "cfg3", "cfg4"])
def test_split_t_across_emulated_ranks(world, i, kw, T, sl):
    w, L = layer(i, **kw)
    T_cap = L.keys.shape[2]
    sl = None if sl is None else np.array(sl, np.int32)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    planes = oracle.cache_write(L.keys[:, :, :T], U, v=L.values[:, :, :T], vmode=w.vmode)
    out_ref, lse_ref = oracle.decode(L.queries, planes, U, v=L.values[:, :, :T], vmode=w.vmode,
                                     seq_lens=sl)
    out, lse = emulated_ranks(w, L, U, world, T_cap, T, sl)
    o = out.view(L.queries.shape).cpu().numpy()
    l_ = lse.view(L.queries.shape[:2]).cpu().numpy()
    fin = np.isfinite(lse_ref)
    assert row_rel_err(o[fin], out_ref[fin]) <= DECODE_RTOL
    np.testing.assert_allclose(l_[fin], lse_ref[fin], rtol=1e-5, atol=1e-4)
    assert (o[~fin] == 0).all() and np.isneginf(l_[~fin]).all()


def test_merge_partials_edge_rows():
    """Rows no part covers, one part only, and a part whose block holds NaN
    garbage but lse = -inf (it must not leak into the result)."""
    import torch
    hq = _headq()
    S, BH, d = 3, 4, 64
    stride = cp.part_stride(BH, d)
    rng = np.random.default_rng(0)
    o = rng.standard_normal((S, BH, d)).astype(np.float32)
    lse = rng.standard_normal((S, BH)).astype(np.float32)
    lse[:, 0] = -np.inf                   # row 0: no part
    lse[1:, 1] = -np.inf                  # row 1: part 0 only
    lse[2, 2] = -np.inf
    o[2, 2] = np.nan                      # row 2: part 2 empty with garbage output
    buf = np.zeros((S, stride), np.float32)
    buf[:, :BH * d] = o.reshape(S, -1)
    buf[:, BH * d:BH * d + BH] = lse
    out, l_ = hq.headq_merge_partials(torch.from_numpy(buf.reshape(-1)).cuda(), S, BH, d, stride)
    ref, ref_l = oracle.merge_partials(np.where(np.isnan(o), 0, o), lse)
    got, got_l = out.cpu().numpy(), l_.cpu().numpy()
    assert (got[0] == 0).all() and np.isneginf(got_l[0])
    np.testing.assert_array_equal(got[1], o[0, 1])
    assert np.isfinite(got).all()
    np.testing.assert_allclose(got[1:], ref[1:], rtol=2e-6, atol=1e-6)
    np.testing.assert_allclose(got_l[1:], ref_l[1:], rtol=1e-6)


def test_context_parallel_decode_nccl_world1():
    """ContextParallelDecode over a real NCCL group of one rank: the exchange is
    a copy and the merge of one part returns it unchanged, so the result equals
    headq_decode_attn bit for bit (the decode is deterministic)."""
    import os
    import socket
    from datetime import timedelta

    import torch
    import torch.distributed as dist
    hq = _headq()
    w, L = layer(2, T=640, B=2)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    _, out_ref, _ = oracle_side(w, L, U)
    cache, Ut = gpu_cache(w, L, U)
    q = gpu_query(w, L)
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        dec = cp.ContextParallelDecode(*L.queries.shape, cache.T_cap)
        ws = hq.decode_workspace(cache, w.Hq, 640)
        out, lse = dec(cache, q, Ut, 640, ws=ws)
        torch.cuda.synchronize()
        direct, direct_lse = hq.headq_decode_attn(cache, q, Ut, T=640)
        assert torch.equal(out, direct) and torch.equal(lse, direct_lse)
        assert row_rel_err(out.cpu().numpy(), out_ref) <= DECODE_RTOL
    finally:
        dist.destroy_process_group()
