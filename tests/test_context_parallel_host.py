"""Context-parallel (split-T across GPUs) decode on the CPU: the shard ranges,
and a world-size-2 gloo run of the real exchange (exchange buffer layout,
all-gather, unpacking) with the oracle standing in for the two GPU stages --
the local decode over a rank's token range and the merge.  The merged result
must equal one oracle decode over all tokens."""

import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from bit_decode_attention_sm_b200 import context_parallel as cp  # noqa: E402


@pytest.mark.parametrize("T_cap", [0, 1, 64, 1000, 131072])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shard_ranges_partition_the_capacity(T_cap, world):
    ranges = [cp.shard_range(T_cap, r, world) for r in range(world)]
    pos = 0
    for t_lo, n in ranges:
        assert t_lo % cp.ALIGN == 0 or n == 0
        if n:
            assert t_lo == pos
        pos += n
    assert pos == T_cap
    for t in {0, T_cap // 2, T_cap - 1} - {-1}:
        if 0 <= t < T_cap:
            r = cp.owner(t, T_cap, world)
            t_lo, n = ranges[r]
            assert t_lo <= t < t_lo + n


def test_part_stride_keeps_blocks_aligned():
    for BH, d in [(1, 8), (3, 64), (32, 128), (1792, 128), (7, 256)]:
        s = cp.part_stride(BH, d)
        assert s % 4 == 0 and s >= BH * (d + 1)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _layer(T):
    from bit_decode_attention_sm_b200 import configs, synth
    w = configs.workload(2).with_(B=3, T=T, n_cal=64)
    return w, synth.make_layer(w)


def _worker(rank, world, port, T_cap, T, seq_lens, q):
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    w, L = _layer(T_cap)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    dec = cp.ContextParallelDecode(w.B, w.Hq, w.d, T_cap, device=torch.device("cpu"),
                                   local_decode=_oracle_local, merge=_oracle_merge)
    # this rank's cache: the planes of its token range, at local positions
    planes = oracle.cache_write(L.keys[:, :, dec.t_lo:dec.t_lo + dec.cap], U, v=None)
    cache = (planes, L.values[:, :, dec.t_lo:dec.t_lo + dec.cap])
    sl = None if seq_lens is None else np.asarray(seq_lens, np.int32)
    out, lse = dec(cache, L.queries, U, T, seq_lens=sl)
    q.put((rank, out.numpy(), lse.numpy()))
    dist.destroy_process_group()


def _oracle_local(self, cache, q, U, T, seq_lens, o, lse, ws):
    import torch

    import oracle
    planes, v = cache
    n = self.local_tokens(T)
    Tb = np.full(self.B, T) if seq_lens is None else np.clip(seq_lens, 0, T)
    loc = np.clip(Tb - self.t_lo, 0, n).astype(np.int32)
    sub = {k: a[:, :, :n] for k, a in planes.items()}
    out, l_ = oracle.decode(q, sub, U, v=v[:, :, :n], seq_lens=loc)
    o.copy_(torch.from_numpy(out.astype(np.float32)))
    lse.copy_(torch.from_numpy(l_.astype(np.float32)))


def _oracle_merge(self, recv):
    import torch

    import oracle
    blocks = recv.view(self.world, self.stride).numpy().astype(np.float64)
    n = self.BH * self.d
    out, lse = oracle.merge_partials(blocks[:, :n].reshape(self.world, self.BH, self.d),
                                     blocks[:, n:n + self.BH])
    return torch.from_numpy(out), torch.from_numpy(lse)


@pytest.mark.parametrize("T,seq_lens", [(300, None), (250, [250, 100, 0])])
def test_context_parallel_gloo_world2(T, seq_lens):
    import oracle
    T_cap = 320
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, T_cap, T, seq_lens, q))
             for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w, L = _layer(T_cap)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    planes = oracle.cache_write(L.keys[:, :, :T], U)
    sl = None if seq_lens is None else np.asarray(seq_lens, np.int32)
    ref, ref_lse = oracle.decode(L.queries, planes, U, v=L.values[:, :, :T], seq_lens=sl)
    # The partials cross the exchange as fp32: each part's lse is rounded to
    # fp32 (relative 2^-24), so a merge weight e^(lse_r - M) carries a relative
    # error up to about 2 * 2^-24 * max|lse|, and an output element up to that
    # times the largest output magnitude, per part.
    fin_ref = np.isfinite(ref_lse)
    lse_max = float(np.abs(ref_lse[fin_ref]).max()) if fin_ref.any() else 0.0
    atol = 4 * 2.0 ** -24 * max(1.0, lse_max) * float(np.abs(ref).max())
    for _, out, lse in res:
        np.testing.assert_allclose(out, ref, rtol=1e-5, atol=atol)
        fin = np.isfinite(ref_lse)
        np.testing.assert_allclose(lse[fin], ref_lse[fin], rtol=1e-6)
        assert np.isneginf(lse[~fin]).all() and (out[~fin] == 0).all()
    # the ranks agree exactly
    np.testing.assert_array_equal(res[0][1], res[1][1])
