"""Split-T decode across GPUs (context parallel): one long context, several devices.

Rank r of a ``torch.distributed`` group keeps the cached tokens
[t_lo, t_lo + cap) of every sequence (``shard_range``), at local positions
[0, cap) of its own HeadQ cache.  One decode step is then

  1. the local decode over the rank's tokens (``headq_shard_seq_lens`` gives the
     local lengths, ``headq_decode_attn`` writes a normalised partial (o, lse)
     straight into this rank's block of the exchange buffer),
  2. one all-gather of the [o | lse] blocks (NCCL over NVLink on GPUs),
  3. ``headq_merge_partials`` on every rank: the flash-decoding split merge,
     exact because HeadQ changes only the logits (summary section 3, step 3).

The exchange is B*Hq*(d+1) floats per rank and step, independent of T.  New
tokens are written by the rank that owns their position (``owner``) with
``headq_cache_write`` at local position t - t_lo.  The two compute stages are
swappable (``local_decode``, ``merge``) so the exchange logic can be exercised
without a GPU.
"""

import torch
import torch.distributed as dist

from . import headq

ALIGN = 64  # tokens; keeps every rank's range on whole tiles and pages


def shard_range(T_cap, rank, world, align=ALIGN):
    """(t_lo, cap): the contiguous token range rank `rank` of `world` holds when
    the global capacity T_cap is split into equal chunks of a multiple of
    `align` tokens (the last ranks may hold fewer, or none)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    chunk = -(-T_cap // world)
    chunk = -(-chunk // align) * align
    t_lo = min(rank * chunk, T_cap)
    return t_lo, max(0, min(chunk, T_cap - t_lo))


def owner(t, T_cap, world, align=ALIGN):
    """The rank whose range holds global token position t."""
    chunk = -(-T_cap // world)
    chunk = -(-chunk // align) * align
    return t // chunk


def part_stride(BH, d):
    """Floats per rank block of the exchange buffer: [o (BH*d) | lse (BH)],
    padded to 16 bytes."""
    return (BH * d + BH + 3) // 4 * 4


class ContextParallelDecode:
    """Exchange buffers and the three steps above for fixed (B, Hq, d) and a
    fixed global capacity T_cap."""

    def __init__(self, B, Hq, d, T_cap, group=None, device=None, local_decode=None,
                 merge=None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.B, self.Hq, self.d, self.T_cap = B, Hq, d, T_cap
        self.BH = B * Hq
        self.t_lo, self.cap = shard_range(T_cap, self.rank, self.world)
        self.stride = part_stride(self.BH, d)
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        self.send = torch.zeros(self.stride, dtype=torch.float32, device=dev)
        self.recv = torch.zeros(self.world * self.stride, dtype=torch.float32, device=dev)
        self.local_lens = torch.zeros(B, dtype=torch.int32, device=dev)
        self._local = self._cuda_local if local_decode is None else local_decode
        self._merge = self._cuda_merge if merge is None else merge

    def partial_views(self):
        """This rank's block of the exchange buffer as (o [B,Hq,d], lse [B,Hq])."""
        n = self.BH * self.d
        return (self.send[:n].view(self.B, self.Hq, self.d),
                self.send[n:n + self.BH].view(self.B, self.Hq))

    def local_tokens(self, T):
        """How many of the first T global tokens this rank holds."""
        return max(0, min(self.cap, T - self.t_lo))

    def __call__(self, cache, q, U, T, seq_lens=None, ws=None, **kw):
        """Attention over global tokens [0, T) (per-sequence T_b = seq_lens[b]);
        `cache` holds this rank's tokens.  Returns (out [B,Hq,d], lse [B,Hq]),
        identical on every rank."""
        if not 0 <= T <= self.T_cap:
            raise ValueError("T must lie in [0, T_cap]")
        o, lse = self.partial_views()
        self._local(self, cache, q, U, T, seq_lens, o, lse, ws, **kw)
        dist.all_gather_into_tensor(self.recv, self.send, group=self.group)
        out, lse_all = self._merge(self, self.recv)
        return out.view(self.B, self.Hq, self.d), lse_all.view(self.B, self.Hq)

    @staticmethod
    def _cuda_local(self, cache, q, U, T, seq_lens, o, lse, ws, sm_scale=None, corr_sign=1):
        n = self.local_tokens(T)
        lens = headq.headq_shard_seq_lens(seq_lens, self.B, T, self.t_lo, n,
                                          out=self.local_lens, device=q.device)
        headq.headq_decode_attn(cache, q, U, T=n, seq_lens=lens, sm_scale=sm_scale,
                                corr_sign=corr_sign, out=o, lse=lse, ws=ws)

    @staticmethod
    def _cuda_merge(self, recv):
        return headq.headq_merge_partials(recv, self.world, self.BH, self.d, self.stride)
