"""Python binding of libheadq (``include/headq.h``): argument marshalling only.

Every computation runs in the CUDA kernels of ``libheadq.so``; this module
only allocates device memory through PyTorch, passes pointers, sizes and the
current CUDA stream, and turns status codes into exceptions.  There is no CPU
fallback: without the built library, or with tensors that are not on a CUDA
device, every call raises.

Names follow the C ABI: :func:`headq_calibrate`, :func:`headq_cache_write`,
:func:`headq_decode_attn`, :func:`headq_attn_kl`, plus :class:`HeadQCache`
which owns the packed cache planes.
"""

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libheadq.so")

HEADQ_F32, HEADQ_BF16 = 0, 1
HEADQ_V_DENSE, HEADQ_V_2BIT = 0, 1
STATUS = {0: "HEADQ_OK", 1: "HEADQ_ERR_INVALID_ARG", 2: "HEADQ_ERR_UNSUPPORTED",
          3: "HEADQ_ERR_WORKSPACE", 4: "HEADQ_ERR_CUDA", 5: "HEADQ_ERR_DEVICE"}

# Every entry point declared in include/headq.h.
EXPORTS = ("headq_version", "headq_status_string", "headq_calibrate",
           "headq_calibrate_workspace_bytes", "headq_cache_write", "headq_decode_attn",
           "headq_decode_workspace_bytes", "headq_decode_plan", "headq_attn_kl",
           "headq_attn_kl_workspace_bytes", "headq_workspace_status",
           "headq_decode_attn_noalloc", "headq_decode_noalloc_status",
           "headq_decode_append", "headq_shard_seq_lens",
           "headq_merge_partials", "headq_a2_workspace_bytes", "headq_a2_scores",
           "headq_a2_select", "headq_a2_value_fixup")


KMODES = {"token": 0, "channel": 1}  # headq_kmode


class HeadQError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__("%s failed: %s" % (fn, STATUS.get(status, status)))


class CacheStruct(ctypes.Structure):
    """Mirror of ``headq_cache``."""
    _fields_ = [("B", ctypes.c_int), ("Hkv", ctypes.c_int), ("T_cap", ctypes.c_int),
                ("d", ctypes.c_int), ("r", ctypes.c_int), ("vmode", ctypes.c_int),
                ("v_dtype", ctypes.c_int),
                ("k_codes", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
                ("k_min", ctypes.c_void_p), ("z_codes", ctypes.c_void_p),
                ("z_scale", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("v_codes", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
                ("v_min", ctypes.c_void_p),
                ("page_size", ctypes.c_int), ("num_pages", ctypes.c_int),
                ("max_pages", ctypes.c_int), ("block_table", ctypes.c_void_p),
                ("kmode", ctypes.c_int)]


_lib = None


def lib():
    """The loaded libheadq; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libheadq.so is not built: run "
                               "`python -m bit_decode_attention_sm_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        F = ctypes.c_float
        CP = ctypes.POINTER(CacheStruct)
        sig = {
            "headq_version": ([], I),
            "headq_status_string": ([I], ctypes.c_char_p),
            "headq_calibrate": ([P, I, I, I, I, I, I, I, P, P, P, Z, P], I),
            "headq_calibrate_workspace_bytes": ([I, I, I, I], Z),
            "headq_cache_write": ([CP, P, P, I, I, I, P, P], I),
            "headq_decode_attn": ([CP, P, I, I, P, I, P, F, I, P, P, P, Z, P], I),
            "headq_decode_workspace_bytes": ([CP, I, I], Z),
            "headq_decode_plan": ([CP, I, I, P, P, P], I),
            "headq_attn_kl": ([CP, P, I, I, P, I, P, P, I, P, F, I, P, P, P, P, P, Z, P], I),
            "headq_attn_kl_workspace_bytes": ([CP, I, I], Z),
            "headq_workspace_status": ([P, P], I),
            "headq_decode_attn_noalloc": ([CP, P, I, I, P, I, P, F, I, P, P, P], I),
            "headq_decode_noalloc_status": ([P], I),
            "headq_decode_append": ([CP, P, P, I, P, I, I, P, I, P, F, I, P, P, P, Z, P], I),
            "headq_shard_seq_lens": ([P, I, I, I, I, P, P], I),
            "headq_merge_partials": ([P, P, I, I, I, Z, P, P, P], I),
            "headq_a2_workspace_bytes": ([CP, I, I, I], Z),
            "headq_a2_scores": ([CP, P, I, I, I, P, I, P, P, I, F, P, P, Z, P], I),
            "headq_a2_select": ([P, I, I, P, I, I, P, I, I, P, P, P], I),
            "headq_a2_value_fixup": ([CP, P, I, I, P, I, P, F, I, P, P, I, I, P, P, P], I),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(fn, st):
    if st != 0:
        raise HeadQError(fn, st)


def _dtype_code(t):
    if t.dtype == torch.float32:
        return HEADQ_F32
    if t.dtype == torch.bfloat16:
        return HEADQ_BF16
    raise TypeError("HeadQ tensors are float32 or bfloat16, got %s" % t.dtype)


def _cuda(t, name):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class HeadQCache:
    """Caller-owned packed HeadQ cache planes on one CUDA device.

    Planes follow ``headq_cache`` in include/headq.h: k_codes u8
    [B,Hkv,T_cap,d/4], k_scale/k_min f32 [B,Hkv,T_cap,NG], z_codes u8
    [B,Hkv,T_cap,r/2], z_scale f32 [B,Hkv,T_cap], and either v
    [B,Hkv,T_cap,d] (dense) or v_codes/v_scale/v_min (2-bit).
    """

    page_size = num_pages = max_pages = 0
    block_table = None
    kmode = "token"

    def __init__(self, B, Hkv, T_cap, d, r, vmode="dense", v_dtype=torch.bfloat16,
                 device="cuda", kmode="token"):
        if T_cap % (64 if kmode == "channel" else 16):
            raise ValueError("T_cap must be a multiple of 16 (64 for per-channel keys)")
        self.B, self.Hkv, self.T_cap, self.d, self.r = B, Hkv, T_cap, d, r
        self._alloc((B, Hkv, T_cap), vmode, v_dtype, device, kmode)

    def _alloc(self, lead, vmode, v_dtype, device, kmode="token"):
        d, r = self.d, self.r
        if kmode not in KMODES:
            raise ValueError("kmode is 'token' or 'channel'")
        self.vmode = vmode
        self.v_dtype = v_dtype
        self.kmode = kmode
        ng = d // min(32, d)
        u8, f32 = torch.uint8, torch.float32
        self.k_codes = torch.zeros(lead + (d // 4,), dtype=u8, device=device)
        # per-token groups, or (per-channel code) one row of d per 64-token block
        sshape = lead + (ng,) if kmode == "token" else lead[:-1] + (lead[-1] // 64, d)
        self.k_scale = torch.zeros(sshape, dtype=f32, device=device)
        self.k_min = torch.zeros(sshape, dtype=f32, device=device)
        self.z_codes = torch.zeros(lead + (max(r // 2, 1),), dtype=u8, device=device)
        self.z_scale = torch.zeros(lead, dtype=f32, device=device)
        self.v = self.v_codes = self.v_scale = self.v_min = None
        if vmode == "dense":
            self.v = torch.zeros(lead + (d,), dtype=v_dtype, device=device)
        elif vmode == "2bit":
            self.v_codes = torch.zeros(lead + (d // 4,), dtype=u8, device=device)
            self.v_scale = torch.zeros(lead + (ng,), dtype=f32, device=device)
            self.v_min = torch.zeros(lead + (ng,), dtype=f32, device=device)
        else:
            raise ValueError("vmode is 'dense' or '2bit'")

    def planes(self):
        out = dict(kc=self.k_codes, ks=self.k_scale, km=self.k_min, zc=self.z_codes,
                   zs=self.z_scale)
        if self.vmode == "2bit":
            out.update(vc=self.v_codes, vs=self.v_scale, vm=self.v_min)
        else:
            out.update(v=self.v)
        return out

    def nbytes_per_token(self):
        """Bytes one cached token of one KV head occupies in HBM."""
        ng = self.d // min(32, self.d)
        b = self.d // 4 + (8 * ng if self.kmode == "token" else self.d // 8) + self.r // 2 + 4
        if self.vmode == "2bit":
            b += self.d // 4 + 8 * ng
        else:
            b += self.d * (2 if self.v_dtype == torch.bfloat16 else 4)
        return b

    def struct(self):
        s = CacheStruct()
        s.B, s.Hkv, s.T_cap, s.d, s.r = self.B, self.Hkv, self.T_cap, self.d, self.r
        s.vmode = HEADQ_V_DENSE if self.vmode == "dense" else HEADQ_V_2BIT
        s.v_dtype = HEADQ_BF16 if self.v_dtype == torch.bfloat16 else HEADQ_F32
        s.k_codes = self.k_codes.data_ptr()
        s.k_scale = self.k_scale.data_ptr()
        s.k_min = self.k_min.data_ptr()
        s.z_codes = self.z_codes.data_ptr()
        s.z_scale = self.z_scale.data_ptr()
        if self.vmode == "dense":
            s.v = self.v.data_ptr()
        else:
            s.v_codes = self.v_codes.data_ptr()
            s.v_scale = self.v_scale.data_ptr()
            s.v_min = self.v_min.data_ptr()
        if self.page_size:
            s.page_size, s.num_pages, s.max_pages = self.page_size, self.num_pages, self.max_pages
            s.block_table = self.block_table.data_ptr()
        s.kmode = KMODES[self.kmode]
        return s


class PagedHeadQCache(HeadQCache):
    """HeadQ cache planes held as pools of fixed-size pages (``headq_cache``
    paged layout): every plane is [num_pages, Hkv, page_size, ...] and
    ``block_table`` int32 [B, max_pages] names the pool page that holds tokens
    [i*page_size, (i+1)*page_size) of sequence b.  page_size is a multiple of
    64; a sequence holds up to T_cap = max_pages * page_size tokens.  The
    default block table gives sequence b pages b*max_pages .. b*max_pages +
    max_pages - 1 (it needs num_pages >= B * max_pages); any other table may be
    assigned to ``block_table`` before a call."""

    def __init__(self, B, Hkv, d, r, page_size, num_pages, max_pages, vmode="dense",
                 v_dtype=torch.bfloat16, device="cuda", block_table=None, kmode="token"):
        if page_size <= 0 or page_size % 64:
            raise ValueError("page_size must be a positive multiple of 64")
        self.B, self.Hkv, self.d, self.r = B, Hkv, d, r
        self.page_size, self.num_pages, self.max_pages = page_size, num_pages, max_pages
        self.T_cap = max_pages * page_size
        if block_table is None:
            if num_pages < B * max_pages:
                raise ValueError("the default block table needs B * max_pages pages")
            block_table = torch.arange(B * max_pages, dtype=torch.int32).view(B, max_pages)
        self.block_table = block_table.to(device=device, dtype=torch.int32).contiguous()
        if tuple(self.block_table.shape) != (B, max_pages):
            raise ValueError("block_table must be [B, max_pages]")
        self._alloc((num_pages, Hkv, page_size), vmode, v_dtype, device, kmode)


def headq_calibrate(q_cal, Hkv, r, center=False, stream=None):
    """Query-PCA basis per KV head: returns (U fp32 [Hkv,d,r], eig fp32 [Hkv,r])."""
    q_cal = _cuda(q_cal, "q_cal")
    N, Hq, d = q_cal.shape
    L = lib()
    U = torch.empty((Hkv, d, r), dtype=torch.float32, device=q_cal.device)
    eig = torch.empty((Hkv, r), dtype=torch.float32, device=q_cal.device)
    nws = L.headq_calibrate_workspace_bytes(N, Hq, Hkv, d)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=q_cal.device)
    _check("headq_calibrate", L.headq_calibrate(
        _ptr(q_cal), _dtype_code(q_cal), N, Hq, Hkv, d, r, int(bool(center)), _ptr(U),
        _ptr(eig), _ptr(ws), nws, _stream(stream)))
    return U, eig


def headq_cache_write(cache, k, v, U, t0=0, stream=None):
    """Encode k (and store v) [B,Hkv,n,d] into cache positions [t0, t0+n)."""
    k = _cuda(k, "k")
    v = _cuda(v, "v")
    if v is not None and v.dtype != k.dtype:
        raise TypeError("k and v must have the same dtype")
    n = k.shape[2]
    U = _cuda(U, "U") if cache.r > 0 else None
    cs = cache.struct()
    _check("headq_cache_write", lib().headq_cache_write(
        ctypes.byref(cs), _ptr(k), _ptr(v), _dtype_code(k), int(t0), int(n), _ptr(U),
        _stream(stream)))


def decode_workspace(cache, Hq, T):
    """A zeroed device workspace sized for headq_decode_attn."""
    cs = cache.struct()
    n = lib().headq_decode_workspace_bytes(ctypes.byref(cs), Hq, T)
    return torch.zeros(n, dtype=torch.uint8, device=cache.k_codes.device)


def decode_plan(cache, Hq, T):
    """(splits, chunk, kernels per headq_decode_attn call, kernels per
    headq_decode_append call) for these sizes on the current device."""
    cs = cache.struct()
    sp, ch, ak = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    nk = lib().headq_decode_plan(ctypes.byref(cs), Hq, T, ctypes.byref(sp), ctypes.byref(ch),
                                 ctypes.byref(ak))
    return sp.value, ch.value, nk, ak.value


def attn_kl_workspace(cache, Hq, T):
    cs = cache.struct()
    n = lib().headq_attn_kl_workspace_bytes(ctypes.byref(cs), Hq, T)
    return torch.zeros(n, dtype=torch.uint8, device=cache.k_codes.device)


def headq_decode_attn(cache, q, U, T=None, seq_lens=None, sm_scale=None, corr_sign=1,
                      out=None, lse=None, ws=None, stream=None):
    """Decode attention over the cache; returns (out fp32 [B,Hq,d], lse fp32 [B,Hq])."""
    q = _cuda(q, "q")
    B, Hq, d = q.shape
    T = cache.T_cap if T is None else int(T)
    sm = 1.0 / math.sqrt(d) if sm_scale is None else float(sm_scale)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = decode_workspace(cache, Hq, T)
    seq_lens = _cuda(seq_lens, "seq_lens")
    U = _cuda(U, "U") if cache.r > 0 else None
    cs = cache.struct()
    _check("headq_decode_attn", lib().headq_decode_attn(
        ctypes.byref(cs), _ptr(q), _dtype_code(q), Hq, _ptr(seq_lens), T, _ptr(U), sm,
        int(corr_sign), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return out, lse


def headq_decode_append(cache, k_new, v_new, q, U, T=None, seq_lens=None, sm_scale=None,
                        corr_sign=1, out=None, lse=None, ws=None, stream=None):
    """One decode step: write each sequence's new token (k_new, v_new [B,Hkv,d]) at
    position T_b - 1, then attend; returns (out fp32 [B,Hq,d], lse fp32 [B,Hq])."""
    q = _cuda(q, "q")
    k_new = _cuda(k_new, "k_new")
    v_new = _cuda(v_new, "v_new")
    if v_new is not None and v_new.dtype != k_new.dtype:
        raise TypeError("k_new and v_new must have the same dtype")
    B, Hq, d = q.shape
    T = cache.T_cap if T is None else int(T)
    sm = 1.0 / math.sqrt(d) if sm_scale is None else float(sm_scale)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = decode_workspace(cache, Hq, T)
    seq_lens = _cuda(seq_lens, "seq_lens")
    U = _cuda(U, "U") if cache.r > 0 else None
    cs = cache.struct()
    _check("headq_decode_append", lib().headq_decode_append(
        ctypes.byref(cs), _ptr(k_new), _ptr(v_new), _dtype_code(k_new), _ptr(q), _dtype_code(q),
        Hq, _ptr(seq_lens), T, _ptr(U), sm, int(corr_sign), _ptr(out), _ptr(lse), _ptr(ws),
        ws.numel(), _stream(stream)))
    return out, lse


def headq_attn_kl(cache, q, U, k_full, v_full, T=None, seq_lens=None, sm_scale=None,
                  corr_sign=1, ws=None, stream=None):
    """Returns (kl, fisher_var, a2_vdist, dout2), each fp32 [B, Hq]."""
    q = _cuda(q, "q")
    k_full = _cuda(k_full, "k_full")
    v_full = _cuda(v_full, "v_full")
    B, Hq, d = q.shape
    T = k_full.shape[2] if T is None else int(T)
    sm = 1.0 / math.sqrt(d) if sm_scale is None else float(sm_scale)
    res = [torch.empty((B, Hq), dtype=torch.float32, device=q.device) for _ in range(4)]
    if ws is None:
        ws = attn_kl_workspace(cache, Hq, T)
    seq_lens = _cuda(seq_lens, "seq_lens")
    U = _cuda(U, "U") if cache.r > 0 else None
    cs = cache.struct()
    _check("headq_attn_kl", lib().headq_attn_kl(
        ctypes.byref(cs), _ptr(q), _dtype_code(q), Hq, _ptr(seq_lens), T, _ptr(k_full),
        _ptr(v_full), _dtype_code(k_full), _ptr(U), sm, int(corr_sign),
        *[_ptr(t) for t in res], _ptr(ws), ws.numel(), _stream(stream)))
    return tuple(res)


def headq_shard_seq_lens(seq_lens, B, T, t_lo, n, out=None, device="cuda", stream=None):
    """int32 [B] local lengths clamp(T_b - t_lo, 0, n) of a token range [t_lo, t_lo+n)."""
    seq_lens = _cuda(seq_lens, "seq_lens")
    dev = seq_lens.device if seq_lens is not None else device
    out = torch.empty(B, dtype=torch.int32, device=dev) if out is None else out
    _check("headq_shard_seq_lens", lib().headq_shard_seq_lens(
        _ptr(seq_lens), int(B), int(T), int(t_lo), int(n), _ptr(out), _stream(stream)))
    return out


def headq_merge_partials(parts, S, BH, d, part_stride, out=None, lse=None, stream=None):
    """Combine S partial decodes held in one fp32 buffer of S blocks of
    part_stride floats, each [out (BH*d) | lse (BH) | padding]; returns
    (out fp32 [BH, d], lse fp32 [BH])."""
    parts = _cuda(parts, "parts")
    if parts.dtype != torch.float32 or parts.numel() < S * part_stride:
        raise ValueError("parts must be fp32 with S * part_stride elements")
    out = torch.empty((BH, d), dtype=torch.float32, device=parts.device) if out is None else out
    lse = torch.empty(BH, dtype=torch.float32, device=parts.device) if lse is None else lse
    _check("headq_merge_partials", lib().headq_merge_partials(
        _ptr(parts), ctypes.c_void_p(parts.data_ptr() + 4 * BH * d), int(S), int(BH), int(d),
        int(part_stride), _ptr(out), _ptr(lse), _stream(stream)))
    return out, lse


def a2_workspace(cache, n_obs, Hq, T):
    cs = cache.struct()
    n = lib().headq_a2_workspace_bytes(ctypes.byref(cs), n_obs, Hq, T)
    return torch.zeros(max(n, 16), dtype=torch.uint8, device=cache.k_codes.device)


def headq_a2_scores(cache, q_obs, k_full, v_full, T=None, seq_lens=None, sm_scale=None,
                    ws=None, out=None, stream=None):
    """A^2 policy scores a_j fp32 [B, Hkv, T] from observation queries
    q_obs [B, n_obs, Hq, d] and the exact keys/values [B, Hkv, T, d]."""
    q_obs = _cuda(q_obs, "q_obs")
    k_full = _cuda(k_full, "k_full")
    v_full = _cuda(v_full, "v_full")
    seq_lens = _cuda(seq_lens, "seq_lens")
    B, n_obs, Hq, d = q_obs.shape
    T = k_full.shape[2] if T is None else int(T)
    sm = 1.0 / math.sqrt(d) if sm_scale is None else float(sm_scale)
    ws = a2_workspace(cache, n_obs, Hq, T) if ws is None else ws
    out = torch.empty((cache.B, cache.Hkv, T), dtype=torch.float32,
                      device=q_obs.device) if out is None else out
    cs = cache.struct()
    _check("headq_a2_scores", lib().headq_a2_scores(
        ctypes.byref(cs), _ptr(q_obs), _dtype_code(q_obs), n_obs, Hq, _ptr(seq_lens), T,
        _ptr(k_full), _ptr(v_full), _dtype_code(k_full), ctypes.c_float(sm), _ptr(out),
        _ptr(ws), ws.numel(), _stream(stream)))
    return out


def headq_a2_select(scores, K, v_full, seq_lens=None, keep_idx=None, keep_v=None, stream=None):
    """Top-K kept positions (int32 [B, Hkv, K], ascending, -1 padded) and their
    exact values [B, Hkv, K, d] (v_full's dtype)."""
    scores = _cuda(scores, "scores")
    v_full = _cuda(v_full, "v_full")
    seq_lens = _cuda(seq_lens, "seq_lens")
    B, Hkv, T = scores.shape
    d = v_full.shape[-1]
    keep_idx = torch.empty((B, Hkv, K), dtype=torch.int32,
                           device=scores.device) if keep_idx is None else keep_idx
    keep_v = torch.empty((B, Hkv, K, d), dtype=v_full.dtype,
                         device=scores.device) if keep_v is None else keep_v
    _check("headq_a2_select", lib().headq_a2_select(
        _ptr(scores), B, Hkv, _ptr(seq_lens), T, int(K), _ptr(v_full), _dtype_code(v_full), d,
        _ptr(keep_idx), _ptr(keep_v), _stream(stream)))
    return keep_idx, keep_v


def headq_a2_value_fixup(cache, q, U, keep_idx, keep_v, out, lse, T=None, seq_lens=None,
                         sm_scale=None, corr_sign=1, stream=None):
    """out += the kept tokens' exact-minus-cached value readout (after a decode
    that wrote out and lse with the same arguments)."""
    q = _cuda(q, "q")
    keep_idx = _cuda(keep_idx, "keep_idx")
    keep_v = _cuda(keep_v, "keep_v")
    seq_lens = _cuda(seq_lens, "seq_lens")
    B, Hq, d = q.shape
    T = cache.T_cap if T is None else int(T)
    sm = 1.0 / math.sqrt(d) if sm_scale is None else float(sm_scale)
    U = _cuda(U, "U") if cache.r > 0 else None
    cs = cache.struct()
    _check("headq_a2_value_fixup", lib().headq_a2_value_fixup(
        ctypes.byref(cs), _ptr(q), _dtype_code(q), Hq, _ptr(seq_lens), T, _ptr(U),
        ctypes.c_float(sm), int(corr_sign), _ptr(keep_idx), _ptr(keep_v), _dtype_code(keep_v),
        keep_idx.shape[-1], _ptr(out), _ptr(lse), _stream(stream)))
    return out


def headq_workspace_status(ws, stream=None):
    """Synchronises and raises HeadQError if a kernel flagged a device-side error."""
    _check("headq_workspace_status", lib().headq_workspace_status(_ptr(ws), _stream(stream)))
