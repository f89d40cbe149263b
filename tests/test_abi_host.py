"""The C ABI on a machine without a GPU: the library loads, exports every entry
point include/headq.h declares, and rejects bad arguments on the host before
anything is launched.  No call here reaches a kernel launch."""

import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "headq.h")


@pytest.fixture(scope="module")
def hq():
    from bit_decode_attention_sm_b200 import build, headq
    build.build()
    return headq


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(headq_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(hq):
    names = declared_functions()
    assert "headq_decode_attn" in names and len(names) >= 10
    lib = hq.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(hq.EXPORTS)
    out = subprocess.check_output(["nm", "-D", "--defined-only", hq.LIB_PATH], text=True)
    exported = set(re.findall(r"\bT (headq_\w+)", out))
    assert set(names) <= exported


def test_version_and_status_strings(hq):
    lib = hq.lib()
    assert lib.headq_version() == 101
    for code in range(6):
        assert lib.headq_status_string(code)
    assert lib.headq_status_string(99) == b"unknown status"


FAKE = 0x7f0000000000  # 16-byte aligned address, never dereferenced


def make_cache(hq, d=128, r=16, T_cap=1024, B=1, Hkv=2, vmode=0, **over):
    s = hq.CacheStruct()
    s.B, s.Hkv, s.T_cap, s.d, s.r, s.vmode, s.v_dtype = B, Hkv, T_cap, d, r, vmode, 1
    for i, f in enumerate(("k_codes", "k_scale", "k_min", "z_codes", "z_scale", "v",
                           "v_codes", "v_scale", "v_min")):
        setattr(s, f, FAKE + 0x100000 * i)
    for k, v in over.items():
        setattr(s, k, v)
    return s


def _write(hq, cs, k=FAKE, t0=0, n=1, U=FAKE):
    return hq.lib().headq_cache_write(ctypes.byref(cs), ctypes.c_void_p(k), None, 1, t0, n,
                                      ctypes.c_void_p(U), None)


def test_cache_write_rejects(hq):
    L = hq.lib()
    assert L.headq_cache_write(None, None, None, 1, 0, 1, None, None) == 1
    assert _write(hq, make_cache(hq, d=48)) == 2
    assert _write(hq, make_cache(hq, r=3)) == 2
    assert _write(hq, make_cache(hq, r=34, d=64)) == 2
    assert _write(hq, make_cache(hq, T_cap=100)) == 2
    assert _write(hq, make_cache(hq, k_codes=FAKE + 1)) == 1
    assert _write(hq, make_cache(hq, z_scale=0)) == 1
    assert _write(hq, make_cache(hq, v=0)) == 1
    assert _write(hq, make_cache(hq, vmode=1, v_codes=0)) == 1
    assert _write(hq, make_cache(hq), k=0) == 1
    assert _write(hq, make_cache(hq), k=FAKE + 8) == 1
    assert _write(hq, make_cache(hq), U=0) == 1
    assert _write(hq, make_cache(hq), t0=1000, n=100) == 1
    assert _write(hq, make_cache(hq), t0=-1) == 1
    # n == 0 is a no-op that launches nothing and reads no input pointer
    assert _write(hq, make_cache(hq), n=0) == 0
    assert _write(hq, make_cache(hq), k=0, U=0, n=0) == 0


def _decode(hq, cs, Hq=4, T=512, corr=1, ws_bytes=1 << 30, q=FAKE, out=FAKE, ws=FAKE):
    return hq.lib().headq_decode_attn(
        ctypes.byref(cs), ctypes.c_void_p(q), 1, Hq, None, T, ctypes.c_void_p(FAKE),
        ctypes.c_float(0.1), corr, ctypes.c_void_p(out), None, ctypes.c_void_p(ws), ws_bytes,
        None)


def test_decode_rejects(hq):
    cs = make_cache(hq)
    assert _decode(hq, cs, Hq=3) == 1
    assert _decode(hq, cs, corr=2) == 1
    assert _decode(hq, cs, T=2048) == 1
    assert _decode(hq, cs, q=0) == 1
    assert _decode(hq, cs, out=FAKE + 4) == 1
    assert _decode(hq, cs, ws=0) == 3
    assert _decode(hq, cs, ws_bytes=16) == 3
    assert _decode(hq, make_cache(hq, d=256), Hq=2 * 9) == 2      # G*d > 2048
    assert _decode(hq, make_cache(hq, d=40)) == 2


def test_workspace_and_plan(hq):
    L = hq.lib()
    cs = make_cache(hq, B=1, Hkv=8)
    sp, ch, ak = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    nk = L.headq_decode_plan(ctypes.byref(cs), 32, 131072 // 128, ctypes.byref(sp),
                             ctypes.byref(ch), ctypes.byref(ak))
    assert nk in (1, 2) and ak.value in (1, 2, 3) and sp.value >= 1 and ch.value % 16 == 0
    assert sp.value * ch.value >= 1024
    n = L.headq_decode_workspace_bytes(ctypes.byref(cs), 32, 1024)
    assert n >= 256 + 4 * 32 * sp.value * (128 + 2)
    assert L.headq_decode_workspace_bytes(None, 32, 1024) == 0
    assert L.headq_attn_kl_workspace_bytes(ctypes.byref(cs), 32, 1024) >= 256
    assert L.headq_calibrate_workspace_bytes(1024, 32, 8, 128) >= 2 * 8 * 128 * 128 * 8
    assert L.headq_workspace_status(None, None) == 1


def test_paged_cache_rejects(hq):
    """Paged layout fields are checked before any launch."""
    def paged(**over):
        kw = dict(T_cap=1024, page_size=64, num_pages=40, max_pages=16, block_table=FAKE + 0x900000)
        kw.update(over)
        return make_cache(hq, **kw)
    assert _write(hq, paged(page_size=48)) == 2
    assert _write(hq, paged(page_size=-64)) == 1
    assert _write(hq, paged(block_table=0)) == 1
    assert _write(hq, paged(block_table=FAKE + 0x900004)) == 1
    assert _write(hq, paged(num_pages=0)) == 1
    assert _write(hq, paged(max_pages=0)) == 1
    assert _write(hq, paged(max_pages=8)) == 1            # 8 * 64 != T_cap
    assert _decode(hq, paged(page_size=96, max_pages=10, T_cap=960)) == 2
    assert _write(hq, paged(), n=0) == 0                  # valid, and a no-op
    # the tensor-core plan keeps every 64-token tile inside one page
    cs = paged(B=1, Hkv=8, T_cap=131072, max_pages=2048, num_pages=2048)
    sp, ch = ctypes.c_int(), ctypes.c_int()
    hq.lib().headq_decode_plan(ctypes.byref(cs), 32, 131072, ctypes.byref(sp), ctypes.byref(ch),
                               None)
    assert ch.value % 64 == 0 and sp.value * ch.value >= 131072


def test_paged_cache_struct_on_host(hq):
    """PagedHeadQCache lays the planes out as page pools and passes its table."""
    import torch
    c = hq.PagedHeadQCache(2, 4, 128, 16, 128, 9, 3, device="cpu")
    assert c.T_cap == 384 and tuple(c.k_codes.shape) == (9, 4, 128, 32)
    assert tuple(c.z_scale.shape) == (9, 4, 128) and tuple(c.v.shape) == (9, 4, 128, 128)
    assert c.block_table.tolist() == [[0, 1, 2], [3, 4, 5]]
    s = c.struct()
    assert (s.page_size, s.num_pages, s.max_pages, s.T_cap) == (128, 9, 3, 384)
    assert s.block_table == c.block_table.data_ptr()
    with pytest.raises(ValueError):
        hq.PagedHeadQCache(2, 4, 128, 16, 100, 9, 3, device="cpu")
    with pytest.raises(ValueError):
        hq.PagedHeadQCache(4, 4, 128, 16, 128, 9, 3, device="cpu")   # pool too small
    t = torch.tensor([[5, 0, 1], [2, 3, 4]], dtype=torch.int32)
    c2 = hq.PagedHeadQCache(2, 4, 128, 16, 128, 9, 3, device="cpu", block_table=t)
    assert c2.block_table.tolist() == t.tolist()


def test_channel_keys_rejects(hq):
    """Per-channel keys: capacity and write offsets on 64-token blocks, no
    single-token append, no A^2 fixup; an unknown key mode is an argument error."""
    L = hq.lib()
    assert _write(hq, make_cache(hq, kmode=7)) == 1
    assert _write(hq, make_cache(hq, kmode=1, T_cap=1040)) == 2      # not a multiple of 64
    assert _write(hq, make_cache(hq, kmode=1), t0=16, n=1) == 2       # not a block start
    assert _write(hq, make_cache(hq, kmode=1), t0=64, n=0) == 0       # valid no-op
    cs = make_cache(hq, kmode=1)
    P = ctypes.c_void_p
    assert L.headq_decode_append(ctypes.byref(cs), P(FAKE), None, 1, P(FAKE), 1, 4, None, 512,
                                 P(FAKE), ctypes.c_float(0.1), 1, P(FAKE), None, P(FAKE),
                                 1 << 30, None) == 2
    assert L.headq_a2_value_fixup(ctypes.byref(cs), P(FAKE), 1, 4, None, 512, P(FAKE),
                                  ctypes.c_float(0.1), 1, P(FAKE), P(FAKE), 1, 8, P(FAKE),
                                  P(FAKE), None) == 2


def test_channel_cache_struct_on_host(hq):
    c = hq.HeadQCache(2, 4, 256, 128, 16, kmode="channel", device="cpu")
    assert tuple(c.k_scale.shape) == (2, 4, 4, 128) and tuple(c.k_codes.shape) == (2, 4, 256, 32)
    assert c.struct().kmode == 1 and c.nbytes_per_token() == 32 + 16 + 8 + 4 + 256
    pc = hq.PagedHeadQCache(2, 4, 64, 8, 128, 5, 2, kmode="channel", device="cpu")
    assert tuple(pc.k_min.shape) == (5, 4, 2, 64)
    with pytest.raises(ValueError):
        hq.HeadQCache(1, 1, 80, 64, 8, kmode="channel", device="cpu")


def test_calibrate_rejects(hq):
    L = hq.lib()
    P = ctypes.c_void_p
    big = 1 << 30
    assert L.headq_calibrate(P(FAKE), 1, 64, 8, 2, 256, 8, 0, P(FAKE), None, P(FAKE), big,
                             None) == 2
    assert L.headq_calibrate(P(FAKE), 1, 64, 8, 3, 64, 8, 0, P(FAKE), None, P(FAKE), big,
                             None) == 1
    assert L.headq_calibrate(P(FAKE), 1, 64, 8, 2, 64, 65, 0, P(FAKE), None, P(FAKE), big,
                             None) == 2
    assert L.headq_calibrate(P(FAKE), 1, 64, 8, 2, 64, 8, 0, P(FAKE), None, P(FAKE), 8,
                             None) == 3
    assert L.headq_calibrate(None, 1, 64, 8, 2, 64, 8, 0, P(FAKE), None, P(FAKE), big,
                             None) == 1


def test_binding_refuses_cpu_tensors(hq):
    import torch
    q = torch.zeros(1, 4, 64)
    with pytest.raises(ValueError):
        hq.headq_calibrate(q, 1, 8)
