"""Build libheadq.so (the CUDA C-ABI library) in-tree for sm_100a with nvcc.

    python -m bit_decode_attention_sm_b200.build [--verbose]

Each translation unit is compiled to an object under ``_build/`` and linked
into ``bit_decode_attention_sm_b200/libheadq.so``.  The shared codec
(``codec.cuh``) states every step with explicit round-to-nearest intrinsics
(``__fmul_rn``, ``__fadd_rn``, ``mul.rn.f32x2``/``add.rn.f32x2``), which the
compiler never contracts, so it is bit-exact in every file that includes it;
``cache_write.cu`` is also compiled with ``-fmad=false`` for its own arithmetic
around the codec.  No file uses fast-math, so division, square root and
denormals keep IEEE semantics.
"""

import concurrent.futures
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libheadq.so")

SOURCES = ["headq_api.cu", "cache_write.cu", "decode_attn.cu", "attn_kl.cu",
           "calibrate.cu", "decode_noalloc.cu", "decode_mma.cu", "decode_hm.cu", "attn_kl_hm.cu", "merge.cu",
           "a2_policy.cu"]
PER_FILE_FLAGS = {"cache_write.cu": ["-fmad=false"]}
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
          "-I" + INCLUDE, "-I" + CSRC]


def nvcc():
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force=False, verbose=False):
    os.makedirs(BUILD, exist_ok=True)
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")]
    headers.append(os.path.join(INCLUDE, "headq.h"))
    objs, cmds = [], []
    for src in SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(BUILD, src.replace(".cu", ".o"))
        objs.append(obj)
        if force or _stale(obj, [path, *headers]):
            cmd = [nvcc(), *ARCH, *COMMON, *PER_FILE_FLAGS.get(src, [])]
            if verbose:
                cmd += ["-Xptxas", "-v"]
            cmds.append(cmd + ["-c", path, "-o", obj])
    # the translation units are independent: compile them side by side
    workers = max(1, min(len(cmds), os.cpu_count() or 1))
    with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as ex:
        for f in [ex.submit(subprocess.check_call, c) for c in cmds]:
            f.result()
    if force or _stale(LIB, objs):
        tmp = LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call([nvcc(), *ARCH, "-shared", "-o", tmp, *objs])
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
