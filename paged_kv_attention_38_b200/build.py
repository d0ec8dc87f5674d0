"""Build libpkv.so in-tree: nvcc for sm_100a, one shared library, C ABI only.

Usage: python -m paged_kv_attention_38_b200.build  (or build() from Python).
Objects are compiled in parallel into paged_kv_attention_38_b200/_build/. An
object is reused only when a SHA-256 over everything that goes into it (the
compiler's version, the command line, the source and every header of the
library) matches the digest stored beside it; the library is relinked unless
the digest of its objects and link line matches too. File times play no part,
so a tree copied to another machine with other mtimes rebuilds exactly what
changed.
"""
from __future__ import annotations

import concurrent.futures as cf
import functools
import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libpkv.so")
INCLUDE = os.path.join(ROOT, "include")

SOURCES = ["api.cu", "planner.cpp", "prefill_sm100.cu", "decode_sm100.cu", "merge.cu", "mla_sm100.cu", "mla_decode_sm100.cu",
           "decode_noalloc.cu", "append.cu", "selftest.cu", "decode_fp8_sm100.cu", "kv_fp8_expand.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", CSRC, "-I", INCLUDE]


def _nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


@functools.lru_cache(maxsize=None)
def _nvcc_version() -> str:
    return subprocess.run([_nvcc(), "--version"], capture_output=True, text=True).stdout


def _headers():
    hs = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh")))
    return hs + [os.path.join(INCLUDE, "pkv.h")]


def _digest(cmd, files) -> str:
    h = hashlib.sha256()
    h.update(_nvcc_version().encode())
    h.update("\0".join(cmd).encode())
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def _up_to_date(out: str, digest: str) -> bool:
    stamp = out + ".sha256"
    if not (os.path.exists(out) and os.path.exists(stamp)):
        return False
    with open(stamp) as f:
        return f.read().strip() == digest


def _stamp(out: str, digest: str) -> None:
    with open(out + ".sha256", "w") as f:
        f.write(digest + "\n")


def _compile(src: str, verbose_ptxas: bool) -> tuple[str, str]:
    obj = os.path.join(BUILD, os.path.basename(src) + ".o")
    if src.endswith(".cpp"):
        cmd = [_nvcc(), *FLAGS, "-x", "c++", "-c", src, "-o", obj]
    else:
        cmd = [_nvcc(), *ARCH, *FLAGS, "-c", src, "-o", obj]
    digest = _digest(cmd, [src, *_headers()])
    if _up_to_date(obj, digest) and not verbose_ptxas:
        return obj, digest
    if verbose_ptxas and src.endswith(".cu"):
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose_ptxas:
        sys.stderr.write(r.stderr)
    _stamp(obj, digest)
    return obj, digest


def build(verbose_ptxas: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        built = list(ex.map(lambda s: _compile(s, verbose_ptxas), srcs))
    objs = [o for o, _ in built]
    tmp = LIB + ".tmp"
    cmd = [_nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static", "-Xcompiler", "-fPIC"]
    h = hashlib.sha256("\0".join(cmd).encode())
    for _, d in built:
        h.update(d.encode())
    digest = h.hexdigest()
    if _up_to_date(LIB, digest):
        return LIB
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    _stamp(LIB, digest)
    return LIB


if __name__ == "__main__":
    print(build(verbose_ptxas="-v" in sys.argv))
