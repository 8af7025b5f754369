"""Build the in-tree CUDA library ``libdvlm.so`` for sm_100a.

Each ``csrc/*.cu`` is compiled to an object under ``_build/`` and the objects
are linked into ``block_diffusion_vlm_b200/libdvlm.so`` with the CUDA runtime
linked statically.  Staleness is decided by content, not by file times: an
object is rebuilt unless the stamp beside it records the SHA-256 of its
source, of every header and of the compiler command, and the library is
relinked unless its stamp records the hashes of all objects.  A copied tree
whose times were reset therefore never reuses objects built from other
sources.  Usage: ``python -m block_diffusion_vlm_b200.build [-j N] [--clean]``.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libdvlm.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr"]
LINK_LIBS = ["-lpthread", "-ldl", "-lrt"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def _sha(paths, extra: str = "") -> str:
    h = hashlib.sha256(extra.encode())
    for p in paths:
        h.update(os.path.basename(p).encode())
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _stamp(path: str) -> str | None:
    try:
        with open(path + ".sha256") as f:
            return f.read().strip()
    except OSError:
        return None


def _write_stamp(path: str, digest: str) -> None:
    with open(path + ".sha256", "w") as f:
        f.write(digest + "\n")


def _compile(src: str, obj: str, digest: str) -> None:
    cmd = [nvcc(), *ARCH, *FLAGS, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {os.path.basename(src)}:\n{r.stderr}")
    _write_stamp(obj, digest)


def build(jobs: int = 8, verbose: bool = False, clean: bool = False) -> str:
    if clean and os.path.isdir(BUILD):
        shutil.rmtree(BUILD)
    os.makedirs(BUILD, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = _headers()
    cmd_key = " ".join([*ARCH, *FLAGS])
    hdr_digest = _sha(headers, cmd_key)
    work, objs = [], []
    for s in srcs:
        o = os.path.join(BUILD, os.path.splitext(os.path.basename(s))[0] + ".o")
        objs.append(o)
        d = _sha([s], hdr_digest)
        if not os.path.exists(o) or _stamp(o) != d:
            work.append((s, o, d))
    if work:
        with cf.ThreadPoolExecutor(max_workers=max(1, jobs)) as ex:
            futs = [ex.submit(_compile, s, o, d) for s, o, d in work]
            for f in futs:
                f.result()
    lib_digest = _sha(objs, " ".join(LINK_LIBS))
    relinked = False
    if not os.path.exists(LIB) or _stamp(LIB) != lib_digest:
        tmp = LIB + ".tmp"
        cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs, *LINK_LIBS]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stderr}")
        os.replace(tmp, LIB)
        _write_stamp(LIB, lib_digest)
        relinked = True
    if verbose:
        print(f"built {LIB} ({len(work)} of {len(srcs)} objects compiled from source"
              f"{', relinked' if relinked else ''})")
    return LIB


if __name__ == "__main__":
    j = 8
    if "-j" in sys.argv:
        j = int(sys.argv[sys.argv.index("-j") + 1])
    build(jobs=j, verbose=True, clean="--clean" in sys.argv)
