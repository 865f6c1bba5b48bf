"""Builds libattnqat.so (sm_100a) in-tree with nvcc.

The library is one translation unit (csrc/libattnqat.cu includes the kernel
sources) linked against the shared CUDA runtime, so it shares the runtime
that PyTorch loads in the same process.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libattnqat.so")
ARCH = "-gencode=arch=compute_100a,code=sm_100a"


def _nvcc() -> str:
    cand = [os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc"),
            shutil.which("nvcc") or ""]
    for c in cand:
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libattnqat.so")


def sources() -> list:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h")))


def sources_digest() -> str:
    """SHA-256 over the library's sources (identifies the kernels a profile
    was taken on)."""
    import hashlib
    h = hashlib.sha256()
    for path in sources():
        h.update(os.path.basename(path).encode())
        h.update(open(path, "rb").read())
    return h.hexdigest()[:16]


# The files that determine the attention kernels' code (their ncu counters
# stay valid while these are unchanged).
ATTENTION_SOURCES = ("fwd.cu", "bwd.cu", "common.cuh", "device.cuh", "internal.h")


def code_only(text: str) -> str:
    """C/C++ source with its comments removed and whitespace collapsed (the
    sources hold no string literal with a comment marker in it)."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def attention_sources_digest(read=None) -> str:
    """SHA-256 over the attention kernels' own sources, comments removed, so
    that a comment edit keeps the digest of the same code.  `read(name)`
    returns a file's text (default: the working tree)."""
    import hashlib
    if read is None:
        read = lambda name: open(os.path.join(CSRC, name), encoding="utf-8").read()  # noqa: E731
    h = hashlib.sha256()
    for name in ATTENTION_SOURCES:
        h.update(name.encode())
        h.update(code_only(read(name)).encode())
    return h.hexdigest()[:16]


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if it is missing or older than its sources."""
    if not force and not stale():
        return LIB
    cuda_home = os.path.dirname(os.path.dirname(_nvcc()))
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = [_nvcc(), "-shared", "-Xcompiler", "-fPIC", "-O3", "-lineinfo", "-std=c++17", ARCH,
           "-I" + INCLUDE, "-cudart", "shared",
           "-Xlinker", "-rpath," + os.path.join(cuda_home, "lib64"),
           "-o", tmp, os.path.join(CSRC, "libattnqat.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose=True))
