"""Build libconvrot.so (the sm_100a CUDA library behind include/convrot.h)
in-tree with nvcc.

The library carries the hash of the sources and flags it was compiled from
(convrot_build_id()).  A library whose id differs from the hash of the
sources next to it -- a stale build, or one copied in from elsewhere -- is
rebuilt; modification times are not trusted.
"""
from __future__ import annotations

import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libconvrot.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-cudart", "static",
]


def sources():
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC))
            if f.endswith((".cu", ".cuh", ".h"))] + [
        os.path.join(HERE, "..", "include", "convrot.h")]


def source_hash(files=None, flags=None) -> str:
    """16 hex digits of SHA-256 over the compile flags and the sources'
    names and contents: the id a library built from them carries."""
    h = hashlib.sha256()
    h.update(" ".join(NVCC_FLAGS if flags is None else flags).encode() + b"\0")
    for f in (sources() if files is None else files):
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode() + b"\0" + fh.read() + b"\0")
    return h.hexdigest()[:16]


def library_build_id(lib: str = LIB):
    """The id compiled into a built library (convrot_build_id()), read in a
    child process so that this process never maps a library it may replace;
    None if it cannot be loaded or has no id."""
    code = ("import ctypes, sys\n"
            "l = ctypes.CDLL(sys.argv[1])\n"
            "f = l.convrot_build_id\n"
            "f.restype = ctypes.c_char_p\n"
            "print(f().decode())\n")
    try:
        out = subprocess.run([sys.executable, "-c", code, lib], capture_output=True, text=True, timeout=120)
    except Exception:  # noqa: BLE001
        return None
    if out.returncode != 0:
        return None
    return out.stdout.strip() or None


def needs_build(lib: str = LIB, expected: str | None = None) -> bool:
    """True when the library is missing or was built from other sources."""
    if not os.path.exists(lib):
        return True
    return library_build_id(lib) != (source_hash() if expected is None else expected)


def build(force: bool = False, verbose: bool = False) -> str:
    if force or needs_build():
        bid = source_hash()
        tmp = LIB + ".tmp.%d" % os.getpid()
        cmd = [NVCC, *NVCC_FLAGS, '-DCONVROT_BUILD_ID="%s"' % bid, "-o", tmp, os.path.join(CSRC, "libconvrot.cu")]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), file=sys.stderr)
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
