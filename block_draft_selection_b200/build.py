"""Build libdflash.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python block_draft_selection_b200/build.py [--force]

(run as a file: importing the package loads the library this script builds)

The library statically links the CUDA runtime and resolves the driver's
tensor-map encoder at run time, so it needs no libcuda at link time.

Staleness is decided by content, not by file times: a SHA-256 over the
sources' paths and bytes is compiled into the library (dflash_build_id())
and written beside it (libdflash.so.srchash); a library whose recorded hash
differs from the current sources is rebuilt.  A copied tree, a checkout that
resets mtimes, or a prebuilt library carried along with other sources can
therefore never stand in for the sources at hand.
"""
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
LIB = os.path.join(PKG, "libdflash.so")
HASH_FILE = LIB + ".srchash"

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libdflash.so")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def source_hash() -> str:
    """First 16 hex digits of a SHA-256 over every input's path (relative to
    the repository) and bytes, in sorted path order, plus the compile flags."""
    h = hashlib.sha256()
    for f in sorted(_inputs()):
        h.update(os.path.relpath(f, ROOT).replace(os.sep, "/").encode() + b"\0")
        with open(f, "rb") as fh:
            h.update(fh.read())
        h.update(b"\0")
    h.update(" ".join(ARCH + FLAGS).encode())
    return h.hexdigest()[:16]


def recorded_hash():
    try:
        with open(HASH_FILE) as f:
            return f.read().strip()
    except OSError:
        return None


def up_to_date() -> bool:
    return os.path.exists(LIB) and recorded_hash() == source_hash()


def build_library(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    digest = source_hash()
    tmp = LIB + ".tmp"
    cmd = [_nvcc(), *ARCH, *FLAGS, f"-DDFLASH_SOURCE_HASH=\"{digest}\"", "-I", INCLUDE, "-o", tmp, *sources()]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    os.replace(tmp, LIB)
    with open(HASH_FILE, "w") as f:
        f.write(digest + "\n")
    return LIB


if __name__ == "__main__":
    print(build_library(force="--force" in sys.argv, verbose=True))
