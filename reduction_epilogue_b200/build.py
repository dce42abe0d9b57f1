"""Builds libfle.so (the CUDA library behind include/fle.h) in-tree for sm_100a,
and its barrier-checking twin libfle_check.so (the same sources compiled with
-DFLE_CHECK_BARRIERS, for tests; the binding loads it when FLE_BUILD=check).

    python -m reduction_epilogue_b200.build [--verbose]

nvcc cross-compiles without a GPU.  The library links the CUDA runtime
statically and reaches the driver's tensor-map encoder through
cudaGetDriverEntryPoint, so it needs no libcuda at link time.
"""
from __future__ import annotations

import argparse
import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libfle.so")
CHECK_LIB = os.path.join(LIBDIR, "libfle_check.so")
SOURCES = [os.path.join(CSRC, "fle_api.cu")]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-cudart", "static"]
CHECK_FLAGS = ["-DFLE_CHECK_BARRIERS"]
# marker before the hash inside the built library (fle_api.cu)
HASH_TAG = b"fle-source-sha256:"


def _inputs():
    """Every file the library is compiled from, in a fixed order."""
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh", ".h"))]
    files += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    return sorted(files, key=lambda f: os.path.relpath(f, ROOT))


def source_hash(check: bool = False) -> str:
    """SHA-256 of the sources (by path relative to the repository root) and
    of the compile flags (of the checking build when check is set)."""
    h = hashlib.sha256()
    h.update(" ".join(ARCH + FLAGS + (CHECK_FLAGS if check else [])).encode())
    for f in _inputs():
        h.update(b"\0" + os.path.relpath(f, ROOT).encode() + b"\0")
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def built_hash(path: str = LIB):
    """The source hash compiled into a built library, or None."""
    if not os.path.exists(path):
        return None
    with open(path, "rb") as f:
        data = f.read()
    i = data.find(HASH_TAG)
    if i < 0:
        return None
    tail = data[i + len(HASH_TAG): i + len(HASH_TAG) + 64]
    try:
        return tail.decode("ascii")
    except UnicodeDecodeError:
        return None


def sources_present() -> bool:
    return all(os.path.exists(f) for f in SOURCES)


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def needs_build(check: bool = False) -> bool:
    """True unless the library exists and was built from exactly these sources."""
    return built_hash(CHECK_LIB if check else LIB) != source_hash(check)


def build(force: bool = False, verbose: bool = False) -> str:
    """Builds whichever of the two libraries is missing or stale (both at
    once, in parallel); returns the product library's path."""
    jobs = []
    os.makedirs(LIBDIR, exist_ok=True)
    for check in (False, True):
        if not force and not needs_build(check):
            continue
        lib = CHECK_LIB if check else LIB
        tmp = lib + ".tmp%d" % os.getpid()
        digest = source_hash(check)
        cmd = [nvcc(), *ARCH, *FLAGS, *(CHECK_FLAGS if check else []), f'-DFLE_SOURCE_HASH="{digest}"',
               "-I", INCLUDE, "-I", CSRC, "-o", tmp, *SOURCES]
        if verbose and not check:
            cmd.insert(1, "-Xptxas=-v")
        jobs.append((subprocess.Popen(cmd), lib, tmp, digest))
    failed = [j for j in jobs if j[0].wait() != 0]
    for proc, lib, tmp, digest in jobs:
        if failed or built_hash(tmp) != digest:
            if os.path.exists(tmp):
                os.unlink(tmp)
            continue
        os.replace(tmp, lib)
    if failed:
        raise subprocess.CalledProcessError(failed[0][0].returncode, failed[0][0].args)
    for _, lib, _, digest in jobs:
        if built_hash(lib) != digest:
            raise RuntimeError(f"{lib} does not carry the source hash it was built with")
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true", help="print ptxas register/spill/smem lines")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force or a.verbose, verbose=a.verbose))
    sys.exit(0)
