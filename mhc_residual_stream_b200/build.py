"""Build libmhc.so in-tree with nvcc for sm_100a.

    python -m mhc_residual_stream_b200.build [--force]

The library links the CUDA runtime statically, so loading it needs only the
NVIDIA driver (and nothing at all until the first CUDA call).
"""

from __future__ import annotations

import hashlib
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libmhc.so")
STAMP = LIB + ".src-sha256"

SOURCES = [os.path.join(CSRC, "mhc_boundary.cu")]
HEADERS = [os.path.join(CSRC, "mhc_device.cuh"), os.path.join(INCLUDE, "mhc.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared", "-cudart", "static",
]


def _nvcc() -> str:
    cand = [os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc"), shutil.which("nvcc")]
    for c in cand:
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found: set CUDA_HOME or put nvcc on PATH")


def source_digest(sources=None, headers=None) -> str:
    h = hashlib.sha256()
    for f in (SOURCES if sources is None else sources) + (HEADERS if headers is None else headers):
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    h.update(" ".join(NVCC_FLAGS).encode())
    return h.hexdigest()


def up_to_date(lib=LIB, sources=None, headers=None) -> bool:
    stamp = lib + ".src-sha256"
    if not (os.path.exists(lib) and os.path.exists(stamp)):
        return False
    with open(stamp) as f:
        return f.read().strip() == source_digest(sources, headers)


def compile_shared(lib, sources, headers, force=False, verbose=False) -> str:
    """Compile `sources` into the shared library `lib` unless its stamp matches
    the sources and headers; return its path."""
    if not force and up_to_date(lib, sources, headers):
        return lib
    tmp = lib + ".tmp"
    cmd = [_nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-o", tmp, *sources]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stderr}")
    if verbose and res.stderr:
        print(res.stderr)
    os.replace(tmp, lib)
    with open(lib + ".src-sha256", "w") as f:
        f.write(source_digest(sources, headers))
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libmhc.so unless it is up to date with the sources; return its path."""
    return compile_shared(LIB, SOURCES, HEADERS, force, verbose)


# The mailbox slot protocol's concurrency check (test infrastructure): one
# cooperative kernel whose blocks play producers and a consumer at the same time.
RACE_LIB = os.path.join(ROOT, "tests", "csrc", "libmhc_mailbox_race.so")
RACE_SOURCES = [os.path.join(ROOT, "tests", "csrc", "mailbox_race.cu")]


def build_race_check(force: bool = False, verbose: bool = False) -> str:
    return compile_shared(RACE_LIB, RACE_SOURCES, HEADERS, force, verbose)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    print(build_race_check(force="--force" in sys.argv, verbose="-v" in sys.argv))
