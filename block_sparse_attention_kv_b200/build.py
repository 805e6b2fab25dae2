"""Build libabsp.so (CUDA, sm_100a) in-tree with nvcc.

    python -m block_sparse_attention_kv_b200.build [--verbose-ptxas]

The shared library lands in block_sparse_attention_kv_b200/lib/ and is what
the ctypes binding loads.  A library is reused only when it was built from
the current sources: the hash of the sources, headers, this script and the
flags is compiled into it (absp_build_id()) and kept beside it.  cudart is linked statically, so the library only
needs the CUDA driver at run time.
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
LIB = os.path.join(LIBDIR, "libabsp.so")
SOURCES = ["abi.cu", "centroids.cu", "decode.cu", "noalloc.cu"]
HEADERS = ["absp_internal.cuh", "absp_trace.h"]

# a second build for profiling only: the decode kernel records phase stamps
# (ABSP_PHASE_STAMPS); the product library never carries them
LIB_STAMPS = os.path.join(LIBDIR, "libabsp_stamps.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17"]
STAMP_FLAGS = ["-DABSP_PHASE_STAMPS"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found (set NVCC or install the CUDA toolkit)")


def source_hash(extra_flags=()) -> str:
    """SHA-256 (first 16 hex digits) of everything the library is built
    from: the CUDA sources and headers, the public header, this script and
    the compile flags.  It is compiled into the library (absp_build_id) and
    decides whether an existing library is reused."""
    h = hashlib.sha256()
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(INCLUDE, "absp.h"))
    deps.append(os.path.abspath(__file__))
    for p in deps:
        h.update(os.path.basename(p).encode())
        with open(p, "rb") as f:
            h.update(f.read())
    h.update(" ".join(ARCH + FLAGS + list(extra_flags)).encode())
    return h.hexdigest()[:16]


def built_id(lib: str = LIB) -> str:
    """Build id recorded beside a library at its last build ('' if none)."""
    try:
        with open(lib + ".build_id") as f:
            return f.read().strip()
    except OSError:
        return ""


def _stale(want: str, lib: str = LIB) -> bool:
    return not os.path.exists(lib) or built_id(lib) != want


def build(force: bool = False, verbose_ptxas: bool = False, stamps: bool = False) -> str:
    """Compile the library unless the one in place was built from exactly
    the current sources (same source hash); return its path.  `stamps`:
    the profiling build with the decode kernel's phase stamps, a separate
    library."""
    extra = STAMP_FLAGS if stamps else []
    lib = LIB_STAMPS if stamps else LIB
    want = source_hash(extra)
    if not force and not verbose_ptxas and not _stale(want, lib):
        return lib
    os.makedirs(LIBDIR, exist_ok=True)
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH, *FLAGS, *extra, f"-DABSP_BUILD_ID=\"{want}\"", "-shared",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "-I", INCLUDE, "-cudart", "static",
           "-o", tmp] + [os.path.join(CSRC, f) for f in SOURCES]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    # exported symbols: everything declared in absp.h is marked visible by
    # the extern "C" block below via a linker version script
    vs = os.path.join(LIBDIR, "absp.map")
    with open(vs, "w") as f:
        f.write("{ global: absp_*; local: *; };\n")
    cmd += ["-Xlinker", f"--version-script={vs}"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libabsp.so")
    if verbose_ptxas:
        sys.stderr.write(res.stderr)
    os.replace(tmp, lib)
    with open(lib + ".build_id", "w") as f:
        f.write(want + "\n")
    return lib


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas))


if __name__ == "__main__":
    main()
