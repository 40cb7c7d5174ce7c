"""Build libretention.so in-tree with nvcc for sm_100a.

    python -m linear_recurrent_sequence_retention_b200.build [--verbose]

Every ``csrc/*.cu`` is compiled to an object under ``_build/`` (in parallel),
then linked into ``linear_recurrent_sequence_retention_b200/libretention.so``
next to the Python binding that loads it.  Objects are rebuilt when their
source, any header of ``csrc/`` or ``include/`` or the flags change.
"""

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
LIB = os.path.join(PKG, "libretention.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + [
    "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-I" + INCLUDE, "-I" + CSRC,
]


def nvcc():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; CUDA toolkit 12.8+ is required to build libretention")


def source_sha():
    """SHA-256 (hex) of the kernel sources and the public header, as the library embeds it."""
    h = hashlib.sha256()
    files = sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                   + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h")))
    for p in files:
        h.update(os.path.basename(p).encode() + b"\0")
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _digest(src, extra_flags):
    h = hashlib.sha256()
    h.update(" ".join(NVCC_FLAGS + extra_flags).encode())
    headers = sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
                     + glob.glob(os.path.join(INCLUDE, "*.h")))
    for p in [src] + headers:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _compile(src, extra_flags, verbose):
    name = os.path.splitext(os.path.basename(src))[0]
    dig = _digest(src, extra_flags)
    obj = os.path.join(BUILD, f"{name}.{dig}.o")
    if os.path.exists(obj):
        return obj
    cmd = [nvcc()] + NVCC_FLAGS + extra_flags + ["-c", src, "-o", obj + ".tmp"]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout.strip() or r.stderr.strip()):
        print(r.stdout + r.stderr, flush=True)
    os.replace(obj + ".tmp", obj)
    return obj


def build(verbose=False, extra_flags=()):
    """Compile every kernel for sm_100a and link libretention.so; returns its path."""
    os.makedirs(BUILD, exist_ok=True)
    extra = list(extra_flags)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    # api.cu carries the sources' hash (retention_source_sha), so a library
    # built from other sources is refused by the binding
    sha_flag = ["-DRET_SOURCE_SHA=" + source_sha()]

    def one(src):
        flags = extra + (sha_flag if os.path.basename(src) == "api.cu" else [])
        return _compile(src, flags, verbose)

    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(one, srcs))
    tmp = LIB + ".tmp"
    cmd = [nvcc()] + ARCH + ["-shared", "-o", tmp] + objs
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    extra = []
    if "--ptxas-verbose" in sys.argv:
        extra = ["-Xptxas", "-v"]
    print(build(verbose="--verbose" in sys.argv or bool(extra), extra_flags=extra))
