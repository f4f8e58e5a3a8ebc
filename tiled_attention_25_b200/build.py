"""Build libattn25.so in-tree with nvcc for sm_100a.

Usage: python tiled_attention_25_b200/build.py [--trace]  (or call build()).
Run it as a script: importing the package would first load the library.
Each .cu file compiles to an object under _build/ in parallel; objects are
reused while their sources and headers are unchanged.
"""
from __future__ import annotations

import concurrent.futures
import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libattn25.so")
TRACE_LIB = os.path.join(HERE, "libattn25_trace.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-I", CSRC, "-I", INCLUDE,
]


def _sources():
    return sorted(f for f in os.listdir(CSRC) if f.endswith(".cu"))


def _headers_digest(flags):
    h = hashlib.sha256()
    for d in (CSRC, INCLUDE):
        for f in sorted(os.listdir(d)):
            if f.endswith((".h", ".cuh")):
                with open(os.path.join(d, f), "rb") as fh:
                    h.update(f.encode() + fh.read())
    h.update(" ".join(flags).encode())
    return h.hexdigest()


def _compile(src, digest, verbose, flags):
    path = os.path.join(CSRC, src)
    with open(path, "rb") as fh:
        key = hashlib.sha256(fh.read() + digest.encode()).hexdigest()[:16]
    obj = os.path.join(BUILD, f"{src[:-3]}.{key}.o")
    if os.path.exists(obj):
        return obj
    cmd = [NVCC, *flags, "-c", path, "-o", obj + ".tmp"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr}")
    if verbose:
        sys.stderr.write(r.stderr)
    os.replace(obj + ".tmp", obj)
    return obj


def build(verbose: bool = False, trace: bool = False) -> str:
    """Build libattn25.so (or, with trace=True, the profiling variant
    libattn25_trace.so whose kernels count cycles per warp role)."""
    os.makedirs(BUILD, exist_ok=True)
    flags = FLAGS + (["-DATTN25_TRACE"] if trace else [])
    lib = TRACE_LIB if trace else LIB
    digest = _headers_digest(flags)
    with concurrent.futures.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        objs = list(ex.map(lambda s: _compile(s, digest, verbose, flags), _sources()))
    link_key = hashlib.sha256("".join(objs).encode()).hexdigest()[:16]
    stamp = os.path.join(BUILD, os.path.basename(lib) + ".stamp")
    if os.path.exists(lib) and os.path.exists(stamp) and open(stamp).read() == link_key:
        return lib
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", lib + ".tmp",
           *objs, "-cudart", "static", "-Xlinker", "--no-undefined"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(lib + ".tmp", lib)
    with open(stamp, "w") as fh:
        fh.write(link_key)
    return lib


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, trace="--trace" in sys.argv))
