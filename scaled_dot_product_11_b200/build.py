"""Build libsdpa_b200.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m scaled_dot_product_11_b200.build [--verbose]

nvcc links the CUDA runtime statically and the library reaches the driver
through the runtime's entry-point query, so the .so loads (and exports its
symbols) on machines without a GPU driver; it only needs one to run.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libsdpa_b200.so")
# translation units, compiled in parallel and linked into one library
SOURCES = [os.path.join(CSRC, "sdpa_api.cu"), os.path.join(CSRC, "sdpa_fwd2q.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))] + \
    [os.path.join(INCLUDE, "sdpa.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-I", INCLUDE, "-I", CSRC,
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def nvcc_available() -> bool:
    exe = nvcc()
    return bool(shutil.which(exe)) or os.path.exists(exe)


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in DEPS)


def build(force: bool = False, verbose: bool = False, out: str = LIB, defines=()) -> str:
    """Compile every translation unit (in parallel) and link the shared
    library at `out`.  `defines` are extra -D flags (tuning knobs)."""
    if out == LIB and not force and not needs_build():
        return out
    tag = "%d" % os.getpid()
    objs, procs = [], []
    extra = ["-D%s" % d for d in defines] + (["-Xptxas", "-v"] if verbose else [])
    for src in SOURCES:
        obj = "%s.%s.%s.o" % (out, os.path.basename(src), tag)
        objs.append(obj)
        procs.append(subprocess.Popen([nvcc()] + NVCC_FLAGS + extra + ["-c", "-o", obj, src]))
    try:
        codes = [pr.wait() for pr in procs]
        if any(codes):
            raise subprocess.CalledProcessError(max(codes), "nvcc -c")
        tmp = out + ".tmp" + tag
        subprocess.run([nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                        "-o", tmp] + objs, check=True)
        os.replace(tmp, out)
    finally:
        for obj in objs:
            if os.path.exists(obj):
                os.remove(obj)
    return out


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
