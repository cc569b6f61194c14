"""Build liblora_b200.so in-tree with nvcc for sm_100a (B200).

    python adapter_deltas_b200/_build.py [--verbose] [--debug]

Compiles every ``csrc/*.cu`` into one shared library next to this file.  The
library exports the C ABI declared in ``include/lora.h``.  ``--debug`` builds
liblora_b200_debug.so instead, with LORA_DEBUG defined: the kernels then check
the indices and pages they are about to use and record LORA_ERR_BOUNDS in the
pool's sticky status instead of touching memory outside the buffers (the
binding loads it when LORA_B200_DEBUG=1).
"""

from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "liblora_b200.so")
LIB_DEBUG = os.path.join(HERE, "liblora_b200_debug.so")
SOURCES = sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))
HEADERS = sorted(glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h")))

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and not stale(lib):
        return lib
    objs = []
    build_dir = os.path.join(ROOT, "_build", "debug" if debug else "release")
    os.makedirs(build_dir, exist_ok=True)
    for src in SOURCES:
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        cmd = [nvcc(), *NVCC_FLAGS, *(["-DLORA_DEBUG"] if debug else []), "-I", os.path.join(ROOT, "include"),
               "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = lib + ".tmp.%d" % os.getpid()
    subprocess.run([nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
                    "-o", tmp, *objs, "-ldl"], check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv, debug="--debug" in sys.argv))
