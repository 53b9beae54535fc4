"""Builds libntx.so in-tree: nvcc for sm_100a, no JIT cache."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
SO = os.path.join(HERE, "libntx.so")
CHECK_SO = os.path.join(HERE, "libntx_check.so")  # the bounds-checked debug build (NTX_CHECK)
SOURCES = ["kernels.cu", "api.cu", "noalloc.cu", "persist.cu", "tiers.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr"]


def _newest_input():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "ntx.h")]
    return max(os.path.getmtime(f) for f in files)


def build(force: bool = False, verbose: bool = False, out: str = SO, defines=()) -> str:
    """Compile libntx.so (or a variant at `out` with extra -D definitions)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= _newest_input():
        return out
    objs = []
    procs = []
    for src in SOURCES:
        obj = out + "." + src.replace(".cu", ".o")
        cmd = [NVCC, *ARCH, *FLAGS, *["-D" + d for d in defines], "-I", INCLUDE, "-c", os.path.join(CSRC, src), "-o",
               obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        procs.append(subprocess.Popen(cmd))
        objs.append(obj)
    for p in procs:
        if p.wait() != 0:
            raise RuntimeError("nvcc failed")
    tmp = out + ".tmp"
    subprocess.check_call([NVCC, *ARCH, "-shared", "-o", tmp, *objs])
    os.replace(tmp, out)
    for o in objs:
        os.remove(o)
    return out


def build_check(force: bool = False) -> str:
    """The bounds-checked debug build (kernels check their buffer indices, see ntx_check_report)."""
    return build(force=force, out=CHECK_SO, defines=("NTX_CHECK",))


if __name__ == "__main__":
    import sys
    if "--check" in sys.argv:
        print(build_check(force="--force" in sys.argv))
    else:
        print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
