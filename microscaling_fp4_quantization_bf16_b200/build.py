"""Builds libfp4q.so (the C-ABI CUDA library) in-tree for sm_100a.

Each .cu under csrc/ is compiled separately (in parallel) with nvcc, then
linked into one shared library with the CUDA runtime linked statically, so the
library only needs the NVIDIA driver at run time. Floating-point flags keep
every operation IEEE round-to-nearest-even with no FMA contraction, no
flush-to-zero and correctly rounded division, which the bit-exact results
depend on.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libfp4q.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ARCH + ["-O3", "-std=c++17", "-lineinfo", "-fmad=false", "-prec-div=true",
                 "-prec-sqrt=true", "-ftz=false", "-Xcompiler", "-fPIC,-O2",
                 "-I" + INCLUDE, "-I" + CSRC]


def _cutlass_include() -> list[str]:
    """CUTLASS/CuTe header trees (vendored with flashinfer in this image),
    used by the GEMM sources only."""
    import importlib.util
    spec = importlib.util.find_spec("flashinfer")
    if spec is None or not spec.submodule_search_locations:
        raise RuntimeError("CUTLASS headers not found (flashinfer's vendored copy)")
    base = os.path.join(list(spec.submodule_search_locations)[0], "data", "cutlass")
    inc = [os.path.join(base, "include"), os.path.join(base, "tools", "util", "include")]
    if not os.path.exists(os.path.join(inc[0], "cutlass", "cutlass.h")):
        raise RuntimeError(f"CUTLASS headers not found under {base}")
    return ["-I" + d for d in inc] + ["--expt-relaxed-constexpr"]


def _flags_for(src: str) -> list[str]:
    name = os.path.basename(src)
    return CFLAGS + (_cutlass_include() if name.startswith("gemm_") else [])


def _nvcc() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found: the CUDA library cannot be built")
    return p


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(
        os.path.join(CSRC, "*.h")) + [os.path.join(INCLUDE, "fp4q.h"), __file__]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in _deps())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    nvcc = _nvcc()
    os.makedirs(BUILD_DIR, exist_ok=True)
    srcs = _sources()
    objs = [os.path.join(BUILD_DIR, os.path.basename(s)[:-3] + ".o") for s in srcs]

    def compile_one(pair):
        src, obj = pair
        cmd = [nvcc] + _flags_for(src) + ["-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        if verbose and r.stderr:
            print(r.stderr, file=sys.stderr)
        return obj

    with ThreadPoolExecutor(max_workers=max(1, min(len(srcs), os.cpu_count() or 4))) as ex:
        list(ex.map(compile_one, zip(srcs, objs)))
    tmp = LIB + ".tmp"
    cmd = [nvcc] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
