"""Build the sm_100a shared library ``libmoe_epilogue.so`` in-tree with nvcc.

    python -m moe_expert_epilogue_b200.build [--force] [-v]

Each ``csrc/*.cu`` is compiled to an object for ``sm_100a`` only (no PTX for
other targets), then linked with the static CUDA runtime into one shared
library next to this file, so the library loads on any machine with an NVIDIA
driver and no CUDA toolkit.  The build needs no GPU.

Tuning builds: ``MOE_BUILD_DEFINES="NAME=VALUE ..."`` in the environment adds
``-DNAME=VALUE`` for the kernels' compile-time knobs (the ``MOE_*`` macros of
``csrc``).  The defines of the library on disk are kept in a stamp file beside
it, and the library counts as up to date only when they equal the
environment's, so ``MOE_BUILD_DEFINES=... python bench.py`` rebuilds with the
knobs and a later plain run rebuilds the defaults.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libmoe_epilogue.so")
STAMP = LIB + ".defines"

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
              "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build")
    return path


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def defines() -> list:
    """The tuning defines requested by MOE_BUILD_DEFINES (sorted), each
    NAME or NAME=VALUE with NAME a MOE_* macro and VALUE an integer."""
    out = []
    for d in os.environ.get("MOE_BUILD_DEFINES", "").split():
        name, _, value = d.partition("=")
        if not name.startswith("MOE_") or not name.replace("_", "").isalnum() or \
                (value and not value.lstrip("-").isdigit()):
            raise ValueError(f"MOE_BUILD_DEFINES: bad define {d!r} (want MOE_NAME=integer)")
        out.append(d)
    return sorted(out)


def built_defines() -> list:
    if not os.path.exists(STAMP):
        return []
    with open(STAMP) as f:
        return sorted(f.read().split())


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _deps()) and built_defines() == defines()


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    cc = nvcc()
    defs = defines()
    extra = ["-Xptxas", "-v"] if ptxas_info else []
    extra += [f"-D{d}" for d in defs]

    def compile_one(src):
        obj = os.path.join(BUILD, os.path.basename(src) + ".o")
        cmd = [cc, *ARCH, *NVCC_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        if verbose or ptxas_info:
            print(r.stderr, end="", flush=True)
        return obj

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, _sources()))
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [cc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    with open(STAMP, "w") as f:
        f.write(" ".join(defs))
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers / spills")
    a = ap.parse_args()
    print(build(force=a.force or a.ptxas_info, verbose=a.verbose, ptxas_info=a.ptxas_info))


if __name__ == "__main__":
    main()
