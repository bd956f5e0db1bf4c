"""In-tree build of the native libraries.

* ``libeta.so``   — the CUDA library (csrc/*.cu + csrc/api.cpp), sm_100a only,
  exported through the C ABI declared in ``include/eta.h``.
* ``synth/libsynth.so`` — the seeded input generator (plain C).

Run ``python -m learned_block_sparse_b200._build`` or call ``build_all()``.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
ETA_LIB = os.path.join(PKG, "libeta.so")
SYNTH_SRC = os.path.join(PKG, "synth", "synth.c")
SYNTH_LIB = os.path.join(PKG, "synth", "libsynth.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    # IEEE division and square root: the screening decisions depend on them.
    "-prec-div=true", "-prec-sqrt=true", "-fmad=true",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(target: str, sources) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def build_synth(force: bool = False) -> str:
    if force or _stale(SYNTH_LIB, [SYNTH_SRC]):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", SYNTH_SRC,
                               "-o", SYNTH_LIB + ".tmp", "-lm", "-lpthread"])
        os.replace(SYNTH_LIB + ".tmp", SYNTH_LIB)
    return SYNTH_LIB


def eta_sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def build_eta(force: bool = False, verbose: bool = False) -> str:
    srcs = eta_sources()
    deps = srcs + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) \
        + glob.glob(os.path.join(INCLUDE, "*.h"))
    if not (force or _stale(ETA_LIB, deps)):
        return ETA_LIB
    nvcc = _nvcc()
    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    procs = []
    for s in srcs:
        o = os.path.join(objdir, os.path.basename(s) + ".o")
        cmd = [nvcc, *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-c", s, "-o", o]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        procs.append((subprocess.Popen(cmd), cmd))
        objs.append(o)
    for p, cmd in procs:
        if p.wait() != 0:
            raise RuntimeError("compile failed: " + " ".join(cmd))
    subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                           "-Xcompiler", "-fPIC", *objs, "-o", ETA_LIB + ".tmp"])
    os.replace(ETA_LIB + ".tmp", ETA_LIB)
    return ETA_LIB


def build_all(force: bool = False) -> None:
    build_synth(force)
    build_eta(force)


if __name__ == "__main__":
    build_all(force="--force" in sys.argv)
    print(ETA_LIB)
