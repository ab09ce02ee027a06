"""Ahead-of-time build of the CUDA libraries for sm_100a (in tree):

* ``expert_offloaded_serving_b200/libftmoe.so`` from ``csrc/*.cu``
* ``synth/libftsynth.so`` (seeded input filler) from ``synth/pool.cu``

    python -m expert_offloaded_serving_b200.build
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _run(cmd: list[str]) -> None:
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("build failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)


def _stale(target: str, sources: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def build_lib(sources: list[str], out: str, deps: list[str], extra: list[str] | None = None, verbose=False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    objs = []
    jobs = []
    for src in sources:
        obj = os.path.join(BUILD, os.path.basename(out) + "." + os.path.basename(src) + ".o")
        objs.append(obj)
        if _stale(obj, [src] + deps):
            cmd = [nvcc()] + ARCH + FLAGS + (extra or []) + ["-c", src, "-o", obj]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
            jobs.append(cmd)
    with cf.ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        list(ex.map(_run, jobs))
    if jobs or _stale(out, objs):
        _run([nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", out] + objs)
    return out


def build(verbose: bool = False) -> list[str]:
    deps = glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))
    lib = build_lib(sorted(glob.glob(os.path.join(CSRC, "*.cu"))), os.path.join(PKG, "libftmoe.so"), deps,
                    verbose=verbose)
    syn = build_lib([os.path.join(ROOT, "synth", "pool.cu")], os.path.join(ROOT, "synth", "libftsynth.so"), [],
                    verbose=verbose)
    return [lib, syn]


if __name__ == "__main__":
    for p in build(verbose="-v" in sys.argv):
        print(p)
