"""Build of the C++ oracle (test infrastructure): oracle/liboracle.so from
oracle/ft_oracle.cpp with g++ (fp64, no fast-math, OpenMP for the timed
multi-threaded CPU baseline).

    python -m oracle.build
"""
from __future__ import annotations

import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ft_oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")


def build() -> str:
    if os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cands = [os.environ.get("CXX"), "/usr/bin/g++", shutil.which("g++")]
    errors = []
    cxxs = [c for c in dict.fromkeys(cands) if c and os.path.exists(c)]
    # OpenMP when a toolchain has it (the multi-threaded CPU baseline), else serial
    for omp in (["-fopenmp"], []):
        for cxx in cxxs:
            cmd = [cxx, "-O2", "-std=c++17", "-fPIC", "-shared", *omp, "-fvisibility=hidden", "-o", LIB, SRC]
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode == 0:
                return LIB
            errors.append(" ".join(cmd) + "\n" + r.stdout + r.stderr)
    raise RuntimeError("oracle build failed:\n" + "\n".join(errors))


if __name__ == "__main__":
    print(build())
