"""Build the fp64 C++ oracle (``oracle/liboracle_f64.so``) with g++.

TEST INFRASTRUCTURE ONLY: the library is loaded by the tests, the smoke check
and the benchmark's host baseline, never by the CUDA library.

    python -m oracle.build [--force]

Plain C++17, host threads through std::thread, no BLAS.  -ffp-contract=off
keeps every multiply and add of the method's steps a separate IEEE operation
(the matrix product's fused multiply-adds are written out explicitly).
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "liboracle_f64.so")
FLAGS = ["-O3", "-std=c++17", "-fPIC", "-shared", "-pthread", "-ffp-contract=off", "-fno-fast-math"]


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cpp"))


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(os.path.join(CSRC, f)) > t for f in os.listdir(CSRC))


def build(force: bool = False) -> str:
    if not force and not stale():
        return LIB
    cxx = shutil.which("g++") or shutil.which("c++")
    if not cxx:
        raise RuntimeError("g++ not found: the C++ oracle needs a host C++ compiler")
    tmp = f"{LIB}.{os.getpid()}.tmp"
    cmd = [cxx] + FLAGS + ["-I" + CSRC] + sources() + ["-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"oracle build failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args(argv)
    print(build(force=a.force))
    return 0


if __name__ == "__main__":
    sys.exit(main())
