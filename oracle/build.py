"""Build the C++ oracle (oracle/liblsa_oracle.so) with the host compiler.

    python -m oracle.build

Test infrastructure: the library is the CPU oracle the tests and the bench's
CPU legs compare against. Built in-tree, rebuilt when the source is newer.
Compiled with -ffp-contract=off and without -ffast-math, so every float64 sum
runs in the order the source writes it.
"""
from __future__ import annotations

import fcntl
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "lsa_oracle.cpp")
LIB = os.path.join(HERE, "liblsa_oracle.so")
FLAGS = ["-O3", "-std=c++17", "-fPIC", "-shared", "-pthread", "-ffp-contract=off", "-fno-fast-math", "-Wall"]


def _cxx() -> str:
    for cand in (os.environ.get("CXX"), shutil.which("g++"), shutil.which("c++")):
        if cand:
            return cand
    raise RuntimeError("no C++ compiler found (g++)")


def stale() -> bool:
    return not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(SRC), os.path.getmtime(__file__))


def build(force: bool = False) -> str:
    """Compile the oracle if it is missing or older than its source."""
    if not force and not stale():
        return LIB
    with open(os.path.join(HERE, ".build.lock"), "w") as lock:
        fcntl.flock(lock, fcntl.LOCK_EX)          # one builder at a time (parallel test workers)
        if not force and not stale():
            return LIB
        tmp = f"{LIB}.{os.getpid()}.tmp"
        r = subprocess.run([_cxx(), *FLAGS, "-o", tmp, SRC], capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("building the C++ oracle failed")
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
