"""Builds the C++ reference (oracle/bq_ref.cpp) into oracle/libbqref.so with g++: -O2, OpenMP,
no fused multiply-add. Test infrastructure: only the tests, the smoke check and the bench's CPU
legs load the result."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bq_ref.cpp")
OUT = os.path.join(HERE, "libbqref.so")
# the system compiler (its OpenMP runtime is installed); an override may lack libgomp, in which
# case the library is built without OpenMP and runs on one thread
CXX = os.environ.get("BQREF_CXX") or ("/usr/bin/g++" if os.path.exists("/usr/bin/g++") else "g++")
FLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fPIC", "-shared"]


def up_to_date() -> bool:
    return os.path.exists(OUT) and os.path.getmtime(OUT) >= os.path.getmtime(SRC)


def build(force: bool = False) -> str:
    if force or not up_to_date():
        tmp = OUT + f".{os.getpid()}.tmp"
        r = subprocess.run([CXX, *FLAGS, "-fopenmp", "-o", tmp, SRC], capture_output=True, text=True)
        if r.returncode != 0:
            subprocess.run([CXX, *FLAGS, "-o", tmp, SRC], check=True)
        os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    import sys
    print(build(force="--force" in sys.argv))
