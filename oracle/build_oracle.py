"""Build oracle/liboracle.so from fp8_oracle.cpp with the host C++ compiler.

    python -m oracle.build_oracle [--force]

Plain C++17, no CUDA: -O2 with -ffp-contract=off and no fast-math, so every
float and double operation in the oracle is the IEEE operation written. The
library is rebuilt whenever the hash of the source and the flags differs from
the one recorded next to it.
"""

import argparse
import hashlib
import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fp8_oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")
STAMP = LIB + ".stamp"
FLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
         "-pthread"]


def _compiler():
    for c in (os.environ.get("CXX"), "g++", "c++", "clang++"):
        if c and shutil.which(c):
            return shutil.which(c)
    raise RuntimeError("no C++ compiler found (g++)")


def _digest():
    h = hashlib.sha256()
    with open(SRC, "rb") as f:
        h.update(f.read())
    h.update(" ".join(FLAGS).encode())
    return h.hexdigest()


def up_to_date():
    if not (os.path.exists(LIB) and os.path.exists(STAMP)):
        return False
    with open(STAMP) as f:
        return f.read().strip() == _digest()


def build(force=False):
    if not force and up_to_date():
        return LIB
    tmp = LIB + ".tmp"
    r = subprocess.run([_compiler()] + FLAGS + [SRC, "-o", tmp], capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("oracle build failed:\n" + r.stdout + r.stderr)
    os.replace(tmp, LIB)
    with open(STAMP, "w") as f:
        f.write(_digest() + "\n")
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    print(build(force=ap.parse_args().force))
