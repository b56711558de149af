"""Builds the CPU oracle shared library (oracle/libehref.so) with g++.

Test infrastructure: the oracle is only loaded by the tests, the smoke check
and the CPU-baseline leg of the benchmark.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libehref.so")


def build(force: bool = False) -> str:
    srcs = [os.path.join(HERE, f) for f in ("ehref.cpp", "zfref.cpp")]
    deps = srcs + [os.path.join(HERE, f) for f in ("ehref.h", "zfref.h")]
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(f) for f in deps)):
        return LIB
    tmp = LIB + ".tmp"
    cmd = ["g++", "-std=c++17", "-O2", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-o", tmp, *srcs]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
