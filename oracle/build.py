"""Builds the C++ oracle (oracle/pi_oracle.cpp) into oracle/libpi_oracle.so.

Test infrastructure.  Plain g++ with IEEE fp64 semantics kept intact: no
fast-math, no fused multiply-add contraction, no threads.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "pi_oracle.cpp")
LIB = os.path.join(HERE, "libpi_oracle.so")
FLAGS = ["-std=c++17", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def compile_source(src: str, out: str) -> str:
    """Compile one C++ oracle source file to a shared library at `out`."""
    tmp = out + f".tmp{os.getpid()}"
    cmd = [os.environ.get("CXX", "g++"), *FLAGS, "-o", tmp, src]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"oracle build failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    os.replace(tmp, out)
    return out


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in (SRC, os.path.abspath(__file__)))


def build(force: bool = False) -> str:
    if force or not up_to_date():
        compile_source(SRC, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
