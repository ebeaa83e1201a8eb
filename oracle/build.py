"""Compile the CPU oracle (test infrastructure) into oracle/liboracle.so.

Plain gcc, -O2, no fast-math, no FMA contraction, so every fp32 operation in
the oracle is the single IEEE operation the source spells out.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bitnet_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def compile_source(src: str, out: str) -> str:
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, src, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    return compile_source(SRC, LIB)


if __name__ == "__main__":
    print(build(force=True))
