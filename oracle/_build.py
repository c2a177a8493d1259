"""Builds the CPU oracle (plain C, OpenMP) in place as liboracle_beam_moe.so.

Compiled at -O2 for the baseline x86-64 target, with no tuning for speed.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "liboracle_beam_moe.so")
SRCS = [os.path.join(HERE, "beam_moe_oracle.c"), os.path.join(HERE, "beam_moe_oracle.h")]


def build(force=False):
    stale = not os.path.exists(LIB) or any(
        os.path.getmtime(s) > os.path.getmtime(LIB) for s in SRCS)
    if force or stale:
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               SRCS[0], "-o", LIB + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
