"""Compile the fp64 row-normalization oracle into ``oracle/liboracle.so``.

Test infrastructure: the product library never links or loads the result.
Plain ``-O2`` with IEEE semantics (no ``-ffast-math``, no FMA contraction),
OpenMP only to spread independent rows over host threads.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "rownorm_oracle.c")
TARGET = os.path.join(HERE, "liboracle.so")


def compile_source(source: str, target: str) -> str:
    cmd = ["gcc", "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off",
           "-fopenmp", "-fPIC", "-shared", source, "-o", target + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(target + ".tmp", target)
    return target


def build(force: bool = False) -> str:
    if (not force and os.path.exists(TARGET)
            and os.path.getmtime(TARGET) >= os.path.getmtime(SOURCE)):
        return TARGET
    return compile_source(SOURCE, TARGET)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
