"""Compile the fp64 oracle (plain C, OpenMP) into oracle/liboracle.so.

Test infrastructure: nothing on the GPU library's path links or loads the result.
No fast-math and no floating-point contraction, so every operation is the single
IEEE double operation written in the source.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def build(src: str = os.path.join(HERE, "oracle.c"),
          out: str = os.path.join(HERE, "liboracle.so")) -> str:
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-fno-fast-math", "-ffp-contract=off", src, "-o", out + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build())
