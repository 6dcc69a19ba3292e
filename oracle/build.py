"""Compile the CPU oracle (plain C, fp64) into oracle/liboracle.so.

No fast-math and no FMA contraction, so the fp32 steps of the quantisers are IEEE-exact."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "hcl_oracle.c")
OUT = os.path.join(HERE, "liboracle.so")


def build_oracle(force: bool = False, src: str = SRC, out: str = OUT) -> str:
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    tmp = out + ".tmp"
    cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-shared", "-fPIC", "-Wall", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build_oracle(force=True))
