"""Build the fp64 oracle library (test infrastructure): oracle/liboracle.so.

Plain gcc, -O3, OpenMP over heads, no CPU-specific instructions, so the
library built here runs on any x86-64 host.
"""
from __future__ import annotations

import subprocess
from pathlib import Path

HERE = Path(__file__).resolve().parent


def build() -> Path:
    src = HERE / "kata_oracle.c"
    out = HERE / "liboracle.so"
    tmp = HERE / "liboracle.so.tmp"
    cmd = ["gcc", "-std=c11", "-O3", "-fopenmp", "-fPIC", "-shared", "-fvisibility=hidden",
           "-Wall", "-Wextra", "-o", str(tmp), str(src), "-lm"]
    subprocess.run(cmd, check=True)
    tmp.replace(out)
    return out


if __name__ == "__main__":
    print(build())
