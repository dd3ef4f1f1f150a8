"""Compile the oracle's plain-C source into a shared library.

Test infrastructure only: the oracle is built for the test suite, the smoke
check and the CPU-baseline leg of the benchmark.  ``plant`` selects one of the
deliberately wrong variants that the test suite uses to show that its pins
catch mistakes; the default (0) is the oracle proper.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "prism_ref.c")


def library_path(plant: int = 0, out_dir: str | None = None) -> str:
    name = "libprism_ref.so" if plant == 0 else f"libprism_ref_plant{plant}.so"
    return os.path.join(out_dir or HERE, name)


def build(plant: int = 0, out_dir: str | None = None, force: bool = False) -> str:
    """Build the oracle library (``gcc -O2 -fopenmp``, strict IEEE double)."""
    out = library_path(plant, out_dir)
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(SOURCE)):
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c99", "-O2", "-fno-fast-math", "-ffp-contract=off",
           "-fopenmp", "-shared", "-fPIC", f"-DPRISM_REF_PLANT={int(plant)}",
           SOURCE, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force=True))
