"""Compile the CPU oracle (plain C, OpenMP) into two shared libraries.

liborc_f64.so computes in double (parity), liborc_f32.so in float (the timed
CPU baseline). Test infrastructure only.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "rlt_oracle.c")
OUT_DIR = os.path.join(HERE, "_build")


def lib_path(precision: str) -> str:
    return os.path.join(OUT_DIR, f"liborc_{precision}.so")


def build(force: bool = False, extra_flags=()) -> None:
    os.makedirs(OUT_DIR, exist_ok=True)
    for prec, ctype in (("f64", "double"), ("f32", "float")):
        out = lib_path(prec)
        if (not force and os.path.exists(out)
                and os.path.getmtime(out) >= os.path.getmtime(SRC)):
            continue
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11",
               "-ffp-contract=off", f"-DORC_REAL={ctype}", *extra_flags,
               SRC, "-o", out + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(out + ".tmp", out)


if __name__ == "__main__":
    build(force="--force" in sys.argv)
