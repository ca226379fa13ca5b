"""Compile the plain C oracle (oracle/lora_oracle_c.c) into
oracle/liblora_oracle.so with gcc.

TEST INFRASTRUCTURE ONLY: the library is the checker, not the product.

    python -m oracle.build_oracle [--force]
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "lora_oracle_c.c")
LIB = os.path.join(HERE, "liblora_oracle.so")


def up_to_date() -> bool:
    return os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC)


def build(force: bool = False, quiet: bool = True) -> str:
    if not force and up_to_date():
        return LIB
    cc = os.environ.get("CC") or shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        raise RuntimeError("no C compiler (gcc) found to build the oracle")
    tmp = LIB + f".{os.getpid()}.tmp"
    # -O2 without -ffast-math: every floating-point operation stays as written
    cmd = [cc, "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", SRC, "-o", tmp, "-lm"]
    if not quiet:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, quiet=False))
