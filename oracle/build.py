"""Builds the float64 CPU oracle (attn_oracle.cpp) into a shared library with g++.

Test infrastructure only. ``plant`` compiles a variant with one deliberate
mistake (ORACLE_PLANT=<n>) so the pin tests can show that they would catch it.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "attn_oracle.cpp")
OUT_DIR = os.path.join(HERE, "_build")


def library_path(plant: int = 0) -> str:
    name = "liboracle.so" if not plant else f"liboracle_plant{plant}.so"
    return os.path.join(OUT_DIR, name)


def build_oracle(plant: int = 0, force: bool = False) -> str:
    out = library_path(plant)
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(SRC):
        return out
    os.makedirs(OUT_DIR, exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread", "-fno-fast-math",
           f"-DORACLE_PLANT={int(plant)}", SRC, "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build_oracle(force="--force" in sys.argv))
