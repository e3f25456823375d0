"""Build the CPU oracle (TEST INFRASTRUCTURE ONLY) into oracle/libtk_oracle.so.

Flags: -O2 for speed, -ffp-contract=off so the compiler never fuses a multiply and an add on
its own, no -ffast-math so every fp32 operation stays one IEEE round-to-nearest operation.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libtk_oracle.so")
SRC = os.path.join(HERE, "tk_oracle.cpp")
HDR = os.path.join(HERE, "tk_oracle.h")


def build_variant(plant: int, out_path: str) -> str:
    """Compile the oracle with planted mistake number `plant` (see TKO_PLANT in tk_oracle.cpp)
    into out_path; used only by the mutation test."""
    cmd = ["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           f"-DTKO_PLANT={int(plant)}", "-o", out_path, SRC]
    subprocess.run(cmd, check=True)
    return out_path


def build_oracle(force: bool = False) -> str:
    """Compile the oracle if the library is missing or older than its sources; return its path."""
    if not force and os.path.exists(LIB):
        lib_m = os.path.getmtime(LIB)
        if lib_m >= os.path.getmtime(SRC) and lib_m >= os.path.getmtime(HDR):
            return LIB
    cmd = ["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
           "-shared", "-Wall", "-Wextra", "-o", LIB + ".tmp", SRC]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build_oracle(force="--force" in sys.argv))
