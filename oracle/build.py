"""Build the CPU oracle (test infrastructure only) into oracle/_oracle.so.

The same C source is compiled twice, once in double precision (suffix _f64,
the parity reference) and once in single precision (suffix _f32, the plain
CPU baseline), then linked into one shared library.  No fast-math and no FMA
contraction, so every operation is the plain IEEE one the source spells out.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle_attn.c")
LIB = os.path.join(HERE, "_oracle.so")

CFLAGS = ["-O2", "-fPIC", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
          "-std=c11", "-Wall", "-Wextra", "-Wno-unused-parameter"]


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)
            and os.path.getmtime(LIB) >= os.path.getmtime(__file__)):
        return LIB
    objs = []
    for real, suffix in (("double", "_f64"), ("float", "_f32")):
        obj = os.path.join(HERE, f"_oracle{suffix}.o")
        subprocess.check_call(["gcc", *CFLAGS, f"-DORACLE_REAL={real}",
                               f"-DORACLE_SUFFIX={suffix}", "-c", SRC, "-o", obj])
        objs.append(obj)
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-shared", "-fopenmp", *objs, "-o", tmp, "-lm"])
    os.replace(tmp, LIB)
    for o in objs:
        os.remove(o)
    return LIB


def build_variant(source_text: str, out_dir: str, name: str) -> str:
    """Compile a modified copy of the oracle source (used by the mutation
    tests, which plant a mistake and check that a pin catches it)."""
    src = os.path.join(out_dir, f"{name}.c")
    with open(src, "w") as f:
        f.write(source_text)
    objs = []
    for real, suffix in (("double", "_f64"), ("float", "_f32")):
        obj = os.path.join(out_dir, f"{name}{suffix}.o")
        subprocess.check_call(["gcc", *CFLAGS, f"-DORACLE_REAL={real}",
                               f"-DORACLE_SUFFIX={suffix}", "-c", src, "-o", obj])
        objs.append(obj)
    lib = os.path.join(out_dir, f"{name}.so")
    subprocess.check_call(["gcc", "-shared", "-fopenmp", *objs, "-o", lib, "-lm"])
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
