"""Build the CUDA library in-tree for sm_100a.

    python -m structured_sparse_attention_fibonacci_b200.build [--force] [--ptxas-v]

Compiles csrc/*.cu with nvcc (one object per source, in parallel) and links
them into two plain C-ABI shared libraries next to this file, which the Python
binding loads with ctypes:
  libsparse_attn.so         the library;
  libsparse_attn_bounds.so  the same sources compiled with SA_DEBUG_BOUNDS:
                            every staged row a kernel reads is checked against
                            the rows its shared-memory ring holds, and every
                            staging round against the ring's size; a violation
                            sets bit 1 of the device error word (no trap), so
                            the parity tests can run under it in place of a
                            memory checker.
"""
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libsparse_attn.so")
LIB_BOUNDS = os.path.join(HERE, "libsparse_attn_bounds.so")
OBJ_DIR = os.path.join(HERE, "_build")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
    "--expt-relaxed-constexpr",
]

VARIANTS = {LIB: [], LIB_BOUNDS: ["-DSA_DEBUG_BOUNDS"]}


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    deps += glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(nvcc, src, obj, extra, verbose):
    cmd = [nvcc, *NVCC_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    return obj


def build(force: bool = False, verbose: bool = False, extra=(), variants=None) -> str:
    """Compile the stale libraries (all with force); returns the main library's path."""
    nvcc = os.environ.get("NVCC", "nvcc")
    todo = [lib for lib in (variants or VARIANTS) if force or _stale(lib)]
    if not todo:
        return LIB
    os.makedirs(OBJ_DIR, exist_ok=True)
    jobs = []
    with cf.ThreadPoolExecutor(max_workers=max(1, min(16, os.cpu_count() or 1))) as ex:
        for lib in todo:
            tag = os.path.splitext(os.path.basename(lib))[0]
            objs = []
            for src in sources():
                obj = os.path.join(OBJ_DIR, f"{tag}.{os.path.basename(src)}.o")
                objs.append(obj)
                jobs.append(ex.submit(_compile, nvcc, src, obj, [*VARIANTS[lib], *extra], verbose))
            jobs.append((lib, objs))
        futures = [j for j in jobs if not isinstance(j, tuple)]
        for f in futures:
            f.result()
    for j in jobs:
        if isinstance(j, tuple):
            lib, objs = j
            tmp = lib + f".tmp{os.getpid()}"
            subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                                   *objs, "-o", tmp])
            os.replace(tmp, lib)
    return LIB


if __name__ == "__main__":
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []
    print(build(force="--force" in sys.argv or bool(extra), verbose=True, extra=extra))
