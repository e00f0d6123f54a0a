"""Build libfp4q.so (the C-ABI library) in-tree for sm_100a with nvcc."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(HERE)
ROOT = os.path.dirname(PKG)
SRCS = [os.path.join(HERE, "fp4q.cu"), os.path.join(HERE, "fp4q_gemm.cu")]
DEPS = SRCS + [os.path.join(HERE, "fp4q_device.cuh"), os.path.join(ROOT, "include", "fp4q.h")]
LIB = os.path.join(PKG, "libfp4q.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "--fmad=false", "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-v",
         "-I", os.path.join(ROOT, "include"), "-I", HERE, "-lcudart"]


def build(force: bool = False, verbose: bool = False, defines=()) -> str:
    if not force and os.path.exists(LIB) and all(os.path.getmtime(LIB) >= os.path.getmtime(d) for d in DEPS):
        return LIB
    cmd = [NVCC] + FLAGS + ["-D" + d for d in defines] + ["-o", LIB] + SRCS
    out = subprocess.run(cmd, capture_output=True, text=True)
    if out.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + out.stdout + out.stderr)
    if verbose:
        sys.stderr.write(out.stderr)
    return LIB


if __name__ == "__main__":
    defs = [a[2:] for a in sys.argv[1:] if a.startswith("-D")]
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, defines=defs))
