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
# The failure-path test library: the product sources built with the GEMM MMA thread's first wait
# treated as timed out (FP4Q_GEMM_FAIL_FIRST_WAIT); loaded only by tests/test_gpu_gemm_failure.py.
TEST_LIB = os.path.join(PKG, "libfp4q_failtest.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "--fmad=false", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-shared", "-Xptxas", "-v",
         "-I", os.path.join(ROOT, "include"), "-I", HERE, "-lcudart"]


def build(force: bool = False, verbose: bool = False, defines=(), out=LIB) -> str:
    if not force and os.path.exists(out) and all(os.path.getmtime(out) >= os.path.getmtime(d) for d in DEPS):
        return out
    cmd = [NVCC] + FLAGS + ["-D" + d for d in defines] + ["-o", out] + SRCS
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stderr)
    return out


def build_test_lib(force: bool = False) -> str:
    return build(force=force, defines=("FP4Q_GEMM_FAIL_FIRST_WAIT=1",), out=TEST_LIB)


if __name__ == "__main__":
    defs = [a[2:] for a in sys.argv[1:] if a.startswith("-D")]
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, defines=defs))
