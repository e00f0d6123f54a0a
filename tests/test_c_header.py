"""include/fp4q.h is a plain C header and libfp4q.so a plain C ABI: a C11 program that includes
the header, links the library and calls entry points that need no GPU (sizes, status strings,
argument checks that return before any launch) compiles without warnings and runs."""
import os
import shutil
import subprocess

import pytest

import fp4_block_scaled_nvfp4_b200 as fq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "fp4q.h"

int main(void) {
    if (fp4q_workspace_bytes() < 16) return 1;
    /* row-major and tiled scale sizes of a 130 x 96 NVFP4 tensor */
    if (fp4q_scale_bytes(130, 96, FP4Q_NVFP4, 0) != 130 * 6) return 2;
    if (fp4q_scale_bytes(130, 96, FP4Q_NVFP4, FP4Q_F_SCALE_TILED) != 2 * 2 * 512) return 3;
    if (fp4q_scale_bytes(130, 96, FP4Q_MXFP4, 0) != 130 * 3) return 4;
    if (strcmp(fp4q_status_string(FP4Q_OK), "ok") != 0) return 5;
    /* argument checks return before any launch */
    if (fp4q_quantize(NULL, FP4Q_IN_BF16, 4, 64, 64, FP4Q_NVFP4, FP4Q_SWEEP_MSE, NULL, NULL, NULL, NULL,
                      NULL, 0u, NULL) != FP4Q_ERR_INVALID_ARG) return 6;
    if (fp4q_quantize((const void*)0x10000, FP4Q_IN_BF16, 4, 60, 64, FP4Q_NVFP4, FP4Q_SWEEP_MSE, NULL,
                      (uint8_t*)0x10000, (uint8_t*)0x10000, (float*)0x10000, (void*)0x10000, 0u, NULL)
        != FP4Q_ERR_SHAPE) return 7;
    if (fp4q_nvfp4_gemm(NULL, NULL, NULL, NULL, NULL, NULL, 100, 128, 256, NULL, 128, NULL, NULL)
        != FP4Q_ERR_SHAPE) return 8;
    if (fp4q_encode(NULL, 8, 7, NULL, NULL) != FP4Q_ERR_INVALID_ARG) return 9;
    if (fp4q_last_launch_count() != 0) return 10;
    printf("ok\n");
    return 0;
}
"""


def test_header_compiles_as_c_and_the_abi_links(tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    lib = fq.LIB_PATH
    if not os.path.exists(lib):
        pytest.skip("library not built")
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    cmd = [gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
           lib, "-Wl,-rpath," + os.path.dirname(lib), "-o", str(exe)]
    out = subprocess.run(cmd, capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip() == "ok", (run.returncode, run.stdout, run.stderr)


LAYOUT = r"""
#include <stddef.h>
#include <stdio.h>
#include "fp4q.h"

int main(void) {
    fp4q_tensor t[2];
    memset(t, 0, sizeof t);
    printf("%zu %zu %zu %zu %zu %zu %zu %zu %zu\n", sizeof(fp4q_tensor), offsetof(fp4q_tensor, x),
           offsetof(fp4q_tensor, rows), offsetof(fp4q_tensor, cols), offsetof(fp4q_tensor, ld),
           offsetof(fp4q_tensor, importance), offsetof(fp4q_tensor, codes), offsetof(fp4q_tensor, scales),
           offsetof(fp4q_tensor, global_scale));
    /* a batch of empty tensors returns before anything runs */
    t[0].cols = 64; t[0].ld = 64; t[1].rows = 3;
    return fp4q_quantize_batch(2, t, FP4Q_IN_BF16, FP4Q_NVFP4, FP4Q_SWEEP_MSE, (void*)0x10000, 0u, NULL) == FP4Q_OK &&
           fp4q_last_launch_count() == 0 ? 0 : 1;
}
"""


def test_batch_descriptor_layout_matches_the_binding(tmp_path):
    # the binding's ctypes fp4q_tensor must have the header struct's size and field offsets
    import ctypes as C
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    lib = fq.LIB_PATH
    if not os.path.exists(lib):
        pytest.skip("library not built")
    src = tmp_path / "layout.c"
    src.write_text("#include <string.h>\n" + LAYOUT)
    exe = tmp_path / "layout"
    cmd = [gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
           lib, "-Wl,-rpath," + os.path.dirname(lib), "-o", str(exe)]
    out = subprocess.run(cmd, capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, (run.stdout, run.stderr)
    got = [int(v) for v in run.stdout.split()]
    T = fq._Tensor
    want = [C.sizeof(T)] + [getattr(T, f).offset for f in
                            ("x", "rows", "cols", "ld", "importance", "codes", "scales", "global_scale")]
    assert got == want
