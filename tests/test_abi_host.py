"""Host-side checks of the C-ABI library (no GPU needed): the library loads, exports every
function include/fp4q.h declares, and rejects bad arguments before launching anything."""
import ctypes as C
import os
import re

import pytest

import fp4_block_scaled_nvfp4_b200 as fq

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fp4q.h")


def declared_functions():
    src = open(HDR).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fp4q_\w+)\s*\(", src)))


def test_header_declarations_match_binding():
    assert declared_functions() == sorted(fq.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = fq.lib()
    for name in declared_functions():
        assert hasattr(L, name), name


def test_scale_bytes():
    # row-major: rows * cols/B; tiled: padded to 128-row x 4-column tiles of 512 bytes
    assert fq.scale_bytes(256, 1024, "nvfp4") == 256 * 64
    assert fq.scale_bytes(256, 1024, "nvfp4", tiled=True) == 256 * 64
    assert fq.scale_bytes(100, 48, "nvfp4", tiled=True) == 128 * 4          # 3 scale columns -> 4
    assert fq.scale_bytes(129, 80, "nvfp4", tiled=True) == 256 * 8          # 5 scale columns -> 8
    assert fq.scale_bytes(300, 8192, "mxfp4", tiled=True) == 384 * 256
    assert fq.scale_bytes(0, 64, "mxfp4", tiled=True) == 0
    L = fq.lib()
    assert L.fp4q_scale_bytes(4, 24, 0, 0) == -1 and L.fp4q_scale_bytes(4, 32, 7, 0) == -1


def test_gemm_rejects_before_launch():
    L = fq.lib()
    F = FAKE
    call = lambda M, N, K, ldd=None, **kw: L.fp4q_nvfp4_gemm(kw.get("a", F), F, F, F, F, F, M, N, K,
                                                             kw.get("d", F), N if ldd is None else ldd,
                                                             kw.get("ws", F), None)
    assert call(100, 128, 256) == fq.ERR_SHAPE          # M % 128
    assert call(128, 64, 256) == fq.ERR_SHAPE           # N % 128
    assert call(128, 128, 128) == fq.ERR_SHAPE          # K % 256
    assert call(128, 128, 256, ldd=64) == fq.ERR_SHAPE  # ldd < N
    assert call(128, 128, 256, a=None) == fq.ERR_INVALID_ARG
    assert call(128, 128, 256, ws=None) == fq.ERR_INVALID_ARG
    assert call(128, 128, 256, d=F + 4) == fq.ERR_ALIGNMENT
    assert call(128, 128, 256, ldd=130) == fq.ERR_ALIGNMENT
    assert call(0, 128, 256, a=None, d=None, ws=None) == fq.OK and L.fp4q_last_launch_count() == 0
    # the MXFP4 form: the same checks, no tensor scales
    mx = lambda M, N, K, ldd=None, **kw: L.fp4q_mxfp4_gemm(kw.get("a", F), F, F, kw.get("bs", F), M, N, K,
                                                           kw.get("d", F), N if ldd is None else ldd,
                                                           kw.get("ws", F), None)
    assert mx(100, 128, 256) == fq.ERR_SHAPE
    assert mx(128, 128, 384) == fq.ERR_SHAPE
    assert mx(128, 128, 256, a=None) == fq.ERR_INVALID_ARG
    assert mx(128, 128, 256, bs=None) == fq.ERR_INVALID_ARG
    assert mx(128, 128, 256, d=F + 8) == fq.ERR_ALIGNMENT
    assert mx(0, 128, 256, a=None, d=None, ws=None) == fq.OK and L.fp4q_last_launch_count() == 0


def test_encode_rejects_before_launch():
    L = fq.lib()
    F = FAKE
    assert L.fp4q_encode(F, 8, 2, F, None) == fq.ERR_INVALID_ARG      # unknown kind
    assert L.fp4q_encode(F, -1, 0, F, None) == fq.ERR_SHAPE
    assert L.fp4q_encode(F, 1 << 41, 1, F, None) == fq.ERR_SHAPE
    assert L.fp4q_encode(None, 8, 0, F, None) == fq.ERR_INVALID_ARG
    assert L.fp4q_encode(F, 8, 0, None, None) == fq.ERR_INVALID_ARG
    assert L.fp4q_encode(F + 4, 8, 0, F, None) == fq.ERR_ALIGNMENT    # x must be 16-byte aligned
    assert L.fp4q_encode(F, 8, 1, F + 2, None) == fq.ERR_ALIGNMENT    # out must be 4-byte aligned
    assert L.fp4q_encode(None, 0, 0, None, None) == fq.OK and L.fp4q_last_launch_count() == 0


def test_status_strings_and_workspace():
    assert fq.status_string(0) == "ok"
    for rc in range(1, 6):
        assert fq.status_string(rc) and fq.status_string(rc) != "unknown status"
    assert fq.status_string(99) == "unknown status"
    assert fq.workspace_bytes() >= 16


FAKE = 0x10000   # 16-byte aligned non-null stand-in; validation rejects before any use


@pytest.mark.parametrize("args,rc", [
    # x, dtype, rows, cols, ld, fmt, obj, imp, codes, scales, gs, ws, flags
    ((FAKE, 1, 4, 24, 24, 0, 2, None, FAKE, FAKE, FAKE, FAKE, 0), fq.ERR_SHAPE),        # cols % 16
    ((FAKE, 1, 4, 32, 16, 0, 2, None, FAKE, FAKE, FAKE, FAKE, 0), fq.ERR_SHAPE),        # ld < cols
    ((FAKE, 1, -1, 32, 32, 0, 2, None, FAKE, FAKE, FAKE, FAKE, 0), fq.ERR_SHAPE),       # rows < 0
    ((FAKE, 1, 4, 48, 48, 2, 0, None, FAKE, FAKE, None, FAKE, 0), fq.ERR_SHAPE),        # MX cols % 32
    ((FAKE, 7, 4, 32, 32, 0, 2, None, FAKE, FAKE, FAKE, FAKE, 0), fq.ERR_INVALID_ARG),  # dtype
    ((FAKE, 1, 4, 32, 32, 5, 2, None, FAKE, FAKE, FAKE, FAKE, 0), fq.ERR_INVALID_ARG),  # fmt
    ((FAKE, 1, 4, 32, 32, 0, 9, None, FAKE, FAKE, FAKE, FAKE, 0), fq.ERR_INVALID_ARG),  # objective
    ((FAKE, 1, 4, 32, 32, 0, 3, None, FAKE, FAKE, FAKE, FAKE, 0), fq.ERR_INVALID_ARG),  # WMSE w/o weights
    ((None, 1, 4, 32, 32, 0, 2, None, FAKE, FAKE, FAKE, FAKE, 0), fq.ERR_INVALID_ARG),  # null x
    ((FAKE, 1, 4, 32, 32, 0, 2, None, FAKE, FAKE, None, FAKE, 0), fq.ERR_INVALID_ARG),  # null S
    ((FAKE, 1, 4, 32, 32, 0, 2, None, FAKE, FAKE, FAKE, None, 0), fq.ERR_INVALID_ARG),  # null workspace
    ((FAKE + 8, 1, 4, 32, 32, 0, 2, None, FAKE, FAKE, FAKE, FAKE, 0), fq.ERR_ALIGNMENT),  # x misaligned
    ((FAKE, 1, 4, 32, 36, 0, 2, None, FAKE, FAKE, FAKE, FAKE, 0), fq.ERR_ALIGNMENT),    # row pitch 72 B
    ((FAKE, 1, 4, 32, 32, 0, 2, None, FAKE + 4, FAKE, FAKE, FAKE, 0), fq.ERR_ALIGNMENT),  # codes
    ((FAKE, 1, 4, 32, 32, 0, 3, FAKE + 4, FAKE, FAKE, FAKE, FAKE, 0), fq.ERR_ALIGNMENT),  # weights
    ((FAKE, 1, 4, 32, 32, 0, 2, None, FAKE, FAKE, FAKE, FAKE, 0x100), fq.ERR_INVALID_ARG),  # unknown flag
    ((FAKE, 1, 4, 32, 32, 1, 0, None, FAKE, FAKE, FAKE, FAKE, 0x80), fq.ERR_UNSUPPORTED),  # tiled scales, IF4
    ((FAKE, 1, 4, 32, 32, 2, 0, None, FAKE, FAKE, None, FAKE, 1), fq.ERR_INVALID_ARG),  # MX with given S
    ((FAKE, 1, 4, 32, 32, 0, 2, None, FAKE, FAKE, FAKE, FAKE, 0x40), fq.ERR_UNSUPPORTED),  # IF4 sweep, NVFP4
    ((FAKE, 1, 4, 64, 64, 2, 0, None, FAKE, FAKE, None, FAKE, 0x40), fq.ERR_UNSUPPORTED),  # IF4 sweep, MXFP4
    ((FAKE, 1, 4, 32, 32, 0, 2, None, FAKE, FAKE, FAKE, FAKE, 0x20), fq.ERR_UNSUPPORTED),  # MX sweep, NVFP4
    ((FAKE, 1, 4, 32, 32, 2, 0, None, FAKE, FAKE, None, FAKE, 0x22), fq.ERR_INVALID_ARG),  # MX sweep + OCP floor
    ((None, 1, 0, 32, 32, 2, 0, None, None, None, None, None, 0x20), fq.OK),             # MX sweep, empty
    ((FAKE, 1, 4, 32, 32, 0, 2, None, FAKE, FAKE, FAKE, FAKE, 0x10), fq.ERR_UNSUPPORTED),  # 32-point rotation, NVFP4
    ((FAKE, 1, 4, 64, 64, 2, 0, None, FAKE, FAKE, None, FAKE, 8), fq.ERR_UNSUPPORTED),  # MX + 16-point rotation
    ((FAKE, 1, 4, 32, 32, 0, 3, FAKE, FAKE, FAKE, FAKE, FAKE, 8), fq.ERR_UNSUPPORTED),  # WMSE + rotation
    ((FAKE, 1, 4, 24, 24, 1, 0, None, FAKE, FAKE, FAKE, FAKE, 8), fq.ERR_SHAPE),        # IF4 + rotation, cols % 16
    ((None, 1, 0, 32, 32, 0, 2, None, None, None, None, None, 8), fq.OK),               # rotated, empty
    ((None, 1, 0, 32, 32, 0, 2, None, None, None, None, None, 0), fq.OK),               # empty: no launch
])
def test_quantize_rejects_before_launch(args, rc):
    L = fq.lib()
    assert L.fp4q_quantize(*args, None) == rc
    if rc == fq.OK:
        assert L.fp4q_last_launch_count() == 0


def test_hadamard_and_dequant_validation():
    L = fq.lib()
    assert L.fp4q_hadamard_quantize(FAKE, 1, 4, 64, 64, 16, FAKE, FAKE, FAKE, 0, None) == fq.ERR_UNSUPPORTED
    assert L.fp4q_hadamard_quantize(FAKE, 1, 4, 48, 48, 32, FAKE, FAKE, FAKE, 0, None) == fq.ERR_SHAPE
    assert L.fp4q_dequantize(FAKE, FAKE, FAKE, 4, 24, 0, 0, FAKE, 0, None) == fq.ERR_SHAPE
    assert L.fp4q_dequantize(FAKE, FAKE, FAKE, 4, 24, 1, 1, FAKE, 0, None) == fq.ERR_SHAPE   # rotated IF4
    assert L.fp4q_dequantize(FAKE, FAKE, None, 4, 32, 0, 0, FAKE, 0, None) == fq.ERR_INVALID_ARG
    assert L.fp4q_dequantize(FAKE, FAKE, FAKE, 4, 32, 0, 0, FAKE + 4, 0, None) == fq.ERR_ALIGNMENT
    assert L.fp4q_dequantize(FAKE, FAKE, FAKE, 4, 32, 0, 0, FAKE, 8, None) == fq.ERR_INVALID_ARG
    assert L.fp4q_dequantize(None, None, None, 0, 32, 0, 0, None, 0, None) == fq.OK
    assert L.fp4q_read_device_status(None, None, None) == fq.ERR_INVALID_ARG


def test_global_scale_validation():
    L = fq.lib()
    assert L.fp4q_global_scale(FAKE, 1, 4, 12, 12, FAKE, FAKE, None) == fq.ERR_SHAPE      # 24-byte rows
    assert L.fp4q_global_scale(FAKE, 1, 4, 16, 20, FAKE, FAKE, None) == fq.ERR_ALIGNMENT  # 40-byte pitch
    assert L.fp4q_global_scale(FAKE, 1, 4, 16, 16, None, FAKE, None) == fq.ERR_INVALID_ARG
    assert L.fp4q_global_scale(FAKE, 3, 4, 16, 16, FAKE, FAKE, None) == fq.ERR_INVALID_ARG
    assert L.fp4q_global_scale(None, 1, 0, 16, 16, None, None, None) == fq.OK
    # rotated tensor scale: 16-point only, whole blocks
    assert L.fp4q_hadamard_global_scale(FAKE, 1, 4, 32, 32, 32, FAKE, FAKE, None) == fq.ERR_UNSUPPORTED
    assert L.fp4q_hadamard_global_scale(FAKE, 1, 4, 8, 8, 16, FAKE, FAKE, None) == fq.ERR_SHAPE   # 16-byte rows
    assert L.fp4q_hadamard_global_scale(FAKE, 1, 4, 32, 36, 16, FAKE, FAKE, None) == fq.ERR_ALIGNMENT  # 72-byte pitch
    assert L.fp4q_hadamard_global_scale(FAKE, 1, 4, 32, 32, 16, None, FAKE, None) == fq.ERR_INVALID_ARG
    assert L.fp4q_hadamard_global_scale(None, 1, 0, 16, 16, 16, None, None, None) == fq.OK


def test_host_async_validation():
    """fp4q_quantize_host_async rejects bad arguments before any copy or launch."""
    L = fq.lib()
    # x_host, dtype, rows, cols, fmt, obj, imp, codes_h, scales_h, S_h, x_dev, codes_dev, scales_dev, S_dev,
    # ws, flags, copy_stream, compute_stream, staged_event, free_event
    ok = [FAKE, 1, 4, 32, 0, 2, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, None, None, FAKE, FAKE]

    def call(**kw):
        a = list(ok)
        names = ["x_host", "dtype", "rows", "cols", "fmt", "obj", "imp", "codes_h", "scales_h", "S_h", "x_dev",
                 "codes_dev", "scales_dev", "S_dev", "ws", "flags", "cs", "ks", "staged", "free"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return L.fp4q_quantize_host_async(*a)

    assert call(cols=24) == fq.ERR_SHAPE
    assert call(fmt=2, cols=48, S_h=None, S_dev=None) == fq.ERR_SHAPE
    assert call(x_host=None) == fq.ERR_INVALID_ARG
    assert call(codes_h=None) == fq.ERR_INVALID_ARG
    assert call(S_h=None) == fq.ERR_INVALID_ARG
    assert call(staged=None) == fq.ERR_INVALID_ARG
    assert call(free=None) == fq.ERR_INVALID_ARG
    assert call(obj=3) == fq.ERR_INVALID_ARG                     # WMSE without weights
    assert call(x_dev=FAKE + 8) == fq.ERR_ALIGNMENT
    assert call(flags=0x8, fmt=2, cols=64) == fq.ERR_UNSUPPORTED  # 16-point rotation on MXFP4
    assert call(flags=0x100) == fq.ERR_INVALID_ARG
    assert call(flags=0x40) == fq.ERR_UNSUPPORTED                 # IF4 sweep on NVFP4
    assert call(flags=0x20) == fq.ERR_UNSUPPORTED                 # MX sweep on NVFP4
    assert call(rows=0, x_host=None, x_dev=None) == fq.OK and L.fp4q_last_launch_count() == 0


def test_quantize_batch_rejects_before_launch():
    L = fq.lib()
    F = FAKE
    T = fq._Tensor

    def call(ts, fmt=0, obj=2, flags=0, dtype=1, ws=F, n=None):
        arr = (T * max(1, len(ts)))(*ts)
        return L.fp4q_quantize_batch(len(ts) if n is None else n, C.cast(arr, C.c_void_p), dtype, fmt, obj, ws,
                                     flags, None)

    good = lambda **kw: T(kw.get("x", F), kw.get("rows", 4), kw.get("cols", 64), kw.get("ld", 64),
                          kw.get("imp", None), kw.get("codes", F), kw.get("scales", F), kw.get("gs", F))
    assert call([good()], n=-1) == fq.ERR_INVALID_ARG
    assert L.fp4q_quantize_batch(2, None, 1, 0, 2, F, 0, None) == fq.ERR_INVALID_ARG
    assert call([good()], fmt=2) == fq.ERR_UNSUPPORTED                  # MXFP4: no tensor scale to batch
    assert call([good()], fmt=3) == fq.ERR_UNSUPPORTED                  # IF6
    assert call([good()], fmt=9) == fq.ERR_INVALID_ARG
    assert call([good(), good(cols=24)]) == fq.ERR_SHAPE                # checked for every tensor
    assert call([good(), good(ld=32)]) == fq.ERR_SHAPE
    assert call([good(), good(x=F + 8)]) == fq.ERR_ALIGNMENT
    assert call([good(), good(gs=None)]) == fq.ERR_INVALID_ARG
    assert call([good(imp=F), good(imp=None)], obj=3) == fq.ERR_INVALID_ARG  # WMSE needs each importance
    assert call([good(imp=F), good(imp=F + 4)], obj=3) == fq.ERR_ALIGNMENT
    assert call([good()], dtype=5) == fq.ERR_INVALID_ARG
    assert call([good()], ws=None) == fq.ERR_INVALID_ARG
    # empty tensors are skipped: a batch of only empty tensors launches nothing
    assert call([good(rows=0, x=None, codes=None, scales=None, gs=None), good(cols=0)]) == fq.OK
    assert L.fp4q_last_launch_count() == 0
    assert call([]) == fq.OK and L.fp4q_last_launch_count() == 0
