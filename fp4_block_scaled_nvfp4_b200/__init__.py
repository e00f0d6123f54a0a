"""Block-scaled FP4 quantization (NVFP4 / IF4 / MXFP4) for NVIDIA B200.

Thin ctypes binding over ``libfp4q.so`` (the C ABI in ``include/fp4q.h``).  Every step of
the quantization runs in the library's sm_100a kernels; this module only marshals torch
tensors (device memory and the current CUDA stream) into the C calls.  There is no CPU
fallback: if the library is missing the functions raise.

    codes, scales, S = quantize(x, fmt="nvfp4", objective="sweep_mse")
    xh = dequantize(codes, scales, S, fmt="nvfp4")
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp4q.so")

OK, ERR_INVALID_ARG, ERR_SHAPE, ERR_ALIGNMENT, ERR_UNSUPPORTED, ERR_CUDA = range(6)
DEVSTAT_OK, DEVSTAT_NONFINITE, DEVSTAT_RANGE, DEVSTAT_TIMEOUT = 0, 1, 2, 4
IN_F32, IN_BF16 = 0, 1
FORMATS = {"nvfp4": 0, "if4": 1, "mxfp4": 2, "if6": 3}
OBJECTIVES = {"absmax": 0, "four_over_six": 1, "sweep_mse": 2, "sweep_wmse": 3}
F_GLOBAL_SCALE_GIVEN, F_MX_OCP_FLOOR, F_OUT_BF16, F_HADAMARD16, F_HADAMARD32, F_MX_SWEEP, F_IF4_SWEEP = (
    0x1, 0x2, 0x4, 0x8, 0x10, 0x20, 0x40)
F_SCALE_TILED = 0x80
BLOCK = {"nvfp4": 16, "if4": 16, "mxfp4": 32, "if6": 16}


def code_bytes_per_row(cols: int, fmt: str) -> int:
    """Bytes of packed codes per row: 4-bit codes (NVFP4, IF4, MXFP4) or 6-bit fields (IF6)."""
    return cols * 3 // 4 if fmt == "if6" else cols // 2

# Names of every function include/fp4q.h declares (checked against the header by the tests).
EXPORTS = ("fp4q_workspace_bytes", "fp4q_scale_bytes", "fp4q_nvfp4_gemm", "fp4q_mxfp4_gemm", "fp4q_gemm", "fp4q_encode", "fp4q_global_scale", "fp4q_if6_global_scale", "fp4q_quantize_batch", "fp4q_hadamard_global_scale", "fp4q_quantize",
           "fp4q_hadamard_quantize", "fp4q_dequantize", "fp4q_quantize_noalloc", "fp4q_quantize_host_async", "fp4q_read_device_status", "fp4q_last_launch_count", "fp4q_last_cuda_error", "fp4q_status_string")

_lib = None


class Fp4qError(RuntimeError):
    pass


def lib():
    """Load libfp4q.so (built in-tree by __graft_entry__.build()); raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise Fp4qError(f"{LIB_PATH} is not built; run `python -c 'import __graft_entry__ as g; g.build()'`")
        L = C.CDLL(LIB_PATH)
        P, i64, u32, i32 = C.c_void_p, C.c_int64, C.c_uint32, C.c_int
        L.fp4q_workspace_bytes.restype = C.c_size_t
        L.fp4q_workspace_bytes.argtypes = []
        L.fp4q_scale_bytes.restype = i64
        L.fp4q_scale_bytes.argtypes = [i64, i64, i32, u32]
        L.fp4q_nvfp4_gemm.restype = i32
        L.fp4q_nvfp4_gemm.argtypes = [P, P, P, P, P, P, i64, i64, i64, P, i64, P, P]
        L.fp4q_mxfp4_gemm.restype = i32
        L.fp4q_gemm.restype = i32
        L.fp4q_gemm.argtypes = [i32, P, P, P, P, P, P, i64, i64, i64, P, i64, u32, P, P]
        L.fp4q_encode.restype = i32
        L.fp4q_encode.argtypes = [P, i64, i32, P, P]
        L.fp4q_mxfp4_gemm.argtypes = [P, P, P, P, i64, i64, i64, P, i64, P, P]
        L.fp4q_quantize.restype = i32
        L.fp4q_quantize.argtypes = [P, i32, i64, i64, i64, i32, i32, P, P, P, P, P, u32, P]
        L.fp4q_quantize_batch.restype = i32
        L.fp4q_quantize_batch.argtypes = [i32, P, i32, i32, i32, P, u32, P]
        L.fp4q_global_scale.restype = i32
        L.fp4q_global_scale.argtypes = [P, i32, i64, i64, i64, P, P, P]
        L.fp4q_if6_global_scale.restype = i32
        L.fp4q_if6_global_scale.argtypes = [P, i32, i64, i64, i64, P, P, P]
        L.fp4q_hadamard_global_scale.restype = i32
        L.fp4q_hadamard_global_scale.argtypes = [P, i32, i64, i64, i64, i32, P, P, P]
        L.fp4q_hadamard_quantize.restype = i32
        L.fp4q_hadamard_quantize.argtypes = [P, i32, i64, i64, i64, i32, P, P, P, u32, P]
        L.fp4q_dequantize.restype = i32
        L.fp4q_dequantize.argtypes = [P, P, P, i64, i64, i32, i32, P, u32, P]
        L.fp4q_quantize_noalloc.restype = i32
        L.fp4q_quantize_noalloc.argtypes = [P, i32, i64, i64, i64, i32, i32, P, P, P, P, P, u32, P]
        L.fp4q_quantize_host_async.restype = i32
        L.fp4q_quantize_host_async.argtypes = [P, i32, i64, i64, i32, i32, P, P, P, P, P, P, P, P, P, u32, P, P, P, P]
        L.fp4q_read_device_status.restype = i32
        L.fp4q_read_device_status.argtypes = [P, C.POINTER(C.c_uint32), P]
        L.fp4q_last_launch_count.restype = i32
        L.fp4q_last_launch_count.argtypes = []
        L.fp4q_last_cuda_error.restype = i32
        L.fp4q_last_cuda_error.argtypes = []
        L.fp4q_status_string.restype = C.c_char_p
        L.fp4q_status_string.argtypes = [i32]
        _lib = L
    return _lib


def status_string(rc: int) -> str:
    return lib().fp4q_status_string(int(rc)).decode()


def _check(rc: int, what: str):
    if rc != OK:
        extra = f", CUDA error {lib().fp4q_last_cuda_error()}" if rc == ERR_CUDA else ""
        raise Fp4qError(f"{what}: {status_string(rc)} ({rc}{extra})")


def _torch():
    import torch
    return torch


def _stream_ptr(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def workspace_bytes() -> int:
    return int(lib().fp4q_workspace_bytes())


def new_workspace(device="cuda"):
    """A zero-filled workspace (the library leaves it zeroed after each call, except the
    device status word)."""
    torch = _torch()
    return torch.zeros(max(workspace_bytes(), 16), dtype=torch.uint8, device=device)


def _dtype_code(x):
    torch = _torch()
    if x.dtype == torch.bfloat16:
        return IN_BF16
    if x.dtype == torch.float32:
        return IN_F32
    raise Fp4qError(f"unsupported input dtype {x.dtype} (bf16 or fp32)")


def alloc_outputs(rows: int, cols: int, fmt: str, device="cuda", tiled: bool = False):
    """(codes, scales, S) device buffers; tiled: a zero-filled 1-D scales buffer in the tiled
    layout of block-scaled GEMMs (scale_bytes(..., tiled=True) bytes)."""
    torch = _torch()
    codes = torch.empty((rows, code_bytes_per_row(cols, fmt)), dtype=torch.uint8, device=device)
    if tiled:
        scales = torch.zeros((scale_bytes(rows, cols, fmt, True),), dtype=torch.uint8, device=device)
    else:
        scales = torch.empty((rows, cols // BLOCK[fmt]), dtype=torch.uint8, device=device)
    gs = torch.empty((1,), dtype=torch.float32, device=device)
    return codes, scales, gs


def _objective(name) -> int:
    if name is None:
        return 0
    if name not in OBJECTIVES:
        raise Fp4qError(f"unknown objective {name!r} (one of {sorted(OBJECTIVES)})")
    return OBJECTIVES[name]


def _format(name) -> int:
    if name not in FORMATS:
        raise Fp4qError(f"unknown format {name!r} (one of {sorted(FORMATS)})")
    return FORMATS[name]


def _need(t, what, device, dtypes, numel=None, min_numel=None, contiguous=True):
    """Raise Fp4qError unless t is a CUDA tensor on `device` of one of `dtypes` with the given
    element count (exact, or at least min_numel), contiguous unless told otherwise.  Every
    wrapper checks its tensors this way before calling into the library, so no pointer the
    kernels would read or write out of bounds ever reaches them."""
    if t is None:
        raise Fp4qError(f"{what} is required")
    if not t.is_cuda or t.device != device:
        raise Fp4qError(f"{what} must be a CUDA tensor on {device} (got {t.device})")
    if t.dtype not in dtypes:
        raise Fp4qError(f"{what} must have dtype {' or '.join(str(d) for d in dtypes)} (got {t.dtype})")
    if contiguous and not t.is_contiguous():
        raise Fp4qError(f"{what} must be contiguous")
    if numel is not None and t.numel() != numel:
        raise Fp4qError(f"{what} must hold {numel} elements (got {t.numel()})")
    if min_numel is not None and t.numel() < min_numel:
        raise Fp4qError(f"{what} must hold at least {min_numel} elements (got {t.numel()})")


def _check_quantize(x, fmt, objective, importance, codes, scales, gs, tiled, workspace=None, device_status=None):
    torch = _torch()
    if x is None or not x.is_cuda:
        raise Fp4qError("x must be a CUDA tensor")
    if x.dim() != 2 or x.stride(1) != 1:
        raise Fp4qError("x must be 2-D with unit column stride")
    _dtype_code(x)
    rows, cols = x.shape
    dev = x.device
    _need(codes, "codes", dev, (torch.uint8,), numel=rows * code_bytes_per_row(cols, fmt))
    _need(scales, "scales", dev, (torch.uint8,), numel=scale_bytes(rows, cols, fmt, tiled))
    if fmt != "mxfp4":
        _need(gs, "global scale", dev, (torch.float32,), min_numel=1)
    if fmt == "nvfp4" and objective == "sweep_wmse":
        _need(importance, "importance", dev, (torch.float32,), min_numel=cols)
    if workspace is not None:
        _need(workspace, "workspace", dev, (torch.uint8, torch.int32, torch.int64, torch.float32),
              contiguous=True)
        if workspace.numel() * workspace.element_size() < workspace_bytes():
            raise Fp4qError(f"workspace must hold at least {workspace_bytes()} bytes")
    if device_status is not None:
        _need(device_status, "device_status", dev, (torch.int32, torch.uint32), min_numel=1)


def _flags(global_scale, mx_ocp_floor, hadamard16, mx_sweep=False, if4_sweep=False, tiled=False):
    return ((F_GLOBAL_SCALE_GIVEN if global_scale is not None else 0) | (F_MX_OCP_FLOOR if mx_ocp_floor else 0)
            | (F_HADAMARD16 if hadamard16 else 0) | (F_MX_SWEEP if mx_sweep else 0)
            | (F_IF4_SWEEP if if4_sweep else 0) | (F_SCALE_TILED if tiled else 0))


def scale_bytes(rows: int, cols: int, fmt: str, tiled: bool = False) -> int:
    """Bytes of the scales buffer: rows * cols/B, or the padded tiled layout (tiled=True)."""
    n = int(lib().fp4q_scale_bytes(rows, cols, FORMATS[fmt], F_SCALE_TILED if tiled else 0))
    if n < 0:
        raise Fp4qError("fp4q_scale_bytes: bad format or shape")
    return n


def quantize(x, fmt: str = "nvfp4", objective: str = "sweep_mse", importance=None, global_scale=None,
             mx_ocp_floor: bool = False, out=None, workspace=None, stream=None, hadamard16: bool = False,
             mx_sweep: bool = False, if4_sweep: bool = False, tiled_scales: bool = False):
    """Quantize a 2-D bf16/fp32 CUDA tensor (row stride may exceed the width).

    Returns (codes [rows, cols/2] uint8, scales [rows, cols/B] uint8, S [1] float32 or None).
    global_scale: a [1] float32 CUDA tensor to use as S (skips the amax pass).
    out: optional preallocated (codes, scales, S) tuple.
    hadamard16: NVFP4/IF4 on blocks rotated by the normalized 16-point Hadamard.
    mx_sweep: MXFP4 with the MX scale sweep (exponents e_c-2 .. e_c by block error).
    if4_sweep: IF4 x ScaleSweep (scale and element type chosen together over the MSE window).
    tiled_scales: NVFP4/MXFP4 scales in the 128x4-tiled layout of block-scaled GEMMs (1-D buffer).
    """
    fcode = _format(fmt)
    ocode = _objective(objective) if fmt == "nvfp4" else 0   # only NVFP4 has objectives
    if x is None or not x.is_cuda or x.dim() != 2 or x.stride(1) != 1:
        raise Fp4qError("x must be a 2-D CUDA tensor with unit column stride")
    rows, cols = x.shape
    if cols % BLOCK[fmt]:
        raise Fp4qError(f"cols must be a multiple of {BLOCK[fmt]}")
    codes, scales, gs = out if out is not None else alloc_outputs(rows, cols, fmt, x.device, tiled=tiled_scales)
    flags = _flags(global_scale, mx_ocp_floor, hadamard16, mx_sweep, if4_sweep, tiled_scales)
    if global_scale is not None:
        gs = global_scale
    ws = workspace if workspace is not None else new_workspace(x.device)
    _check_quantize(x, fmt, objective, importance, codes, scales, gs, tiled_scales, workspace=ws)
    rc = lib().fp4q_quantize(_ptr(x), _dtype_code(x), rows, cols, x.stride(0), fcode,
                             ocode, _ptr(importance), _ptr(codes), _ptr(scales),
                             _ptr(gs) if fmt != "mxfp4" else None, _ptr(ws), flags, _stream_ptr(stream))
    _check(rc, "fp4q_quantize")
    return codes, scales, (gs if fmt != "mxfp4" else None)


class _Tensor(C.Structure):
    """fp4q_tensor of include/fp4q.h."""
    _fields_ = [("x", C.c_void_p), ("rows", C.c_int64), ("cols", C.c_int64), ("ld", C.c_int64),
                ("importance", C.c_void_p), ("codes", C.c_void_p), ("scales", C.c_void_p),
                ("global_scale", C.c_void_p)]


class BatchPlan:
    """A checked, marshalled fp4q_quantize_batch call over fixed buffers, for callers that run
    the same batch repeatedly (the descriptors are built once; each call is the C call only).

    xs: 2-D CUDA tensors of one dtype on one device; fmt "nvfp4" or "if4".
    importance: one float32 [cols] tensor per input (SWEEP_WMSE), or None.
    global_scales: one [1] float32 tensor per input to use as S (no amax passes), or None.
    outs: optional list of preallocated (codes, scales, S) tuples (entries may repeat: later
    tensors overwrite earlier results, as separate calls would).
    """

    def __init__(self, xs, fmt: str = "nvfp4", objective: str = "sweep_mse", importance=None, global_scales=None,
                 outs=None, workspace=None, hadamard16: bool = False, if4_sweep: bool = False,
                 tiled_scales: bool = False):
        if fmt not in ("nvfp4", "if4"):
            raise Fp4qError(f"a batch holds nvfp4 or if4 tensors, not {fmt!r}")
        self.fcode = _format(fmt)
        self.ocode = _objective(objective) if fmt == "nvfp4" else 0
        xs = list(xs)
        n = len(xs)
        for name, seq in (("importance", importance), ("global_scales", global_scales), ("outs", outs)):
            if seq is not None and len(seq) != n:
                raise Fp4qError(f"{name} must have one entry per tensor")
        self.n, self.results, self.dcode, self.ws = n, [], IN_BF16, None
        self.arr = (_Tensor * max(n, 1))()
        self.flags = _flags(global_scales, False, hadamard16, False, if4_sweep, tiled_scales)
        self._keep = (xs, importance, global_scales)
        if n == 0:
            return
        dev = xs[0].device if xs[0] is not None else None
        dcode = None
        for i, x in enumerate(xs):
            if x is None or not x.is_cuda or x.dim() != 2 or (x.numel() and x.stride(1) != 1):
                raise Fp4qError("every input must be a 2-D CUDA tensor with unit column stride")
            if x.device != dev:
                raise Fp4qError("every input must be on the same device")
            code = _dtype_code(x)
            if dcode is not None and code != dcode:
                raise Fp4qError("every input must have the same dtype")
            dcode = code
            rows, cols = x.shape
            if cols % 16:
                raise Fp4qError("cols must be a multiple of 16")
            codes, scales, gs = outs[i] if outs is not None else alloc_outputs(rows, cols, fmt, dev,
                                                                               tiled=tiled_scales)
            if global_scales is not None:
                gs = global_scales[i]
            if x.numel() == 0:   # skipped by the library; nothing is read or written
                self.arr[i] = _Tensor(None, rows, cols, cols, None, None, None, None)
                self.results.append((codes, scales, gs))
                continue
            imp = importance[i] if importance is not None else None
            _check_quantize(x, fmt, objective, imp, codes, scales, gs, tiled_scales)
            ld = x.stride(0) if rows > 1 else cols   # the row pitch of a tensor with one row or none is unused
            self.arr[i] = _Tensor(x.data_ptr(), rows, cols, ld, None if imp is None else imp.data_ptr(),
                                  codes.data_ptr(), scales.data_ptr(), gs.data_ptr())
            self.results.append((codes, scales, gs))
        torch = _torch()
        ws = workspace if workspace is not None else new_workspace(dev)
        _need(ws, "workspace", dev, (torch.uint8, torch.int32, torch.int64, torch.float32))
        if ws.numel() * ws.element_size() < workspace_bytes():
            raise Fp4qError(f"workspace must hold at least {workspace_bytes()} bytes")
        self.dcode, self.ws = dcode, ws

    def __call__(self, stream=None):
        """Run the batch on `stream` (default: the current stream); returns [(codes, scales, S)]."""
        if self.n:
            rc = lib().fp4q_quantize_batch(self.n, C.cast(self.arr, C.c_void_p), self.dcode, self.fcode, self.ocode,
                                           _ptr(self.ws), self.flags, _stream_ptr(stream))
            _check(rc, "fp4q_quantize_batch")
        return self.results


def quantize_batch(xs, fmt: str = "nvfp4", objective: str = "sweep_mse", importance=None, global_scales=None,
                   outs=None, workspace=None, stream=None, hadamard16: bool = False, if4_sweep: bool = False,
                   tiled_scales: bool = False):
    """NVFP4 / IF4 quantization of a sequence of 2-D CUDA tensors of one dtype in one call
    (fp4q_quantize_batch): the results of quantize() on each, with each tensor's amax pass folded
    into the previous tensor's quantize kernel.  Arguments as BatchPlan; returns the list of
    (codes, scales, S)."""
    return BatchPlan(xs, fmt, objective, importance=importance, global_scales=global_scales, outs=outs,
                     workspace=workspace, hadamard16=hadamard16, if4_sweep=if4_sweep,
                     tiled_scales=tiled_scales)(stream)


def global_scale(x, out=None, workspace=None, stream=None, hadamard16: bool = False, fmt: str = "nvfp4"):
    """Tensor scale S = RN(max|x| / 1536) as a [1] float32 CUDA tensor (amax pass only);
    hadamard16: of the 16-point block-rotated tensor; fmt "if6": IF6's S = RN(max|x| / 1920)."""
    torch = _torch()
    if x is None or not x.is_cuda or x.dim() != 2 or x.stride(1) != 1:
        raise Fp4qError("x must be a 2-D CUDA tensor with unit column stride")
    _dtype_code(x)
    rows, cols = x.shape
    gs = out if out is not None else torch.empty((1,), dtype=torch.float32, device=x.device)
    ws = workspace if workspace is not None else new_workspace(x.device)
    _need(gs, "out", x.device, (torch.float32,), min_numel=1)
    _need(ws, "workspace", x.device, (torch.uint8,), min_numel=workspace_bytes())
    if fmt not in ("nvfp4", "if4", "if6"):
        raise Fp4qError(f"no tensor scale for format {fmt!r}")
    if fmt == "if6":
        if hadamard16:
            raise Fp4qError("IF6 has no rotated form")
        rc = lib().fp4q_if6_global_scale(_ptr(x), _dtype_code(x), rows, cols, x.stride(0), _ptr(gs), _ptr(ws),
                                         _stream_ptr(stream))
    elif hadamard16:
        rc = lib().fp4q_hadamard_global_scale(_ptr(x), _dtype_code(x), rows, cols, x.stride(0), 16, _ptr(gs),
                                              _ptr(ws), _stream_ptr(stream))
    else:
        rc = lib().fp4q_global_scale(_ptr(x), _dtype_code(x), rows, cols, x.stride(0), _ptr(gs), _ptr(ws),
                                     _stream_ptr(stream))
    _check(rc, "fp4q_global_scale")
    return gs


def hadamard_quantize(x, mx_ocp_floor: bool = False, out=None, workspace=None, stream=None, mx_sweep: bool = False,
                      tiled_scales: bool = False):
    """MXFP4 quantization after a normalized 32-point block Hadamard rotation (mx_sweep: with
    the MX scale sweep)."""
    if x is None or not x.is_cuda or x.dim() != 2 or x.stride(1) != 1:
        raise Fp4qError("x must be a 2-D CUDA tensor with unit column stride")
    rows, cols = x.shape
    if cols % 32:
        raise Fp4qError("cols must be a multiple of 32")
    codes, scales, _ = out if out is not None else alloc_outputs(rows, cols, "mxfp4", x.device, tiled=tiled_scales)
    ws = workspace if workspace is not None else new_workspace(x.device)
    _check_quantize(x, "mxfp4", None, None, codes, scales, None, tiled_scales, workspace=ws)
    rc = lib().fp4q_hadamard_quantize(_ptr(x), _dtype_code(x), rows, cols, x.stride(0), 32, _ptr(codes),
                                      _ptr(scales), _ptr(ws), _flags(None, mx_ocp_floor, False, mx_sweep,
                                                                     tiled=tiled_scales),
                                      _stream_ptr(stream))
    _check(rc, "fp4q_hadamard_quantize")
    return codes, scales


def dequantize(codes, scales, global_scale, fmt: str = "nvfp4", inverse_hadamard: bool = False,
               out_dtype=None, out=None, stream=None, tiled_scales: bool = False):
    torch = _torch()
    fcode = _format(fmt)
    out_dtype = out_dtype or torch.float32
    if codes is None or not codes.is_cuda or codes.dim() != 2:
        raise Fp4qError("codes must be a 2-D CUDA tensor [rows, code bytes per row]")
    rows = codes.shape[0]
    cols = codes.shape[1] * 4 // 3 if fmt == "if6" else codes.shape[1] * 2
    dev = codes.device
    if cols % BLOCK[fmt] or code_bytes_per_row(cols, fmt) != codes.shape[1]:
        raise Fp4qError(f"cols must be a multiple of {BLOCK[fmt]}")
    _need(codes, "codes", dev, (torch.uint8,), numel=rows * code_bytes_per_row(cols, fmt))
    _need(scales, "scales", dev, (torch.uint8,), numel=scale_bytes(rows, cols, fmt, tiled_scales))
    if fmt != "mxfp4":
        _need(global_scale, "global_scale", dev, (torch.float32,), min_numel=1)
    if out is None:
        out = torch.empty((rows, cols), dtype=out_dtype, device=dev)
    _need(out, "out", dev, (torch.float32, torch.bfloat16), numel=rows * cols)
    flags = (F_OUT_BF16 if out.dtype == torch.bfloat16 else 0) | (F_SCALE_TILED if tiled_scales else 0)
    rc = lib().fp4q_dequantize(_ptr(codes), _ptr(scales), _ptr(global_scale) if fmt != "mxfp4" else None,
                               rows, cols, fcode,
                               int(inverse_hadamard), _ptr(out), flags, _stream_ptr(stream))
    _check(rc, "fp4q_dequantize")
    return out


def quantize_noalloc(x, fmt: str = "nvfp4", objective: str = "sweep_mse", importance=None, global_scale=None,
                     mx_ocp_floor: bool = False, out=None, device_status=None, stream=None,
                     hadamard16: bool = False, mx_sweep: bool = False, if4_sweep: bool = False,
                     tiled_scales: bool = False):
    """quantize() for callers that cannot allocate device memory: the library's own
    per-GPU scratch replaces the workspace (see fp4q_quantize_noalloc in include/fp4q.h).
    Outputs must be passed in `out`; device_status is an optional [1] int32 CUDA tensor."""
    fcode = _format(fmt)
    ocode = _objective(objective) if fmt == "nvfp4" else 0   # only NVFP4 has objectives
    if x is None or not x.is_cuda or x.dim() != 2 or x.stride(1) != 1:
        raise Fp4qError("x must be a 2-D CUDA tensor with unit column stride")
    if out is None:
        raise Fp4qError("quantize_noalloc needs preallocated outputs (codes, scales, S)")
    rows, cols = x.shape
    if cols % BLOCK[fmt]:
        raise Fp4qError(f"cols must be a multiple of {BLOCK[fmt]}")
    codes, scales, gs = out
    flags = _flags(global_scale, mx_ocp_floor, hadamard16, mx_sweep, if4_sweep, tiled_scales)
    if global_scale is not None:
        gs = global_scale
    _check_quantize(x, fmt, objective, importance, codes, scales, gs, tiled_scales, device_status=device_status)
    rc = lib().fp4q_quantize_noalloc(_ptr(x), _dtype_code(x), rows, cols, x.stride(0), fcode,
                                     ocode, _ptr(importance), _ptr(codes), _ptr(scales),
                                     _ptr(gs) if fmt != "mxfp4" else None, _ptr(device_status), flags,
                                     _stream_ptr(stream))
    _check(rc, "fp4q_quantize_noalloc")
    return codes, scales, (gs if fmt != "mxfp4" else None)


def _check_gemm_operands(ac, asc, bc, bsc, fmt):
    torch = _torch()
    if ac is None or not ac.is_cuda or ac.dim() != 2 or bc is None or bc.dim() != 2:
        raise Fp4qError("operand codes must be 2-D CUDA tensors [rows, K/2]")
    M, K, N = ac.shape[0], ac.shape[1] * 2, bc.shape[0]
    if bc.shape[1] * 2 != K:
        raise Fp4qError("a and b must have the same K")
    dev = ac.device
    _need(ac, "a codes", dev, (torch.uint8,))
    _need(bc, "b codes", dev, (torch.uint8,))
    _need(asc, "a scales", dev, (torch.uint8,), numel=scale_bytes(M, K, fmt, True))
    _need(bsc, "b scales", dev, (torch.uint8,), numel=scale_bytes(N, K, fmt, True))
    return M, K, N


def _check_gemm_out(d, M, N, ws):
    torch = _torch()
    if not d.is_cuda or d.dim() != 2 or d.shape[0] != M or d.shape[1] != N or d.stride(1) != 1:
        raise Fp4qError(f"out must be a CUDA [{M}, {N}] tensor with unit column stride")
    if d.dtype not in (torch.float32, torch.bfloat16):
        raise Fp4qError("out must be float32 or bfloat16")
    _need(ws, "workspace", d.device, (torch.uint8,), min_numel=workspace_bytes())


def nvfp4_gemm(a, b, out=None, workspace=None, stream=None, out_dtype=None):
    """Block-scaled NVFP4 GEMM on the tensor cores: a = (codes [M, K/2], tiled scales, S) and
    b = (codes [N, K/2], tiled scales, S) as returned by quantize(..., tiled_scales=True);
    returns [M, N] = S_a S_b A B^T in fp32, or bf16 (out_dtype=torch.bfloat16, or a bf16 out).
    M, N multiples of 128, K a multiple of 256."""
    torch = _torch()
    ac, asc, ag = a
    bc, bsc, bg = b
    M, K, N = _check_gemm_operands(ac, asc, bc, bsc, "nvfp4")
    d = out if out is not None else torch.empty((M, N), dtype=out_dtype or torch.float32, device=ac.device)
    ws = workspace if workspace is not None else new_workspace(ac.device)
    _need(ag, "a's S", ac.device, (torch.float32,), min_numel=1)
    _need(bg, "b's S", ac.device, (torch.float32,), min_numel=1)
    _check_gemm_out(d, M, N, ws)
    rc = lib().fp4q_gemm(FORMATS["nvfp4"], _ptr(ac), _ptr(asc), _ptr(ag), _ptr(bc), _ptr(bsc), _ptr(bg), M, N, K,
                         _ptr(d), d.stride(0), F_OUT_BF16 if d.dtype == torch.bfloat16 else 0, _ptr(ws),
                         _stream_ptr(stream))
    _check(rc, "fp4q_gemm")
    return d


def mxfp4_gemm(a, b, out=None, workspace=None, stream=None, out_dtype=None):
    """Block-scaled MXFP4 GEMM on the tensor cores: a = (codes [M, K/2], tiled E8M0 scales) and
    b = (codes [N, K/2], tiled E8M0 scales) as returned by quantize / hadamard_quantize(...,
    "mxfp4", tiled_scales=True) (a third element, the absent tensor scale, is ignored);
    returns [M, N] = A B^T in fp32, or bf16 (out_dtype=torch.bfloat16, or a bf16 out).  M, N
    multiples of 128, K a multiple of 256."""
    torch = _torch()
    ac, asc = a[0], a[1]
    bc, bsc = b[0], b[1]
    M, K, N = _check_gemm_operands(ac, asc, bc, bsc, "mxfp4")
    d = out if out is not None else torch.empty((M, N), dtype=out_dtype or torch.float32, device=ac.device)
    ws = workspace if workspace is not None else new_workspace(ac.device)
    _check_gemm_out(d, M, N, ws)
    rc = lib().fp4q_gemm(FORMATS["mxfp4"], _ptr(ac), _ptr(asc), None, _ptr(bc), _ptr(bsc), None, M, N, K, _ptr(d),
                         d.stride(0), F_OUT_BF16 if d.dtype == torch.bfloat16 else 0, _ptr(ws), _stream_ptr(stream))
    _check(rc, "fp4q_gemm")
    return d


def encode(x, kind: str, out=None, stream=None):
    """The hardware element codec on a CUDA fp32 tensor: kind "e2m1" -> 4-bit E2M1 codes (sign
    in bit 3), "e4m3" -> E4M3FN bytes; both round to nearest even and saturate."""
    torch = _torch()
    if x is None or not x.is_cuda or x.dtype != torch.float32:
        raise Fp4qError("x must be a float32 CUDA tensor")
    x = x.contiguous().view(-1)
    out = out if out is not None else torch.empty(x.numel(), dtype=torch.uint8, device=x.device)
    _need(out, "out", x.device, (torch.uint8,), numel=x.numel())
    rc = lib().fp4q_encode(_ptr(x), x.numel(), {"e2m1": 0, "e4m3": 1}[kind], _ptr(out), _stream_ptr(stream))
    _check(rc, "fp4q_encode")
    return out


def read_device_status(workspace, stream=None) -> int:
    st = C.c_uint32(0)
    _check(lib().fp4q_read_device_status(_ptr(workspace), C.byref(st), _stream_ptr(stream)), "read_device_status")
    return int(st.value)


def last_launch_count() -> int:
    return int(lib().fp4q_last_launch_count())


def split_fmt(fmt: str):
    """'nvfp4_had' / 'if4_had' -> 16-point rotated NVFP4 / IF4, 'mxfp4_had' -> rotated MXFP4;
    returns (base format, flags)."""
    if not fmt.endswith("_had"):
        return fmt, 0
    base = fmt[:-4]
    return base, (F_HADAMARD32 if base == "mxfp4" else F_HADAMARD16)


def alloc_host_outputs(rows: int, cols: int, fmt: str):
    """Pinned host buffers for (codes, scales, S)."""
    torch = _torch()
    base, _ = split_fmt(fmt)
    return (torch.empty((rows, code_bytes_per_row(cols, base)), dtype=torch.uint8, pin_memory=True),
            torch.empty((rows, cols // BLOCK[base]), dtype=torch.uint8, pin_memory=True),
            torch.empty((1,), dtype=torch.float32, pin_memory=True))


class HostQuantizer:
    """Quantize tensors that live in pinned host memory (fp4q_quantize_host_async).

    Holds `depth` device staging sets (input, codes, scales, S, workspace and two events)
    used in turn, a copy stream for the input copies and a compute stream for the kernels
    and the output copies, so the input copy of one call overlaps the previous call's
    kernels and output copies.  Each call returns the host (codes, scales, S) it will fill;
    they are valid once `synchronize()` (or the compute stream) has passed the call.
    fmt: "nvfp4", "if4", "mxfp4", or the rotated "nvfp4_had", "if4_had", "mxfp4_had";
    mx_sweep: MXFP4 with the MX scale sweep; if4_sweep: IF4 x ScaleSweep."""

    def __init__(self, rows, cols, fmt="nvfp4", objective="sweep_mse", importance=None, dtype=None, depth=2,
                 device="cuda", copy_stream=None, compute_stream=None, mx_sweep: bool = False,
                 if4_sweep: bool = False):
        torch = _torch()
        self.rows, self.cols, self.fmt, self.objective = rows, cols, fmt, objective
        self.base, self.flags = split_fmt(fmt)
        if mx_sweep:
            self.flags |= F_MX_SWEEP
        if if4_sweep:
            self.flags |= F_IF4_SWEEP
        self.dtype = dtype or torch.bfloat16
        self.importance = importance
        self.copy_stream = copy_stream or torch.cuda.Stream(device=device)
        self.compute_stream = compute_stream or torch.cuda.Stream(device=device)
        self.sets = []
        for _ in range(max(1, depth)):
            codes, scales, gs = alloc_outputs(rows, cols, self.base, device)
            st = {"x": torch.empty((rows, cols), dtype=self.dtype, device=device), "codes": codes, "scales": scales,
                  "S": gs, "ws": new_workspace(device), "staged": torch.cuda.Event(), "free": torch.cuda.Event()}
            st["free"].record(self.compute_stream)   # the first use of the set waits on nothing
            st["staged"].record(self.copy_stream)
            self.sets.append(st)
        self.turn = 0

    def __call__(self, x_host, host_out=None):
        if tuple(x_host.shape) != (self.rows, self.cols) or x_host.dtype != self.dtype or not x_host.is_contiguous():
            raise Fp4qError("x_host must be a contiguous [rows, cols] tensor of the quantizer's dtype")
        st = self.sets[self.turn]
        self.turn = (self.turn + 1) % len(self.sets)
        hc, hs, hg = host_out if host_out is not None else alloc_host_outputs(self.rows, self.cols, self.fmt)
        rc = lib().fp4q_quantize_host_async(
            _ptr(x_host), _dtype_code(x_host), self.rows, self.cols, FORMATS[self.base],
            _objective(self.objective) if self.base == "nvfp4" else 0, _ptr(self.importance), _ptr(hc), _ptr(hs),
            _ptr(hg) if self.base != "mxfp4" else None, _ptr(st["x"]), _ptr(st["codes"]), _ptr(st["scales"]),
            _ptr(st["S"]) if self.base != "mxfp4" else None, _ptr(st["ws"]), self.flags,
            C.c_void_p(self.copy_stream.cuda_stream), C.c_void_p(self.compute_stream.cuda_stream),
            C.c_void_p(st["staged"].cuda_event), C.c_void_p(st["free"].cuda_event))
        _check(rc, "fp4q_quantize_host_async")
        return hc, hs, (hg if self.base != "mxfp4" else None)

    def synchronize(self):
        self.compute_stream.synchronize()


def quantize_host(x_host, fmt="nvfp4", objective="sweep_mse", importance=None, host_out=None):
    """One end-to-end call on host (pinned) memory: copy in, quantize, copy codes, scales and
    S back; returns the host (codes, scales, S) after the copies have completed."""
    q = HostQuantizer(x_host.shape[0], x_host.shape[1], fmt, objective, importance=importance, dtype=x_host.dtype,
                      depth=1)
    out = q(x_host, host_out)
    q.synchronize()
    return out
