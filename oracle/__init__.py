"""CPU oracle for block-scaled FP4 quantization -- TEST INFRASTRUCTURE ONLY.

Plain, slow, single-threaded C (``fp4q_oracle.c``) behind ctypes.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import this
package; the library's product path never does.  It shares no code with the CUDA path.

Each function follows the passage its C counterpart cites:
  ScaleSweep (gist.science/ko/paper/2606.07618) "Methodology": global scale, base scale,
      candidate windows [-3,+7] (MSE) / [-8,+7] (WMSE), MSE and WMSE objectives.
  Adaptive Block-Scaled Data Types (gist.science/ko/paper/2603.28765) "Methodology":
      IF4 selection, 7/6 and 6/7, indicator in the scale sign bit; "Problem": 4/6.
  Bridging the Gap ... Microscaling FP4 (gist.science/ko/paper/2509.23202) "Methodology":
      MXFP4 (32-element blocks, power-of-two scales), block-wise Hadamard.
  TORQ (gist.science/ko/paper/2605.19561) "Method", S-step: block max onto the largest code.
The GEMM products (``nvfp4_gemm``, ``mxfp4_gemm``) are the plain definition of the product of
two quantized operands, in float64 from the oracle's own code tables; ``encode`` is the
oracle's element codec over arrays.

Pins (tests/test_oracle_pins.py): exact rationals, brute-force argmins, closed forms and
hand-worked blocks.  Parity unpinned against the pages for end-to-end reconstruction MSE
values per configuration: the pages print no worked numbers.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

ST_OK, ST_NONFINITE, ST_RANGE = 0, 1, 2
OBJ = {"absmax": 0, "four_over_six": 1, "sweep_mse": 2, "sweep_wmse": 3, "brute_mse": 4, "brute_wmse": 5}
FMT = {"nvfp4": 0, "if4": 1, "mxfp4": 2}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        P = C.c_void_p
        i64 = C.c_int64
        L.fp4q_o_e4m3_value.restype = C.c_double
        L.fp4q_o_e4m3_value.argtypes = [C.c_int]
        L.fp4q_o_e4m3_encode.restype = C.c_int
        L.fp4q_o_e4m3_encode.argtypes = [C.c_float]
        L.fp4q_o_e2m1_value.restype = C.c_float
        L.fp4q_o_e2m1_value.argtypes = [C.c_int]
        L.fp4q_o_e2m1_encode.restype = C.c_int
        L.fp4q_o_e2m1_encode.argtypes = [C.c_float]
        L.fp4q_o_encode.restype = C.c_int
        L.fp4q_o_encode.argtypes = [P, i64, C.c_int, P]
        L.fp4q_o_global_scale.restype = C.c_float
        L.fp4q_o_global_scale.argtypes = [C.c_float]
        L.fp4q_o_tensor_scale.restype = C.c_int
        L.fp4q_o_tensor_scale.argtypes = [P, i64, i64, i64, P]
        L.fp4q_o_mx_exponent.restype = C.c_int
        L.fp4q_o_mx_exponent.argtypes = [C.c_float, C.c_int]
        L.fp4q_o_hadamard16.restype = None
        L.fp4q_o_hadamard16.argtypes = [P]
        L.fp4q_o_rotate16.restype = C.c_int
        L.fp4q_o_rotate16.argtypes = [P, i64, i64, i64, P]
        L.fp4q_o_hadamard32.restype = None
        L.fp4q_o_hadamard32.argtypes = [P]
        L.fp4q_o_nvfp4_quantize.restype = C.c_int
        L.fp4q_o_nvfp4_quantize.argtypes = [P, i64, i64, i64, C.c_int, P, C.c_int, P, P, P, P, P, P, P, P, P]
        L.fp4q_o_if4_quantize.restype = C.c_int
        L.fp4q_o_if4_quantize.argtypes = [P, i64, i64, i64, C.c_int, C.c_int, P, P, P, P, P, P, P]
        L.fp4q_o_mxfp4_quantize.restype = C.c_int
        L.fp4q_o_mxfp4_quantize.argtypes = [P, i64, i64, i64, C.c_int, C.c_int, C.c_int, P, P, P, P]
        L.fp4q_o_e2m3_value.restype = C.c_double
        L.fp4q_o_e2m3_value.argtypes = [C.c_int]
        L.fp4q_o_e2m3_encode.restype = C.c_int
        L.fp4q_o_e2m3_encode.argtypes = [C.c_float]
        L.fp4q_o_global_scale_if6.restype = C.c_float
        L.fp4q_o_global_scale_if6.argtypes = [C.c_float]
        L.fp4q_o_if6_quantize.restype = C.c_int
        L.fp4q_o_if6_quantize.argtypes = [P, i64, i64, i64, C.c_int, P, P, P, P, P, P, P]
        L.fp4q_o_if6_dequantize.restype = C.c_int
        L.fp4q_o_if6_dequantize.argtypes = [P, P, C.c_float, i64, i64, P, C.c_int]
        L.fp4q_o_f32_to_bf16.restype = None
        L.fp4q_o_f32_to_bf16.argtypes = [P, i64, P]
        L.fp4q_o_undecided.restype = C.c_long
        L.fp4q_o_undecided.argtypes = []
        L.fp4q_o_inexact.restype = C.c_long
        L.fp4q_o_inexact.argtypes = []
        L.fp4q_o_mx_block_errors.restype = C.c_int
        L.fp4q_o_mx_block_errors.argtypes = [P, i64, i64, i64, C.c_int, P, P]
        L.fp4q_o_dequantize.restype = C.c_int
        L.fp4q_o_dequantize.argtypes = [P, P, C.c_float, i64, i64, C.c_int, C.c_int, P, C.c_int]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _f32(x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    if x.ndim == 1:
        x = x.reshape(1, -1)
    return x


# --- codec -------------------------------------------------------------------------
def e4m3_value(p: int) -> float:
    return lib().fp4q_o_e4m3_value(int(p))


def e4m3_encode(v: float) -> int:
    return lib().fp4q_o_e4m3_encode(float(v))


def e2m1_value(code: int) -> float:
    return lib().fp4q_o_e2m1_value(int(code))


def e2m1_encode(y: float) -> int:
    return lib().fp4q_o_e2m1_encode(float(y))


def global_scale(amax: float) -> float:
    return lib().fp4q_o_global_scale(float(amax))


def tensor_scale(x):
    """(S, status) of a whole float32 tensor: S = RN(max|x| / 1536)."""
    x = _f32(x)
    S = np.zeros(1, np.float32)
    st = lib().fp4q_o_tensor_scale(_p(x), x.shape[0], x.shape[1], x.shape[1], _p(S))
    return float(S[0]), st


def mx_exponent(a: float, ocp_floor: bool = False) -> int:
    return lib().fp4q_o_mx_exponent(float(a), int(ocp_floor))


def hadamard32(v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32).copy()
    assert v.size == 32
    lib().fp4q_o_hadamard32(_p(v))
    return v


def hadamard16(v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32).copy()
    assert v.size == 16
    lib().fp4q_o_hadamard16(_p(v))
    return v


def rotate16(x) -> np.ndarray:
    """Every 16-element block of every row rotated by the normalized 16-point Hadamard."""
    x = _f32(x)
    out = np.empty_like(x)
    if lib().fp4q_o_rotate16(_p(x), x.shape[0], x.shape[1], x.shape[1], _p(out)) < 0:
        raise ValueError("oracle: bad shape")
    return out


# --- quantizers --------------------------------------------------------------------
class OracleUndecided(RuntimeError):
    """Two candidates came within the rounding of an inexact (brute-force-only) evaluation."""


def _decided():
    n = lib().fp4q_o_undecided()
    if n:
        raise OracleUndecided(f"oracle: {n} comparisons too close to decide without exact sums")


def inexact_count() -> int:
    """Exact-error evaluations since the last call whose sums did not stay exact (the windows
    never produce one; only the brute-force window checks may)."""
    return int(lib().fp4q_o_inexact())


def nvfp4_quantize(x, objective="sweep_mse", importance=None, S=None, hadamard16=False):
    """NVFP4 quantization of a float32 [rows, cols] array; returns a dict with packed codes
    [rows, cols/2], scale bytes [rows, cols/16], S, status and per-block diagnostics:
    p (chosen pattern), err (the exact block error E as float64; WMSE: the binary32 weighted
    accumulator), gap (runner-up's (E2 - E1) / max(E1, FLT_MIN), +inf with one candidate),
    tie (runner-up exactly equal), p2 (runner-up's pattern), nvalid (candidates).
    hadamard16: quantize the blockwise-rotated tensor (S taken over the rotated values)."""
    x = rotate16(x) if hadamard16 else _f32(x)
    rows, cols = x.shape
    nb = cols // 16
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, nb), np.uint8)
    Sarr = np.array([0.0 if S is None else S], np.float32)
    bp = np.zeros((rows, nb), np.int32)
    be = np.zeros((rows, nb), np.float64)
    bg = np.zeros((rows, nb), np.float64)
    bt = np.zeros((rows, nb), np.int32)
    b2 = np.zeros((rows, nb), np.int32)
    bn = np.zeros((rows, nb), np.int32)
    w = None if importance is None else np.ascontiguousarray(importance, np.float32)
    st = lib().fp4q_o_nvfp4_quantize(_p(x), rows, cols, cols, OBJ[objective], _p(w), int(S is not None),
                                     _p(Sarr), _p(codes), _p(scales), _p(bp), _p(be), _p(bg), _p(bt), _p(b2), _p(bn))
    if st < 0:
        raise ValueError("oracle: bad shape")
    _decided()
    return {"codes": codes, "scales": scales, "S": float(Sarr[0]), "S_f32": Sarr, "status": st,
            "p": bp, "err": be, "gap": bg, "tie": bt.astype(bool), "p2": b2, "nvalid": bn}


IF4_SWEEP = {"absmax": 0, "sweep": 1, "brute": 2}


def if4_quantize(x, S=None, hadamard16=False, sweep="absmax"):
    """IF4 codes, scale bytes (indicator in bit 7) and S.  sweep: "absmax" (the AbsMax scale),
    "sweep" (IF4 x ScaleSweep over the MSE window), "brute" (every E4M3 pattern).  Diagnostics:
    err_fp / err_int (both types' exact block errors at the chosen pattern), gap / tie (the
    runner-up over every (pattern, type) candidate)."""
    x = rotate16(x) if hadamard16 else _f32(x)
    rows, cols = x.shape
    nb = cols // 16
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, nb), np.uint8)
    Sarr = np.array([0.0 if S is None else S], np.float32)
    ef = np.zeros((rows, nb), np.float64)
    ei = np.zeros((rows, nb), np.float64)
    bg = np.zeros((rows, nb), np.float64)
    bt = np.zeros((rows, nb), np.int32)
    st = lib().fp4q_o_if4_quantize(_p(x), rows, cols, cols, IF4_SWEEP[sweep], int(S is not None), _p(Sarr),
                                   _p(codes), _p(scales), _p(ef), _p(ei), _p(bg), _p(bt))
    if st < 0:
        raise ValueError("oracle: bad shape")
    _decided()
    return {"codes": codes, "scales": scales, "S": float(Sarr[0]), "S_f32": Sarr, "status": st,
            "err_fp": ef, "err_int": ei, "gap": bg, "tie": bt.astype(bool)}


MX_SWEEP = {"rule": 0, "sweep": 1, "brute": 2}


def mxfp4_quantize(x, hadamard=False, ocp_floor=False, sweep="rule"):
    """MXFP4 codes and E8M0 scale bytes.  sweep: "rule" (the max rule, ceil or OCP floor),
    "sweep" (the MX scale sweep over e_c - 2 .. e_c), "brute" (every exponent); gap / tie: the
    near-tie statistic of the sweep modes."""
    x = _f32(x)
    rows, cols = x.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 32), np.uint8)
    bg = np.zeros((rows, cols // 32), np.float64)
    bt = np.zeros((rows, cols // 32), np.int32)
    st = lib().fp4q_o_mxfp4_quantize(_p(x), rows, cols, cols, int(hadamard), int(ocp_floor), MX_SWEEP[sweep],
                                     _p(codes), _p(scales), _p(bg), _p(bt))
    if st < 0:
        raise ValueError("oracle: bad shape")
    _decided()
    return {"codes": codes, "scales": scales, "status": st, "gap": bg, "tie": bt.astype(bool)}


def mx_block_errors(x, scales, hadamard=False):
    """Exact block errors sum (v - q 2^e)^2 (float64) of MXFP4 blocks at the exponents of `scales`."""
    x = _f32(x)
    rows, cols = x.shape
    scales = np.ascontiguousarray(scales, np.uint8)
    err = np.zeros((rows, cols // 32), np.float64)
    if lib().fp4q_o_mx_block_errors(_p(x), rows, cols, cols, int(hadamard), _p(scales), _p(err)) < 0:
        raise ValueError("oracle: bad shape")
    return err


def e2m3_value(code: int) -> float:
    return lib().fp4q_o_e2m3_value(int(code))


def e2m3_encode(y: float) -> int:
    return lib().fp4q_o_e2m3_encode(float(y))


def if6_tensor_scale(x) -> float:
    """IF6's tensor scale of a whole float32 tensor: S = RN(max|x| / 1920) (finite tensors)."""
    x = _f32(x)
    return float(lib().fp4q_o_global_scale_if6(float(np.max(np.abs(x))) if x.size else 0.0))


def if6_quantize(x, S=None):
    """IF6 (FP6 E2M3 or scaled INT6 per 16-element block, indicator in bit 7 of the E4M3 scale
    byte): packed 6-bit codes [rows, cols * 3/4], scale bytes [rows, cols/16], S = RN(amax / 1920)
    and diagnostics (both types' exact errors, runner-up gap and exact-tie flag)."""
    x = _f32(x)
    rows, cols = x.shape
    nb = cols // 16
    codes = np.zeros((rows, cols * 3 // 4), np.uint8)
    scales = np.zeros((rows, nb), np.uint8)
    Sarr = np.array([0.0 if S is None else S], np.float32)
    ef = np.zeros((rows, nb), np.float64)
    ei = np.zeros((rows, nb), np.float64)
    bg = np.zeros((rows, nb), np.float64)
    bt = np.zeros((rows, nb), np.int32)
    st = lib().fp4q_o_if6_quantize(_p(x), rows, cols, cols, int(S is not None), _p(Sarr), _p(codes), _p(scales),
                                   _p(ef), _p(ei), _p(bg), _p(bt))
    if st < 0:
        raise ValueError("oracle: bad shape")
    _decided()
    return {"codes": codes, "scales": scales, "S": float(Sarr[0]), "status": st, "err_fp": ef, "err_int": ei,
            "gap": bg, "tie": bt.astype(bool)}


def if6_dequantize(codes, scales, S, out_bf16=False):
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    rows, cols = codes.shape[0], codes.shape[1] * 4 // 3
    out = np.zeros((rows, cols), np.uint16 if out_bf16 else np.float32)
    if lib().fp4q_o_if6_dequantize(_p(codes), _p(scales), float(S), rows, cols, _p(out), int(out_bf16)) < 0:
        raise ValueError("oracle: bad shape")
    return out


def near_ties(r, threshold=1e-6):
    """The near-tie statistic of a quantizer result: among blocks with a runner-up, those whose
    runner-up is within `threshold` relative of the best ((E2 - E1) / max(E1, FLT_MIN) <
    threshold), and, separately, exact ties."""
    gap = np.asarray(r["gap"]).ravel()
    has = np.isfinite(gap) | np.asarray(r["tie"]).ravel()
    near = (gap < threshold) & has
    out = {"blocks": int(gap.size), "with_runner_up": int(has.sum()), "near": int(near.sum()),
           "exact": int(np.asarray(r["tie"]).ravel().sum())}
    out["near_frac"] = out["near"] / max(out["blocks"], 1)
    if "p2" in r:
        p, p2 = np.asarray(r["p"]).ravel(), np.asarray(r["p2"]).ravel()
        t = np.asarray(r["tie"]).ravel()
        out["exact_octave_pairs"] = int(np.sum(t & (np.abs(p2 - p) == 8)))
    return out


def dequantize(codes, scales, S, fmt, inverse_hadamard=False, out_bf16=False):
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    rows, cols = codes.shape[0], codes.shape[1] * 2
    out = np.zeros((rows, cols), np.uint16 if out_bf16 else np.float32)
    st = lib().fp4q_o_dequantize(_p(codes), _p(scales), float(S), rows, cols, FMT[fmt], int(inverse_hadamard),
                                 _p(out), int(out_bf16))
    if st < 0:
        raise ValueError("oracle: bad shape")
    return out


def tile_scales(scales) -> np.ndarray:
    """Row-major [rows][J] scale bytes -> the 1-D tiled layout block-scaled tensor-core GEMMs read
    (the library's FP4Q_F_SCALE_TILED): the matrix padded with zeros to whole 128-row x 4-column
    tiles of 512 bytes, tiles in row-major order over (row / 128, column / 4), and inside a tile
    the byte of row r, column c at 16 * (r % 32) + 4 * ((r // 32) % 4) + c % 4.  Written as the
    plain element-by-element placement."""
    scales = np.asarray(scales, np.uint8)
    rows, J = scales.shape
    rt, jt = (rows + 127) // 128, (J + 3) // 4
    out = np.zeros(rt * 128 * jt * 4, np.uint8)
    for r in range(rows):
        for c in range(J):
            off = (r // 128) * (jt * 512) + (c // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + c % 4
            out[off] = scales[r, c]
    return out


def nvfp4_gemm(a_codes, a_scales, Sa, b_codes, b_scales, Sb):
    """D[m][n] = Sa * Sb * sum_k qa[m][k] e(pa[m][k/16]) qb[n][k] e(pb[n][k/16]) in float64: the
    product of two NVFP4 operands stored with K contiguous (codes [rows][K/2], row-major scale
    bytes [rows][K/16]), every element value q * e(p) formed from the oracle's own code tables.
    Each term is exact in float64 and the sums are a float64 matmul."""
    def values(codes, scales):
        codes = np.asarray(codes, np.uint8)
        rows, half = codes.shape
        q = np.empty((rows, 2 * half), np.float64)
        tab = np.array([lib().fp4q_o_e2m1_value(c) for c in range(16)], np.float64)
        q[:, 0::2] = tab[codes & 0xF]
        q[:, 1::2] = tab[codes >> 4]
        e = np.array([lib().fp4q_o_e4m3_value(p) for p in range(128)], np.float64)
        sc = e[np.asarray(scales, np.uint8) & 0x7F]
        return q * np.repeat(sc, 16, axis=1)
    return float(Sa) * float(Sb) * (values(a_codes, a_scales) @ values(b_codes, b_scales).T)


def encode(x, kind: str) -> np.ndarray:
    """Element codec over an fp32 array: kind "e2m1" gives the 4-bit E2M1 code of each value
    (sign << 3 | magnitude index), "e4m3" the E4M3FN byte (sign in bit 7); both round to
    nearest with ties to even and saturate."""
    x = np.ascontiguousarray(x, np.float32).ravel()
    out = np.empty(x.size, np.uint8)
    st = lib().fp4q_o_encode(_p(x), x.size, {"e2m1": 0, "e4m3": 1}[kind], _p(out))
    if st != 0:
        raise ValueError(kind)
    return out


def mxfp4_gemm(a_codes, a_scales, b_codes, b_scales):
    """D[m][n] = sum_k qa[m][k] 2^(sa[m][k/32]-127) qb[n][k] 2^(sb[n][k/32]-127) in float64: the
    product of two MXFP4 operands stored with K contiguous (codes [rows][K/2], row-major E8M0
    scale bytes [rows][K/32]); MXFP4 has no tensor scale.  Element values from the oracle's own
    E2M1 table times the E8M0 power of two (byte 0xFF, E8M0's NaN, gives NaN).  Each term is
    exact in float64 (the products span far fewer than 2^10 binades here) and the sums are a
    float64 matmul."""
    def values(codes, scales):
        codes = np.asarray(codes, np.uint8)
        rows, half = codes.shape
        q = np.empty((rows, 2 * half), np.float64)
        tab = np.array([lib().fp4q_o_e2m1_value(c) for c in range(16)], np.float64)
        q[:, 0::2] = tab[codes & 0xF]
        q[:, 1::2] = tab[codes >> 4]
        e = np.array([np.ldexp(1.0, b - 127) if b != 0xFF else np.nan for b in range(256)], np.float64)
        return q * np.repeat(e[np.asarray(scales, np.uint8)], 32, axis=1)
    return values(a_codes, a_scales) @ values(b_codes, b_scales).T


def f32_to_bf16(x) -> np.ndarray:
    """The oracle's own float32 -> bf16 rounding (nearest, ties to even; NaN stays NaN), as bit
    patterns: the reference for the bf16 dequantize output."""
    x = np.ascontiguousarray(x, np.float32).ravel()
    out = np.empty(x.size, np.uint16)
    lib().fp4q_o_f32_to_bf16(_p(x), x.size, _p(out))
    return out


def widen_bf16(bits) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact), the oracle's own input widening."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)
