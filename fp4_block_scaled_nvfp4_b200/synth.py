"""Seeded synthetic inputs shaped like the LLM weights and activations the pages quantize.

This module is the only code shared by the CUDA path's tests/bench and the CPU oracle's
tests.  It holds no quantization arithmetic: it draws numbers and rounds them to the
storage dtype, nothing else.

Generator (counter based, so any element can be regenerated on its own):
    word(seed, stream, i) = mix(mix(seed * G ^ stream * H) + (i + 1) * G)
    mix = the SplitMix64 output finalizer (Steele, Lea & Flood, "Fast splittable
          pseudorandom number generators", OOPSLA 2014), G = 0x9E3779B97F4A7C15.
    uniform in (0, 1) = ((word >> 11) + 0.5) * 2**-53.
Transforms (all in float64, then rounded once to float32, then to bf16 by
round-to-nearest-even when the config stores bf16):
    normal       Box-Muller on a pair of uniforms from two streams
    Laplace(s)   inverse CDF with scale b = s / sqrt(2) (standard deviation s)
    Student-t(n) Z / sqrt(chi2_n / n); chi2_4 = -2 ln(u1 u2), chi2_5 = chi2_4 + Z'^2
    lognormal    exp(mu + sigma * Z)

The five workloads follow the quantization configurations the pages evaluate on
(weights and activations of Llama/Qwen-sized linear layers): see CONFIGS.
"""
from __future__ import annotations

import numpy as np

_G = np.uint64(0x9E3779B97F4A7C15)
_H = np.uint64(0xD1B54A32D192ED03)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * _M1
    z = z ^ (z >> np.uint64(27))
    z = z * _M2
    return z ^ (z >> np.uint64(31))


def uniform(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """Uniforms in (0,1) for counters start .. start+count-1 of (seed, stream)."""
    with np.errstate(over="ignore"):
        key = _mix(np.array([np.uint64(seed) * _G ^ np.uint64(stream) * _H], dtype=np.uint64))[0]
        idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        w = _mix(key + idx * _G)
    return ((w >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normal(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    u1 = uniform(seed, stream, start, count)
    u2 = uniform(seed, stream + 1, start, count)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def laplace(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """Unit-variance Laplace."""
    u = uniform(seed, stream, start, count) - 0.5
    b = 1.0 / np.sqrt(2.0)
    return -b * np.sign(u) * np.log1p(-2.0 * np.abs(u))


def student_t(seed: int, stream: int, start: int, count: int, df: int) -> np.ndarray:
    z = normal(seed, stream, start, count)
    if df not in (4, 5):
        raise ValueError("student_t: df 4 or 5")
    chi = -2.0 * np.log(uniform(seed, stream + 2, start, count) * uniform(seed, stream + 3, start, count))
    if df == 5:
        chi = chi + normal(seed, stream + 4, start, count) ** 2
    return z / np.sqrt(chi / df)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _permutation(seed: int, stream: int, n: int) -> np.ndarray:
    return np.argsort(uniform(seed, stream, 0, n), kind="stable")


def _channel_std(seed: int, stream: int, cols: int, sigma: float, n_out: int, out_mult: float):
    std = np.exp(sigma * normal(seed, stream, 0, cols))
    std[_permutation(seed, stream + 2, cols)[:n_out]] *= out_mult
    return std


def _fill(rows: int, cols: int, fn) -> np.ndarray:
    """Evaluate fn(start, count) -> float64 values over the row-major index space in chunks."""
    out = np.empty(rows * cols, dtype=np.float32)
    n = rows * cols
    for s in range(0, n, _CHUNK):
        c = min(_CHUNK, n - s)
        out[s:s + c] = fn(s, c).astype(np.float32)
    return out.reshape(rows, cols)


# ----------------------------------------------------------------------------------------
# Workloads.  Each returns a dict: x (float32 array, or uint16 bf16 bits when dtype='bf16'),
# dtype, rows, cols, and for WMSE the float32 importance vector.
# ----------------------------------------------------------------------------------------

def cfg1(rows=256, cols=1024, seed=0):
    """fp32 weight, 0.02*N(0,1); each entry independently (p=0.001) multiplied by 20."""
    def fn(s, c):
        v = 0.02 * normal(seed, 10, s, c)
        hit = uniform(seed, 20, s, c) < 0.001
        return np.where(hit, v * 20.0, v)
    return {"name": "cfg1", "dtype": "f32", "rows": rows, "cols": cols, "x": _fill(rows, cols, fn)}


def importance_from_activations(seed: int, tokens: int, cols: int) -> np.ndarray:
    """w_j = mean over tokens of a_tj^2 for a Gaussian activation matrix whose channel std is
    lognormal(0,1) with 8 channels (seeded permutation) scaled by 50; fp64 then fp32."""
    std = _channel_std(seed, 30, cols, 1.0, 8, 50.0)
    acc = np.zeros(cols, dtype=np.float64)
    step = max(1, _CHUNK // cols)
    for t0 in range(0, tokens, step):
        t = min(step, tokens - t0)
        a = normal(seed, 40, t0 * cols, t * cols).reshape(t, cols) * std
        a = a.astype(np.float32).astype(np.float64)
        acc += (a * a).sum(axis=0)
    return (acc / tokens).astype(np.float32)


def cfg2(rows=14336, cols=4096, seed=1, tokens=2048):
    """bf16 weight 0.02*t5 with per-input-column importance from a synthetic activation matrix."""
    x = _fill(rows, cols, lambda s, c: 0.02 * student_t(seed, 10, s, c, 5))
    return {"name": "cfg2", "dtype": "bf16", "rows": rows, "cols": cols, "x": f32_to_bf16_bits(x),
            "importance": importance_from_activations(seed, tokens, cols)}


def _activation(rows, cols, seed, sigma, n_out, out_mult):
    std = _channel_std(seed, 30, cols, sigma, n_out, out_mult)

    def fn(s, c):
        col = np.arange(s, s + c, dtype=np.int64) % cols
        return laplace(seed, 10, s, c) * std[col]
    return _fill(rows, cols, fn)


def cfg3(rows=8192, cols=4096, seed=2):
    """bf16 activations: Laplace within channel, channel std lognormal(0,1.5), 8 channels x50."""
    x = _activation(rows, cols, seed, 1.5, 8, 50.0)
    return {"name": "cfg3", "dtype": "bf16", "rows": rows, "cols": cols, "x": f32_to_bf16_bits(x)}


def cfg4(rows=4096, cols=14336, seed=3):
    """bf16 weight 0.02*t4 (IF4 workload)."""
    x = _fill(rows, cols, lambda s, c: 0.02 * student_t(seed, 10, s, c, 4))
    return {"name": "cfg4", "dtype": "bf16", "rows": rows, "cols": cols, "x": f32_to_bf16_bits(x)}


def cfg5(rows=16384, cols=8192, seed=4):
    """bf16 activations: Laplace, channel std lognormal(0,1.5), 16 channels x100 (MXFP4)."""
    x = _activation(rows, cols, seed, 1.5, 16, 100.0)
    return {"name": "cfg5", "dtype": "bf16", "rows": rows, "cols": cols, "x": f32_to_bf16_bits(x)}


CONFIGS = {"cfg1": cfg1, "cfg2": cfg2, "cfg3": cfg3, "cfg4": cfg4, "cfg5": cfg5}


def make(name: str, rows: int | None = None, cols: int | None = None, seed: int | None = None):
    """Build a workload; rows/cols override the full size (same distribution, smaller tensor),
    seed another draw of the same distribution."""
    fn = CONFIGS[name]
    kw = {} if seed is None else {"seed": seed}
    if rows is not None:
        kw["rows"] = rows
    if cols is not None:
        kw["cols"] = cols
    return fn(**kw)


def as_f32(w) -> np.ndarray:
    """Float32 view of a workload's x (exact widening for bf16)."""
    return w["x"] if w["dtype"] == "f32" else bf16_bits_to_f32(w["x"])
