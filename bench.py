#!/usr/bin/env python
"""Throughput benchmark: NVFP4 ScaleSweep-MSE dynamic activation quantization of a bf16
8192x4096 activation tensor (amax pass + sweep quantization), on B200.

One step = the whole hot path over one tensor: tensor scale S = max|x|/1536 (amax kernel),
then base scale, 11-candidate sweep, RTN, error, argmin, nibble pack and scale write (sweep
kernel).  value = algorithmic bytes per step (2 B/element read + 0.5 B codes + 1/16 B scales
+ 4 B S) x steps / device time.  Inputs rotate over distinct buffer sets whose total exceeds
the 126 MB L2, so every step reads its input from HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU (torchrun): every rank quantizes its own tensor (weak scaling, no collective on
the data path); time = max over ranks of the device time.
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {
    # name: (synth config, fmt, objective, description)
    "cfg3": ("cfg3", "nvfp4", "sweep_mse",
             "NVFP4 ScaleSweep-MSE dynamic activation quantization, bf16 8192x4096 (tokens x hidden), "
             "Laplace values, lognormal(0,1.5) channel std, 8 outlier channels x50, dynamic S"),
    "cfg2": ("cfg2", "nvfp4", "sweep_wmse",
             "NVFP4 ScaleSweep-WMSE, bf16 weight 14336x4096, 0.02*t5, per-input-column importance"),
    "cfg4": ("cfg4", "if4", None, "IF4 per-block FP4/INT4 selection, bf16 weight 4096x14336, 0.02*t4"),
    "cfg4s": ("cfg4", "if4", "if4_sweep",
              "IF4 x ScaleSweep (scale and FP4/INT4 type chosen together over offsets [-3,+7]), bf16 weight "
              "4096x14336, 0.02*t4"),
    "cfg5": ("cfg5", "mxfp4", None, "MXFP4, bf16 activations 16384x8192"),
    "cfg5h": ("cfg5", "mxfp4_had", None, "MXFP4 after 32x32 block Hadamard, bf16 activations 16384x8192"),
    "cfg5s": ("cfg5", "mxfp4", "mx_sweep",
              "MXFP4 with the MX scale sweep (E8M0 exponents e_c-2..e_c by block MSE), bf16 activations 16384x8192"),
    "cfg5hs": ("cfg5", "mxfp4_had", "mx_sweep",
               "MXFP4 with the MX scale sweep after 32x32 block Hadamard, bf16 activations 16384x8192"),
    "cfg3h": ("cfg3", "nvfp4_had", "sweep_mse",
              "NVFP4 ScaleSweep-MSE on 16x16 block-Hadamard-rotated blocks, bf16 activations 8192x4096, "
              "dynamic S of the rotated tensor"),
    "cfg4h": ("cfg4", "if4_had", None, "IF4 on 16x16 block-Hadamard-rotated blocks, bf16 weight 4096x14336"),
    "cfg4i6": ("cfg4", "if6", None,
               "IF6 per-block FP6 (E2M3) / scaled INT6 selection, 6-bit codes, S = amax/1920, bf16 weight "
               "4096x14336, 0.02*t4"),
    # the NVFP4 operator ScaleSweep measures its overhead against: AbsMax on the same tensor
    "cfg3_absmax": ("cfg3", "nvfp4", "absmax",
                    "NVFP4 AbsMax (one scale per block, no search) dynamic activation quantization, bf16 8192x4096, "
                    "the same tensor as the ScaleSweep-MSE line"),
}
# Dequantization (codes + scales + S -> fp32), on the quantizer's own output of the same tensors
DEQUANT_WORKLOADS = {
    "dq_nvfp4": ("cfg3", "nvfp4", "sweep_mse", "NVFP4 dequantize to fp32 of the 8192x4096 activation tensor's "
                                               "ScaleSweep-MSE codes and scales"),
    "dq_mxfp4": ("cfg5", "mxfp4", None, "MXFP4 dequantize to fp32 of the 16384x8192 activation tensor's codes and "
                                        "E8M0 scales"),
}
DEQUANT_METRIC = "dequantize GB/s (fp32 out) and % of B200 HBM peak, 1 GPU"
METRIC = "quantize GB/s (input bf16) and % of B200 HBM peak, 1 GPU, vs CPU oracle"
# The consumer of the quantized operands (--workload gemm): the block-scaled NVFP4 GEMM on the
# tcgen05 tensor cores, activations [M][K] (the 8192x4096 activation workload) times a weight
# [N][K] (Llama-3-8B-shaped MLP up-projection, 14336x4096, Student-t weights), K contiguous.
GEMM_METRIC = "NVFP4 block-scaled GEMM TFLOP/s (tcgen05), 1 GPU"
GEMM_MX_METRIC = "MXFP4 block-scaled GEMM TFLOP/s (tcgen05), 1 GPU"
GEMM_DYN_METRIC = ("NVFP4 dynamic-activation GEMM TFLOP/s (amax + ScaleSweep quantize of the activation, then the "
                   "tcgen05 GEMM), 1 GPU")
# gemm / gemm_mx: the GEMM alone on pre-quantized operands (fp32 D); gemm_bf16: the same with bf16 D;
# gemm_dyn: each step quantizes the bf16 activation (amax + ScaleSweep-MSE, tiled scales) and runs the
# NVFP4 GEMM against the pre-quantized weight with bf16 D
GEMM_WORKLOADS = ("gemm", "gemm_mx", "gemm_bf16", "gemm_dyn")
GEMM_SHAPE = (8192, 14336, 4096)
# Arithmetic the method itself needs per element for the ALU-bound searches: per candidate
# scale one multiply (x/s), one E2M1 rounding, and the two accumulations of the exact block
# error (sum q^2 and sum |x| q) -- for WMSE the binary32 residual, weight multiply and fused
# square-accumulate instead -- over 11 (MSE) or 16 (WMSE) candidates, plus the block maximum and
# the final multiply + rounding.
ALU_OPS_PER_ELEMENT = {"sweep_mse": 11 * 4 + 3, "sweep_wmse": 16 * 5 + 3,
                       # IF4 x ScaleSweep: per candidate the FP4 four plus the INT4 pre-scale,
                       # rounding, clamp, the two accumulations and the code lookup
                       "if4_sweep": 11 * (4 + 6) + 3}
# the 16-point rotation adds four butterfly additions and one multiplication per element
ROTATION_OPS_PER_ELEMENT = 4 + 1


def split_fmt(fmt):
    """'nvfp4_had' -> ('nvfp4', True); MXFP4's rotated form keeps its own name."""
    if fmt.endswith("_had") and not fmt.startswith("mxfp4"):
        return fmt[:-4], True
    return fmt, False
L2_BYTES = 126 * 2 ** 20


def code_bytes(n, fmt):
    """Bytes of packed element codes for n elements: 4 bits (FP4 formats) or 6 bits (IF6)."""
    return n * 3 // 4 if fmt == "if6" else n // 2


def algorithmic_bytes(rows, cols, fmt, in_bytes=2, wmse=False):
    B = 32 if fmt.startswith("mxfp4") else 16
    n = rows * cols
    b = n * in_bytes + code_bytes(n, fmt) + n // B
    if not fmt.startswith("mxfp4"):
        b += 4
    if wmse:
        b += 4 * cols
    return b


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


QUANT_SOURCES = ("fp4_block_scaled_nvfp4_b200/csrc/fp4q.cu", "fp4_block_scaled_nvfp4_b200/csrc/fp4q_device.cuh")
GEMM_SOURCES = ("fp4_block_scaled_nvfp4_b200/csrc/fp4q_gemm.cu",)


def kernel_source_hash(files=QUANT_SOURCES):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_key, files=QUANT_SOURCES):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current
    kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel_key)
    if not e or e.get("source_hash") != kernel_source_hash(files):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Polls NVML for SM clock and throttle reasons while the timed region runs."""

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = str(torch.cuda.get_device_properties(index).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: report no samples
            self.nv = None

    def _run(self):
        nv = self.nv
        names = {
            getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8): "hw_slowdown",
            getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40): "hw_thermal_slowdown",
            getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20): "sw_thermal_slowdown",
            getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4): "sw_power_cap",
            getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80): "hw_power_brake_slowdown",
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in names.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                break
            time.sleep(0.002)

    def __enter__(self):
        if self.nv:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        return {"sm_mhz": (statistics.median(self.samples) if self.samples else None), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml polled every ~2 ms"}


def device_tensor_from_bits(bits, torch):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def blas_threads() -> int:
    """Threads of the BLAS behind numpy's float64 matmul (the oracle GEMM's one library step)."""
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def _oracle_rows(args):
    """One worker task of the all-cores baseline: the oracle on a contiguous row shard."""
    import oracle as O
    xs, fmt, obj, imp = args
    base, had16 = split_fmt(fmt)
    if base == "nvfp4":
        O.nvfp4_quantize(xs, obj, importance=imp, hadamard16=had16)
    elif base == "if4":
        O.if4_quantize(xs, hadamard16=had16, sweep="sweep" if obj == "if4_sweep" else "absmax")
    elif base == "if6":
        O.if6_quantize(xs)
    else:
        O.mxfp4_quantize(xs, hadamard=fmt.endswith("had"), sweep="sweep" if obj == "mx_sweep" else "rule")
    return xs.shape[0]


def cpu_baseline_all_cores(w, fmt, obj, budget_s=6.0, cpu_budget_s=30.0):
    """The same oracle on row shards over the host cores this process may run on (at most 128):
    one process per core (started with spawn), each quantizing a contiguous shard of rows (rows
    are independent); whole passes over the tensor until about min(budget_s, cpu_budget_s /
    cores) of wall time (at least one pass), so that the sample stays near cpu_budget_s of CPU
    work."""
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor
    import oracle as O
    O.lib()   # built once here, so the workers only load it
    x = O.widen_bf16(w["x"]) if w["dtype"] == "bf16" else w["x"]
    rows, cols = x.shape
    n = max(1, min(128, len(os.sched_getaffinity(0))))
    budget_s = min(budget_s, cpu_budget_s / n)
    step = -(-rows // n)
    shards = [(np.ascontiguousarray(x[a:a + step]), fmt, obj, w.get("importance")) for a in range(0, rows, step)]
    # a worker that dies raises BrokenProcessPool here instead of leaving the map waiting
    with ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn")) as pool:
        list(pool.map(_oracle_rows, shards))   # start-up and first touch, untimed
        done, passes, t0 = 0, 0, time.perf_counter()
        while passes == 0 or time.perf_counter() - t0 < budget_s:
            done += sum(pool.map(_oracle_rows, shards))
            passes += 1
        dt = time.perf_counter() - t0
    nbytes = algorithmic_bytes(done, cols, fmt, wmse=(obj == "sweep_wmse"))
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": n, "kind": "oracle",
            "sample": f"{passes} pass(es) over all {rows} rows of the {rows}x{cols} tensor in {len(shards)} row "
                      f"shards (S over each shard's rows) on {n} processes, {dt:.1f} s"}


def cpu_baseline(w, fmt, obj, budget_s=12.0, S=None, gpu=None):
    """The oracle as it stands, single-threaded, on whole rows of the same tensor until about
    budget_s of CPU time has been spent; returns its throughput in the same unit.  With S (the
    whole tensor's scale) and gpu = (codes, scales) of the CUDA path for the whole tensor, the
    same oracle run also checks those rows: mismatching blocks, the near-tie statistic and the
    reconstruction MSE of both sides (dequantized with the oracle's own decoder)."""
    import oracle as O
    x = O.widen_bf16(w["x"]) if w["dtype"] == "bf16" else w["x"]
    rows, cols = x.shape
    chunk = max(1, min(rows, 256))
    done, t0 = 0, time.perf_counter()
    imp = w.get("importance")
    base, had16 = split_fmt(fmt)
    results = []
    while done < rows and time.perf_counter() - t0 < budget_s:
        xs = x[done:done + chunk]
        if base == "nvfp4":
            r = O.nvfp4_quantize(xs, obj, importance=imp, hadamard16=had16, S=S)
        elif base == "if4":
            r = O.if4_quantize(xs, hadamard16=had16, sweep="sweep" if obj == "if4_sweep" else "absmax", S=S)
        elif base == "if6":
            r = O.if6_quantize(xs, S=S)
        else:
            r = O.mxfp4_quantize(xs, hadamard=fmt.endswith("had"), sweep="sweep" if obj == "mx_sweep" else "rule")
        results.append(r)
        done += xs.shape[0]
    dt = time.perf_counter() - t0
    nbytes = algorithmic_bytes(done, cols, fmt, wmse=(obj == "sweep_wmse"))
    out = {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
           "sample": f"{done} of {rows} rows of the {rows}x{cols} tensor ({done * cols} elements), "
                     f"S {'of the whole tensor' if S is not None else 'over the sampled rows'}, {dt:.1f} s single-threaded"}
    if gpu is not None:
        oc = np.concatenate([r["codes"] for r in results])
        osc = np.concatenate([r["scales"] for r in results])
        gc, gsc = gpu[0][:done], gpu[1][:done]
        B = 32 if fmt.startswith("mxfp4") else 16
        cb = code_bytes(B, base)   # code bytes per block
        bad = (gsc != osc) | (gc.reshape(done, -1, cb) != oc.reshape(done, -1, cb)).any(axis=2)
        near = O.near_ties({k: np.concatenate([r[k] for r in results]) for k in ("gap", "tie")})
        dfmt = "mxfp4" if fmt.startswith("mxfp4") else base
        xr = O.rotate16(x[:done]) if had16 else x[:done]
        if fmt.startswith("mxfp4") and fmt.endswith("had"):
            xr = np.stack([O.hadamard32(v) for v in x[:done].reshape(-1, 32)]).reshape(done, cols)
        Sd = 0.0 if S is None else S
        deq = (lambda c, sc: O.if6_dequantize(c, sc, Sd)) if base == "if6" else (lambda c, sc: O.dequantize(c, sc, Sd, dfmt))
        mse_o = float(np.mean((xr.astype(np.float64) - deq(oc, osc).astype(np.float64)) ** 2))
        mse_g = float(np.mean((xr.astype(np.float64) - deq(gc, gsc).astype(np.float64)) ** 2))
        out["parity"] = {"rows_checked": done, "blocks_checked": int(bad.size), "mismatching_blocks": int(bad.sum()),
                         "bit_exact": bool(not bad.any()),
                         "near_tie_frac": round(near["near_frac"], 6), "near_tie_blocks": near["near"],
                         "exact_tie_blocks": near["exact"],
                         "recon_mse": mse_g, "recon_mse_oracle": mse_o,
                         "recon_mse_rel_diff": (abs(mse_g - mse_o) / mse_o) if mse_o > 0 else 0.0,
                         "how": "the CUDA path's codes and scales of the sampled rows against the oracle's at the "
                                "whole tensor's S; near ties: runner-up within 1e-6 relative of the best block error"}
    return out


def run_reference(args, rank, world):
    """The oracle on the host cores as the reference arm: K steps, each a bounded row sample."""
    if args.workload in GEMM_WORKLOADS:
        return run_reference_gemm(args, rank, world)
    if args.workload in DEQUANT_WORKLOADS:
        return run_reference_dequant(args, rank, world)
    cfg, fmt, obj, desc = WORKLOADS[args.workload]
    from fp4_block_scaled_nvfp4_b200 import synth
    import oracle as O
    if rank != 0:
        return
    w = synth.make(cfg)
    x = O.widen_bf16(w["x"]) if w["dtype"] == "bf16" else w["x"]
    rows, cols = x.shape
    sample_rows = 16
    imp = w.get("importance")
    base, had16 = split_fmt(fmt)

    def step(i):
        r0 = (i * sample_rows) % rows
        xs = x[r0:r0 + sample_rows]
        if base == "nvfp4":
            O.nvfp4_quantize(xs, obj, importance=imp, hadamard16=had16)
        elif base == "if4":
            O.if4_quantize(xs, hadamard16=had16, sweep="sweep" if obj == "if4_sweep" else "absmax")
        elif base == "if6":
            O.if6_quantize(xs)
        else:
            O.mxfp4_quantize(xs, hadamard=fmt.endswith("had"), sweep="sweep" if obj == "mx_sweep" else "rule")

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = time.perf_counter() - t0
    nbytes = algorithmic_bytes(sample_rows, cols, fmt, wmse=(obj == "sweep_wmse")) * args.steps
    val = nbytes / dt / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": desc, "rows": rows, "cols": cols, "input_dtype": w["dtype"],
                       "step_sample_rows": sample_rows},
            "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": f"{sample_rows} rows per step of the {rows}x{cols} tensor"},
            "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_reference_dequant(args, rank, world):
    """The oracle's decoder on the host as the reference arm: each step 64 rows."""
    cfg, fmt, obj, desc = DEQUANT_WORKLOADS[args.workload]
    from fp4_block_scaled_nvfp4_b200 import synth
    import oracle as O
    if rank != 0:
        return
    w = synth.make(cfg)
    rows, cols = w["rows"], w["cols"]
    sample = 64
    x = O.widen_bf16(w["x"][:sample * 4])
    r = O.mxfp4_quantize(x) if fmt == "mxfp4" else O.nvfp4_quantize(x, obj)
    S = r.get("S", 0.0)
    B = 32 if fmt == "mxfp4" else 16

    def step(i):
        a = (i % 4) * sample
        O.dequantize(r["codes"][a:a + sample], r["scales"][a:a + sample], S, fmt)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = time.perf_counter() - t0
    per_row = cols // 2 + cols // B + cols * 4
    val = sample * per_row * args.steps / dt / 1e9
    line = {"impl": "reference", "metric": DEQUANT_METRIC, "value": round(val, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": desc, "rows": rows, "cols": cols, "step_sample_rows": sample},
            "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": f"{sample} rows per step of the {rows}x{cols} tensor"},
            "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world):
    import torch
    import torch.distributed as dist

    import fp4_block_scaled_nvfp4_b200 as fq
    from fp4_block_scaled_nvfp4_b200 import synth

    cfg, fmt, obj, desc = WORKLOADS[args.workload]
    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    fq.lib()

    w = synth.make(cfg)
    rows, cols = w["rows"], w["cols"]
    x_host = device_tensor_from_bits(w["x"], torch)
    in_bytes = x_host.numel() * 2
    alg = algorithmic_bytes(rows, cols, fmt, wmse=(obj == "sweep_wmse"))
    out_bytes = code_bytes(rows * cols, fmt) + rows * cols // (32 if fmt.startswith("mxfp4") else 16)
    nsets = max(2, int(np.ceil(3.0 * L2_BYTES / (in_bytes + out_bytes))))
    xs = [x_host.to(dev) for _ in range(nsets)]
    base, had16 = split_fmt(fmt)
    outs = [fq.alloc_outputs(rows, cols, "mxfp4" if fmt.startswith("mxfp4") else base, dev) for _ in range(nsets)]
    imp = torch.from_numpy(w["importance"]).to(dev) if obj == "sweep_wmse" else None
    wss = [fq.new_workspace(dev) for _ in range(nsets)]   # one per buffer set: steps may overlap
    launches_per_step = 0

    def amax(s):
        fq.global_scale(xs[s], out=outs[s][2], workspace=wss[s], hadamard16=had16)
        return 1

    def quant(s):
        c, sc, g = outs[s]
        if fmt.startswith("mxfp4"):   # one kernel, no tensor scale
            if fmt.endswith("had"):
                fq.hadamard_quantize(xs[s], out=(c, sc, None), workspace=wss[s], mx_sweep=(obj == "mx_sweep"))
            else:
                fq.quantize(xs[s], "mxfp4", out=(c, sc, None), workspace=wss[s], mx_sweep=(obj == "mx_sweep"))
        else:
            fq.quantize(xs[s], base, obj or "absmax", importance=imp, global_scale=g, out=(c, sc, g),
                        workspace=wss[s], hadamard16=had16, if4_sweep=(obj == "if4_sweep"))
        return 1

    if fmt == "if6":   # its own tensor scale (amax / 1920): one public call runs the amax pass and the quantizer
        def quant(s):
            c, sc, g = outs[s]
            fq.quantize(xs[s], "if6", out=(c, sc, g), workspace=wss[s])
            return 2

    def step(s):
        return (0 if fmt.startswith("mxfp4") or fmt == "if6" else amax(s)) + quant(s)

    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            launches_per_step = step(i % nsets)
    torch.cuda.synchronize()

    def capture(body):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            body()
        return g

    # CUDA graphs without timing nodes inside (an event recorded between two kernels of a graph
    # costs several microseconds): one per buffer set, for a remainder of steps, and one that
    # runs every set once in turn
    graphs = [capture(lambda s=s: step(s)) for s in range(nsets)]
    two_pass = not (fmt.startswith("mxfp4") or fmt == "if6")
    side = torch.cuda.Stream(device=dev)

    def pipelined_cycle():
        # every set's amax + quantize in turn, with the next set's amax pass (HBM-bound) on a
        # second stream under this set's quantize (compute-bound); each quantize waits for its
        # own set's amax, and each amax for the quantize two sets back (at most one of each runs)
        done_amax, done_quant = [], []
        fork = torch.cuda.Event()
        fork.record(stream)
        side.wait_event(fork)
        for s in range(nsets):
            with torch.cuda.stream(side):
                if s >= 2:
                    side.wait_event(done_quant[s - 2])
                amax(s)
                e = torch.cuda.Event()
                e.record(side)
                done_amax.append(e)
            stream.wait_event(done_amax[s])
            quant(s)
            e = torch.cuda.Event()
            e.record(stream)
            done_quant.append(e)
        join = torch.cuda.Event()
        join.record(side)
        stream.wait_event(join)

    cycle = capture(pipelined_cycle if two_pass else (lambda: [step(s) for s in range(nsets)]))
    serial_cycle = capture(lambda: [step(s) for s in range(nsets)]) if two_pass else cycle
    with torch.cuda.stream(stream):
        for s in range(nsets):
            graphs[s].replay()
        cycle.replay()
        serial_cycle.replay()
    torch.cuda.synchronize()
    full_cycles, rest = divmod(args.steps, nsets)

    # the batched form (NVFP4 / IF4 without rotation or WMSE): the K steps' tensors, the buffer
    # sets in turn, in one fp4q_quantize_batch call -- one amax kernel, then K quantize kernels,
    # each also taking the next tensor's amax
    fused = two_pass and not had16 and obj != "sweep_wmse"
    if fused:
        def plan_over(k):
            return fq.BatchPlan([xs[i % nsets] for i in range(k)], base, obj or "absmax",
                                outs=[outs[i % nsets] for i in range(k)], workspace=wss[0],
                                if4_sweep=(obj == "if4_sweep"))
        plan = plan_over(args.steps)
        with torch.cuda.stream(stream):
            plan_over(max(args.warmup, nsets + 1))(stream)
        torch.cuda.synchronize()
        batch_graph = capture(lambda: plan(stream))   # the K + 1 launches as one CUDA graph
        with torch.cuda.stream(stream):
            batch_graph.replay()
        torch.cuda.synchronize()

    def timed(run):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            start.record()
            run()
            end.record()
        end.synchronize()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        t_ms = start.elapsed_time(end)
        if world > 1:
            t = torch.tensor([t_ms], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            t_ms = float(t.item())
        return t_ms

    def run_cycles():
        for _ in range(full_cycles):
            cycle.replay()
        for i in range(rest):
            graphs[i].replay()

    with ClockSampler(local) as clk:
        ms = timed(batch_graph.replay if fused else run_cycles)
    two_stream_ms = timed(run_cycles) if fused else None

    # the same steps with no overlap between them (one stream, amax then quantize per step)
    def run_serial():
        for _ in range(full_cycles):
            serial_cycle.replay()
        for i in range(rest):
            graphs[i].replay()

    serial_ms = timed(run_serial) if two_pass else ms

    # per-kernel launch durations for the roofline: the same launches, one kernel kind at a
    # time (every buffer set in turn, so reads still come from HBM), timed with CUDA events on
    # the launching stream over kernel_reps launches
    kernel_reps = max(nsets, (min(args.steps, 400) // nsets) * nsets)

    def time_kernel(fn):
        g = capture(lambda: [fn(s) for s in range(nsets)])
        with torch.cuda.stream(stream):
            g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record()
            for _ in range(kernel_reps // nsets):
                g.replay()
            b.record()
        b.synchronize()
        return a.elapsed_time(b) / kernel_reps

    t_q = time_kernel(quant)
    t_amax = None if not two_pass else time_kernel(amax)

    # per-step distribution: up to 200 steps, each between its own pair of CUDA events on the
    # stream (the buffer sets in turn)
    n_dist = max(1, min(args.steps, 200))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_dist)]
    with torch.cuda.stream(stream):
        for i, (a, b) in enumerate(evs):
            a.record()
            graphs[i % nsets].replay()
            b.record()
    torch.cuda.synchronize()
    per_step = sorted(a.elapsed_time(b) for a, b in evs)
    pick = lambda q: round(per_step[min(n_dist - 1, int(q * (n_dist - 1) + 0.5))], 5)
    step_dist = {"p10": pick(0.1), "p50": pick(0.5), "p90": pick(0.9), "steps": n_dist,
                 "how": "each step between its own CUDA events on the launching stream"}

    # every buffer set's status word must be clean
    st = next((v for v in (fq.read_device_status(w_) for w_ in wss) if v), 0)

    # end to end through the public API with host buffers: every step copies its input in
    # from pinned memory, quantizes, and copies codes, scales and S out; two staging sets let
    # one step's input copy overlap the previous step's kernels and output copies
    e2e_steps = max(1, min(args.steps, 50))
    x_pin = x_host.pin_memory()
    hq = fq.HostQuantizer(rows, cols, fmt, obj or "absmax", importance=imp, dtype=x_host.dtype, depth=2,
                          device=dev, mx_sweep=(obj == "mx_sweep"), if4_sweep=(obj == "if4_sweep"))
    host_outs = [fq.alloc_host_outputs(rows, cols, fmt) for _ in range(2)]
    for i in range(3):
        hq(x_pin, host_outs[i % 2])
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(hq.copy_stream)
    hq.compute_stream.wait_event(e0)
    for i in range(e2e_steps):
        hq(x_pin, host_outs[i % 2])
    e1.record(hq.compute_stream)
    e1.synchronize()
    e2e_launches = fq.last_launch_count()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if world > 1:
        t = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    h2d = in_bytes
    d2h = out_bytes + (4 if not fmt.startswith("mxfp4") else 0)

    if rank != 0:
        return
    peak, peak_src = load_peaks()
    per_step_ms = ms / args.steps
    value = alg * args.steps * world / (ms * 1e-3) / 1e9
    tq = t_q
    kernel_key = f"{args.workload}:quantize"
    kernel_name = "quantize (" + (obj or fmt) + ")"
    t_fused = None
    if fused:
        # the dominant kernel of the timed region: K quantize kernels that also take the next
        # tensor's amax, and one amax kernel (timed alone above) for the first tensor
        t_fused = (ms - t_amax) / args.steps
        tq = t_fused
        kernel_key = f"{args.workload}:quantize_next"
        kernel_name += " + the next tensor's amax"
    achieved = alg / (tq * 1e-3) / 1e9
    clocks = clk.summary()
    traffic = profiled_traffic(kernel_key)
    hbm_roof = {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": traffic, "kernel": kernel_name,
                "peak_source": f"{peak_src} hbm_gbs (copy, burst) from MEASURED_PEAKS.json"}
    ops = ALU_OPS_PER_ELEMENT.get(obj or fmt)
    if ops is not None and had16:
        ops += ROTATION_OPS_PER_ELEMENT
    if ops is not None and fused:
        ops += 1   # the tensor maximum
    if ops is not None:
        # the candidate search is bound by plain FP32/convert arithmetic, not by HBM: the peak is
        # 148 SMs x 128 FP32 lanes x the SM clock sampled during the timed region
        mhz = clocks["sm_mhz"] or clocks["sm_max_mhz"] or 1965.0
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        alu_peak = sms * 128 * mhz * 1e6 / 1e9
        alu_ach = ops * rows * cols / (tq * 1e-3) / 1e9
        roofline = {"bound": "alu", "achieved": round(alu_ach, 1), "peak": round(alu_peak, 1), "unit": "Gop/s",
                    "frac": round(alu_ach / alu_peak, 4), "traffic": traffic, "kernel": kernel_name,
                    "ops_per_element": ops,
                    "peak_source": f"{sms} SMs x 128 FP32 lanes x {mhz:.0f} MHz (median SM clock in the timed region)",
                    "hbm": {k: hbm_roof[k] for k in ("achieved", "peak", "unit", "frac")}}
    else:
        roofline = hbm_roof
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(per_step_ms, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": desc, "rows": rows, "cols": cols, "input_dtype": w["dtype"],
                   "method": obj or fmt, "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": f"{nsets} rotating input/output buffer sets, {nsets * (in_bytes + out_bytes) / 2**20:.0f} MB "
                         f"total (at least 3x the 126 MB L2)",
                   "timing": ("one fp4q_quantize_batch call over the K steps' tensors (the buffer sets in turn), "
                              "captured as a CUDA graph: an amax kernel for the first tensor, then K quantize "
                              "kernels, each also taking the next tensor's amax" +
                              ("; the AbsMax kernel marks that read evict-last in L2, so the tensor's second read "
                               "(its quantization, one kernel later) comes mostly from L2" if obj == "absmax" else "") +
                              "; CUDA events on the launching stream" if fused else
                              "CUDA graph over the buffer sets (no timing nodes inside); each step's amax pass runs on "
                              "a second stream under the previous step's quantize kernel, each quantize after its own "
                              "amax; CUDA events on the launching stream" if two_pass else
                              "CUDA graph over the buffer sets (no timing nodes inside), replayed on one stream; CUDA "
                              "events on that stream")},
        "hbm_frac": round(value / world / peak, 4),
        "input_gbps": round(in_bytes * args.steps * world / (ms * 1e-3) / 1e9, 2),
        "elements_per_s": round(rows * cols * args.steps * world / (ms * 1e-3), 1),
        "kernels_ms": {"amax": (None if t_amax is None else round(t_amax, 5)), "quantize": round(t_q, 5),
                       "how": f"each kernel alone, {kernel_reps} launches over the rotating buffer sets, CUDA events",
                       **({"quantize_next_amax": round(t_fused, 5),
                           "how_next": "the timed region's K batched quantize kernels: (region - one amax) / K"}
                          if fused else {})},
        "step_ms": step_dist,
        "serial": {"value": round(alg * args.steps * world / (serial_ms * 1e-3) / 1e9, 2),
                   "ms_per_step": round(serial_ms / args.steps, 5),
                   "how": "the same steps with no overlap: amax then quantize per step on one stream"},
        **({"two_stream": {"value": round(alg * args.steps * world / (two_stream_ms * 1e-3) / 1e9, 2),
                           "ms_per_step": round(two_stream_ms / args.steps, 5),
                           "how": "the same steps as separate amax and quantize kernels, each amax on a second "
                                  "stream under the previous step's quantize"}} if fused else {}),
        "roofline": roofline,
        "device_status": st,
        "gpu_launches": args.steps + 1 if fused else launches_per_step * args.steps,
        "clocks": clocks,
        "e2e": {"value": round(alg / (e2e_ms * 1e-3) / 1e9 * world, 3), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4), "steps": e2e_steps,
                "launches_per_step": e2e_launches,
                "api": "HostQuantizer -> fp4q_quantize_host_async, 2 staging sets: each step's H2D (copy stream) "
                       "overlaps the previous step's kernels and D2H (compute stream)"},
    }
    if args.cpu_baseline and world == 1:
        # the oracle on every host core (reported), and single-threaded (nested); the
        # single-threaded run works at the whole tensor's S and checks the CUDA path's output
        # for the rows it covers (the line's correctness fields)
        c0, s0, g0 = outs[0]
        S_gpu = None if fmt.startswith("mxfp4") else float(g0.cpu().numpy()[0])
        single = cpu_baseline(w, fmt, obj, budget_s=args.cpu_seconds, S=S_gpu,
                              gpu=(c0.cpu().numpy(), s0.cpu().numpy()))
        line["parity"] = single.pop("parity")
        if S_gpu is not None:
            import oracle as O
            xo = O.widen_bf16(w["x"]) if w["dtype"] == "bf16" else w["x"]
            S_o = O.if6_tensor_scale(xo) if base == "if6" else O.tensor_scale(O.rotate16(xo) if had16 else xo)[0]
            line["parity"]["S_bit_exact"] = bool(np.float32(S_o).view(np.uint32) == np.float32(S_gpu).view(np.uint32))
        line["cpu_baseline"] = cpu_baseline_all_cores(w, fmt, obj, budget_s=args.cpu_seconds / 2)
        line["cpu_baseline"]["single_core"] = single
    print(json.dumps(line), flush=True)


def run_dequant(args, rank, world):
    """Dequantization throughput: codes + scales (+ S) -> fp32, one kernel per step, on the
    quantizer's own output for the workload's tensor, over rotating buffer sets."""
    import torch
    import torch.distributed as dist
    import fp4_block_scaled_nvfp4_b200 as fq
    from fp4_block_scaled_nvfp4_b200 import synth
    cfg, fmt, obj, desc = DEQUANT_WORKLOADS[args.workload]
    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    fq.lib()
    w = synth.make(cfg)
    rows, cols = w["rows"], w["cols"]
    x = device_tensor_from_bits(w["x"], torch).to(dev)
    codes, scales, gs = fq.quantize(x, fmt, obj or "absmax")
    B = fq.BLOCK[fmt]
    in_b = rows * cols // 2 + rows * cols // B + (4 if fmt != "mxfp4" else 0)
    out_b = rows * cols * 4
    alg = in_b + out_b
    nsets = max(2, int(np.ceil(3.0 * L2_BYTES / alg)))
    sets = [(codes.clone(), scales.clone(), None if gs is None else gs.clone(),
             torch.empty((rows, cols), dtype=torch.float32, device=dev)) for _ in range(nsets)]
    del x
    stream = torch.cuda.Stream(device=dev)

    def step(i):
        c, sc, g, o = sets[i % nsets]
        fq.dequantize(c, sc, g, fmt, out=o)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(nsets):
            step(i)
    with torch.cuda.stream(stream):
        graph.replay()
    torch.cuda.synchronize()
    cycles = max(1, args.steps // nsets)
    steps = cycles * nsets
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            start.record()
            for _ in range(cycles):
                graph.replay()
            end.record()
        end.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = start.elapsed_time(end) / steps
    if world > 1:
        t = torch.tensor([ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    # end to end through the public API: codes, scales (and S) from pinned host memory, the
    # dequantize call, the fp32 values back to pinned host memory, every step
    hosts = [t.cpu().pin_memory() for t in (codes, scales) + ((gs,) if gs is not None else ())]
    devs = [torch.empty_like(t, device=dev) for t in hosts]
    out_host = torch.empty((rows, cols), dtype=torch.float32, pin_memory=True)
    out_dev = torch.empty((rows, cols), dtype=torch.float32, device=dev)
    e_steps = max(1, min(args.steps, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record()
        for _ in range(e_steps):
            for h, d in zip(hosts, devs):
                d.copy_(h, non_blocking=True)
            fq.dequantize(devs[0], devs[1], devs[2] if gs is not None else None, fmt, out=out_dev)
            out_host.copy_(out_dev, non_blocking=True)
        e1.record()
    e1.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e_steps
    if rank != 0:
        return
    peak, peak_src = load_peaks()
    achieved = alg / (ms * 1e-3) / 1e9
    line = {"metric": DEQUANT_METRIC, "value": round(achieved * world, 2), "unit": "GB/s", "n_gpus": world,
            "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": desc, "rows": rows, "cols": cols, "format": fmt, "out_dtype": "fp32",
                       "parallelism": f"replicas{world}" if world > 1 else "single",
                       "l2": f"{nsets} rotating buffer sets, {nsets * alg / 2**20:.0f} MB total (> 3x the 126 MB L2)",
                       "timing": "CUDA graph over the buffer sets, replayed on one stream; CUDA events on that stream"},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": profiled_traffic(f"{args.workload}:dequant"),
                         "kernel": "dequant_mx_kernel" if fmt == "mxfp4" else "dequant16_kernel",
                         "peak_source": f"{peak_src} hbm_gbs (copy, burst) from MEASURED_PEAKS.json"},
            "kernels_ms": {"dequantize": round(ms, 5)},
            "gpu_launches": steps, "clocks": clk.summary(),
            "e2e": {"value": round(alg / (e2e_ms * 1e-3) / 1e9 * world, 3), "unit": "GB/s",
                    "h2d_bytes_per_step": int(sum(h.numel() * h.element_size() for h in hosts)),
                    "d2h_bytes_per_step": out_b, "ms_per_step": round(e2e_ms, 4), "steps": e_steps,
                    "api": "codes, scales and S from pinned host memory, fp4q_dequantize, fp32 values back"}}
    if args.cpu_baseline and world == 1:
        import oracle as O
        hc, hs = hosts[0].numpy(), hosts[1].numpy()
        S = float(hosts[2].numpy()[0]) if gs is not None else 0.0
        got = sets[0][3].cpu().numpy()
        done, t0 = 0, time.perf_counter()
        chunk = 256
        same = True
        while done < rows and time.perf_counter() - t0 < args.cpu_seconds:
            ref = O.dequantize(hc[done:done + chunk], hs[done:done + chunk], S, fmt)
            same &= bool(np.array_equal(ref.view(np.uint32), got[done:done + chunk].view(np.uint32)))
            done += ref.shape[0]
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": round(done * cols * (alg / (rows * cols)) / dt / 1e9, 4), "unit": "GB/s",
                                "cores": 1, "kind": "oracle",
                                "sample": f"{done} of {rows} rows dequantized single-threaded, {dt:.1f} s"}
        line["parity"] = {"rows_checked": done, "bit_exact": same,
                          "how": "the CUDA path's fp32 values of the sampled rows against the oracle's decoder"}
    print(json.dumps(line), flush=True)


def fp4_peak_tflops():
    """Dense FP4 tensor peak: the measured bf16 GEMM peak times the nominal FP4 / bf16 ratio (4)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return 4.0 * float(json.load(f)["bf16_tflops"]), "measured bf16_tflops (burst) x 4, the nominal FP4/bf16 ratio"
    return 4.0 * 1590.0, "fallback bf16 1.59 PFLOP/s x 4"


def gemm_operands(torch, fq, synth, dev, mx=False):
    M, N, K = GEMM_SHAPE
    wa = synth.make("cfg3", rows=M, cols=K)
    wb = synth.make("cfg2", rows=N, cols=K)
    xa = device_tensor_from_bits(wa["x"], torch).to(dev)
    xb = device_tensor_from_bits(wb["x"], torch).to(dev)
    if mx:
        # MXFP4 with the 32-point rotation on both operands (it cancels in the product)
        qa = fq.hadamard_quantize(xa, tiled_scales=True)[:2]
        qb = fq.hadamard_quantize(xb, tiled_scales=True)[:2]
    else:
        qa = fq.quantize(xa, "nvfp4", "sweep_mse", tiled_scales=True)
        qb = fq.quantize(xb, "nvfp4", "sweep_mse", tiled_scales=True)
    return (M, N, K), qa, qb, wa, wb


def run_reference_gemm(args, rank, world):
    """The oracle's float64 NVFP4 product on the host: each step 16 activation rows times a
    1024-row slice of the weight."""
    from fp4_block_scaled_nvfp4_b200 import synth
    import oracle as O
    if rank != 0:
        return
    M, N, K = GEMM_SHAPE
    mx = args.workload == "gemm_mx"
    if args.workload == "gemm_dyn":
        print(json.dumps({"impl": "reference", "unavailable": "the dynamic GEMM line has no CPU arm; the oracle's "
                          "quantize and GEMM are timed by the quantize and gemm workloads"}), flush=True)
        return
    wa = synth.make("cfg3", rows=16 * max(1, args.steps + args.warmup), cols=K)
    wb = synth.make("cfg2", rows=1024, cols=K)
    if mx:
        ra = O.mxfp4_quantize(O.widen_bf16(wa["x"]), hadamard=True)
        rb = O.mxfp4_quantize(O.widen_bf16(wb["x"]), hadamard=True)
    else:
        ra = O.nvfp4_quantize(O.widen_bf16(wa["x"]), "sweep_mse")
        rb = O.nvfp4_quantize(O.widen_bf16(wb["x"]), "sweep_mse")
    def step(i):
        sl = slice(16 * i, 16 * i + 16)
        if mx:
            O.mxfp4_gemm(ra["codes"][sl], ra["scales"][sl], rb["codes"], rb["scales"])
        else:
            O.nvfp4_gemm(ra["codes"][sl], ra["scales"][sl], ra["S"], rb["codes"], rb["scales"], rb["S"])
    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = time.perf_counter() - t0
    val = 2.0 * 16 * 1024 * K * args.steps / dt / 1e12
    line = {"impl": "reference", "metric": GEMM_MX_METRIC if mx else GEMM_METRIC, "value": round(val, 6),
            "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": ("MXFP4 (rotated)" if mx else "NVFP4") + " GEMM on the oracle", "M": M, "N": N,
                       "K": K, "step_sample": "16 x 1024 x K"},
            "cpu_baseline": {"value": round(val, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": "16 activation rows times 1024 weight rows per step (the float64 matmul on "
                                       "the BLAS threads counted in cores)"},
            "e2e": {"value": round(val, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_gemm(args, rank, world):
    import torch
    import fp4_block_scaled_nvfp4_b200 as fq
    from fp4_block_scaled_nvfp4_b200 import synth
    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    fq.lib()
    mx = args.workload == "gemm_mx"
    dyn = args.workload == "gemm_dyn"
    out_bf16 = args.workload in ("gemm_bf16", "gemm_dyn")
    gemm = fq.mxfp4_gemm if mx else fq.nvfp4_gemm
    (M, N, K), qa, qb, wa, wb = gemm_operands(torch, fq, synth, dev, mx=mx)
    d = torch.empty((M, N), dtype=torch.bfloat16 if out_bf16 else torch.float32, device=dev)
    ws = fq.new_workspace(dev)
    stream = torch.cuda.Stream(device=dev)
    if dyn:
        # the activation in bf16, quantized every step into qa's buffers (S, codes, tiled scales)
        xa = device_tensor_from_bits(wa["x"], torch).to(dev)
        ws_q = fq.new_workspace(dev)

        def one_step():
            fq.global_scale(xa, out=qa[2], workspace=ws_q)
            fq.quantize(xa, "nvfp4", "sweep_mse", global_scale=qa[2], out=qa, workspace=ws_q, tiled_scales=True)
            gemm(qa, qb, out=d, workspace=ws)
    else:
        def one_step():
            gemm(qa, qb, out=d, workspace=ws)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            one_step()
    torch.cuda.synchronize()
    flops = 2.0 * M * N * K
    steps = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            start.record()
            for _ in range(steps):
                one_step()
            end.record()
        end.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = start.elapsed_time(end) / steps
    if world > 1:
        t = torch.tensor([ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    st = fq.read_device_status(ws)
    gemm_only_ms = ms
    if dyn:   # the GEMM alone on the same operands, for the split of the step
        st = st or fq.read_device_status(ws_q)
        with torch.cuda.stream(stream):
            start.record()
            for _ in range(steps):
                gemm(qa, qb, out=d, workspace=ws)
            end.record()
        end.synchronize()
        gemm_only_ms = start.elapsed_time(end) / steps
    # end to end through the public API: operands (codes, tiled scales, S) copied in from pinned
    # host memory, the GEMM, and the fp32 product copied back, every step
    hosts = [t.cpu().pin_memory() for t in (*qa, *qb)]
    d_host = torch.empty((M, N), dtype=d.dtype, pin_memory=True)
    devs = [torch.empty_like(t, device=dev) for t in hosts]
    e_steps = max(1, min(steps, 5))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record()
        for _ in range(e_steps):
            for h, g in zip(hosts, devs):
                g.copy_(h, non_blocking=True)
            na = len(qa)
            gemm(tuple(devs[:na]), tuple(devs[na:]), out=d, workspace=ws)
            d_host.copy_(d, non_blocking=True)
        e1.record()
    e1.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e_steps
    if world > 1:
        t = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    if rank != 0:
        return
    peak, peak_src = fp4_peak_tflops()
    tf = flops / (ms * 1e-3) / 1e12
    out_desc = "bf16 out" if out_bf16 else "fp32 out"
    workload = ("MXFP4 GEMM, activations 8192x4096 (activation workload) times weight 14336x4096 (Student-t), both "
                "rotated by the 32-point block Hadamard, K contiguous, tiled E8M0 scales, fp32 out") if mx else (
               "NVFP4 GEMM, activations 8192x4096 (activation workload, sweep-MSE) times weight 14336x4096 "
               f"(Student-t, sweep-MSE), K contiguous, tiled scales, {out_desc}")
    if dyn:
        workload = ("per step: amax + ScaleSweep-MSE quantization of the bf16 activation 8192x4096 (tiled scales), "
                    "then the NVFP4 GEMM against the pre-quantized 14336x4096 weight, bf16 out")
    line = {"metric": GEMM_DYN_METRIC if dyn else (GEMM_MX_METRIC if mx else GEMM_METRIC), "value": round(tf * world, 1),
            "unit": "TFLOP/s", "n_gpus": world, "steps": steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e2m1xe2m1->" + ("bf16" if out_bf16 else "f32"), "data": "synthetic",
            "config": {"workload": workload,
                       "M": M, "N": N, "K": K, "parallelism": f"replicas{world}" if world > 1 else "single",
                       "l2": "operands 46 MB stay L2-resident across steps (a GEMM reuses them by design)",
                       "timing": "CUDA events around back-to-back launches on one stream"},
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": round(peak, 1), "unit": "TFLOP/s",
                         "frac": round(tf / peak, 4), "traffic": profiled_traffic(f"{args.workload}:gemm", GEMM_SOURCES),
                         "kernel": f"fp4_gemm_kernel<{'true' if mx else 'false'}>",
                         "peak_source": peak_src},
            "device_status": st, "gpu_launches": steps * (3 if dyn else 1), "clocks": clk.summary(),
            "e2e": {"value": round(flops / (e2e_ms * 1e-3) / 1e12 * world, 3), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": int(sum(h.numel() * h.element_size() for h in hosts)),
                    "d2h_bytes_per_step": M * N * 4, "ms_per_step": round(e2e_ms, 3), "steps": e_steps,
                    "api": f"operands from pinned host memory, fp4q_{'mx' if mx else 'nv'}fp4_gemm, product back to "
                           "pinned host memory"}}
    if args.cpu_baseline:
        import oracle as O
        if mx:
            ra = O.mxfp4_quantize(O.widen_bf16(wa["x"][:64]), hadamard=True)
            rb = O.mxfp4_quantize(O.widen_bf16(wb["x"]), hadamard=True)
            t0 = time.perf_counter()
            O.mxfp4_gemm(ra["codes"], ra["scales"], rb["codes"], rb["scales"])
        else:
            ra = O.nvfp4_quantize(O.widen_bf16(wa["x"][:64]), "sweep_mse", S=float(qa[2].cpu()[0]))
            rb = O.nvfp4_quantize(O.widen_bf16(wb["x"]), "sweep_mse")
            t0 = time.perf_counter()
            O.nvfp4_gemm(ra["codes"], ra["scales"], ra["S"], rb["codes"], rb["scales"], rb["S"])
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": round(2.0 * 64 * N * K / dt / 1e12, 6), "unit": "TFLOP/s",
                                "cores": blas_threads(),
                                "kind": "oracle", "sample": f"64 of {M} activation rows times the whole weight, "
                                                            f"float64 matmul of the decoded operands on the BLAS threads counted "
                                                            f"in cores, {dt:.1f} s"}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + list(GEMM_WORKLOADS) + sorted(DEQUANT_WORKLOADS),
                    default="cfg3")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1 and args.impl == "ours":
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        elif args.workload in GEMM_WORKLOADS:
            run_gemm(args, rank, world)
        elif args.workload in DEQUANT_WORKLOADS:
            run_dequant(args, rank, world)
        else:
            run_ours(args, rank, world)
    finally:
        if world > 1 and args.impl == "ours":
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
