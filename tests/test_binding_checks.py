"""The Python binding rejects bad tensors before any call into the library (no GPU needed):
host tensors, unknown format or objective names, missing outputs.  On the GPU the same
checks cover wrong devices, dtypes and sizes (tests/test_gpu_host.py)."""
import pytest

torch = pytest.importorskip("torch")

import fp4_block_scaled_nvfp4_b200 as fq


def test_unknown_names_raise():
    x = torch.zeros(4, 32)
    with pytest.raises(fq.Fp4qError, match="objective"):
        fq.quantize(x, "nvfp4", "sweep-mse")
    with pytest.raises(fq.Fp4qError, match="format"):
        fq.quantize(x, "nvfp5", "sweep_mse")
    with pytest.raises(fq.Fp4qError, match="objective"):
        fq.quantize_noalloc(x, "nvfp4", "weighted")


def test_host_tensors_raise():
    x = torch.zeros(4, 32)
    with pytest.raises(fq.Fp4qError, match="CUDA"):
        fq.quantize(x, "nvfp4", "absmax")
    with pytest.raises(fq.Fp4qError, match="CUDA"):
        fq.hadamard_quantize(x)
    with pytest.raises(fq.Fp4qError, match="CUDA"):
        fq.global_scale(x)
    with pytest.raises(fq.Fp4qError, match="CUDA"):
        fq.encode(x, "e2m1")
    codes = torch.zeros(4, 16, dtype=torch.uint8)
    scales = torch.zeros(4, 2, dtype=torch.uint8)
    with pytest.raises(fq.Fp4qError, match="CUDA"):
        fq.dequantize(codes, scales, torch.ones(1), "nvfp4")
    with pytest.raises(fq.Fp4qError, match="CUDA"):
        fq.nvfp4_gemm((codes, scales, torch.ones(1)), (codes, scales, torch.ones(1)))


def test_noalloc_needs_outputs():
    x = torch.zeros(4, 32)
    with pytest.raises(fq.Fp4qError):
        fq.quantize_noalloc(x, "nvfp4", "absmax", out=None)


def test_batch_rejects_before_the_library():
    x = torch.zeros(4, 32)
    with pytest.raises(fq.Fp4qError, match="nvfp4 or if4"):
        fq.quantize_batch([x], "mxfp4")
    with pytest.raises(fq.Fp4qError, match="nvfp4 or if4"):
        fq.quantize_batch([x], "if6")
    with pytest.raises(fq.Fp4qError, match="objective"):
        fq.quantize_batch([x], "nvfp4", "sweep-mse")
    with pytest.raises(fq.Fp4qError, match="one entry per tensor"):
        fq.quantize_batch([x, x], "nvfp4", global_scales=[torch.ones(1)])
    with pytest.raises(fq.Fp4qError, match="CUDA"):
        fq.quantize_batch([x], "nvfp4", "absmax")
    assert fq.quantize_batch([], "nvfp4") == []
