"""Host-side accounting of bench.py (no GPU): the algorithmic bytes per step that every GB/s
figure divides by, against the per-configuration byte counts of the measurement contract
(input + codes + scales + S, + the importance vector for WMSE; MXFP4 has no S), and the
operation counts behind the ALU roofline."""
import pytest

import bench

# rows, cols, format, input bytes per element, WMSE, the contract's byte count per step
CASES = [
    (256, 1024, "nvfp4", 4, False, 1_196_036),          # cfg1: fp32 input
    (14336, 4096, "nvfp4", 2, True, 150_487_044),       # cfg2: WMSE, importance[4096]
    (8192, 4096, "nvfp4", 2, False, 85_983_236),        # cfg3
    (4096, 14336, "if4", 2, False, 150_470_660),        # cfg4
    (16384, 8192, "mxfp4", 2, False, 339_738_624),      # cfg5 (no tensor scale)
    (16384, 8192, "mxfp4_had", 2, False, 339_738_624),  # cfg5 with the rotation: same bytes
]


@pytest.mark.parametrize("rows,cols,fmt,in_bytes,wmse,want", CASES)
def test_algorithmic_bytes_match_the_contract(rows, cols, fmt, in_bytes, wmse, want):
    assert bench.algorithmic_bytes(rows, cols, fmt, in_bytes=in_bytes, wmse=wmse) == want


def test_every_bench_workload_has_a_shape_and_method():
    for name, (cfg, fmt, obj, desc) in bench.WORKLOADS.items():
        assert cfg.startswith("cfg") and fmt and desc
    assert "cfg3" in bench.WORKLOADS and set(bench.GEMM_WORKLOADS) == {"gemm", "gemm_mx", "gemm_bf16", "gemm_dyn"}
