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


def test_if6_algorithmic_bytes():
    # IF6: 6-bit codes (12 bytes per 16-element block), one scale byte per block, S
    n = 4096 * 14336
    assert bench.algorithmic_bytes(4096, 14336, "if6") == 2 * n + n * 3 // 4 + n // 16 + 4


def test_reference_arm_prints_the_contract_line(capsys):
    # the reference arm (the oracle on the host) on the default workload: one JSON line with the
    # keys the driver reads, its own cpu_baseline and a zero-copy e2e of the same value
    import argparse
    import json
    args = argparse.Namespace(workload="cfg3", steps=2, warmup=1, impl="reference", gpus=1, cpu_baseline=True,
                              cpu_seconds=1.0)
    bench.run_reference(args, 0, 1)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["metric"] == bench.METRIC and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["value"] == line["value"] and line["e2e"]["h2d_bytes_per_step"] == 0
