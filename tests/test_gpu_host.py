"""GPU parity of the host-memory entry point (fp4q_quantize_host_async via HostQuantizer).

Several calls are kept in flight over two staging sets, each with its own input tensor and
host outputs; after one synchronize every call's codes, scales and S must equal the
oracle's for its own input, bit for bit.  This checks the copy-in / compute / copy-out
ordering between the copy stream and the compute stream (an input overwritten before its
kernels ran, or outputs copied before the kernels finished, shows up as a mismatch).
"""
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


def oracle_for(x, fmt, obj):
    base, had = (fmt[:-4], True) if fmt.endswith("_had") else (fmt, False)
    if base == "nvfp4":
        return O.nvfp4_quantize(x, obj, hadamard16=had)
    if base == "if4":
        return O.if4_quantize(x, hadamard16=had)
    return O.mxfp4_quantize(x, hadamard=had)


@pytest.mark.parametrize("fmt,obj", [("nvfp4", "sweep_mse"), ("nvfp4", "absmax"), ("if4", None), ("mxfp4", None),
                                     ("nvfp4_had", "sweep_mse"), ("if4_had", None), ("mxfp4_had", None)])
def test_pipelined_host_calls(fmt, obj):
    rows, cols, calls = 64, 2048, 5
    inputs = [synth.make("cfg3", rows=rows, cols=cols, seed=100 + i) for i in range(calls)]
    hq = fq.HostQuantizer(rows, cols, fmt, obj or "absmax", dtype=torch.bfloat16, depth=2)
    pinned = [torch.from_numpy(w["x"].view(np.int16)).view(torch.bfloat16).pin_memory() for w in inputs]
    outs = [hq(p, fq.alloc_host_outputs(rows, cols, fmt)) for p in pinned]
    assert fq.last_launch_count() == (1 if fmt.startswith("mxfp4") else 2)
    hq.synchronize()
    for w, (hc, hs, hg) in zip(inputs, outs):
        r = oracle_for(O.widen_bf16(w["x"]), fmt, obj)
        assert np.array_equal(hs.numpy(), r["scales"])
        assert np.array_equal(hc.numpy(), r["codes"])
        if hg is not None:
            assert np.float32(hg.numpy()[0]).view(np.uint32) == np.float32(r["S"]).view(np.uint32)
    for st in hq.sets:
        assert fq.read_device_status(st["ws"]) == 0


def test_one_shot_quantize_host_wmse():
    w = synth.make("cfg2", rows=24, cols=4096)
    imp = torch.from_numpy(w["importance"]).cuda()
    x = torch.from_numpy(w["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
    hc, hs, hg = fq.quantize_host(x, "nvfp4", "sweep_wmse", importance=imp)
    r = O.nvfp4_quantize(O.widen_bf16(w["x"]), "sweep_wmse", importance=w["importance"])
    assert np.array_equal(hs.numpy(), r["scales"]) and np.array_equal(hc.numpy(), r["codes"])
    assert np.float32(hg.numpy()[0]).view(np.uint32) == np.float32(r["S"]).view(np.uint32)
