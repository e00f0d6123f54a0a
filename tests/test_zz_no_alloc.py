"""fp4q_quantize_noalloc: the quantize entry point for callers that cannot allocate device
memory (code running inside someone else's stream capture or memory pool, plugins handed
only their tensors, engines that plan every allocation up front).  It keeps its scratch in
a small array built into the library instead of a caller workspace.

Checked through the C ABI against fp4q_quantize (the workspace entry point), bit for bit,
on two calls in a row; the second call must not see anything the first one left behind.
This file is collected last on purpose and also passes on its own in a fresh process.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import fp4_block_scaled_nvfp4_b200 as fq
from fp4_block_scaled_nvfp4_b200 import synth


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fq.lib()


def _dev(w):
    if w["dtype"] == "bf16":
        return torch.from_numpy(w["x"].view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(w["x"])).cuda()


CASES = [("cfg3", 64, 4096, "nvfp4", "sweep_mse"), ("cfg2", 24, 4096, "nvfp4", "sweep_wmse"),
         ("cfg1", None, None, "nvfp4", "four_over_six"), ("cfg4", 16, 14336, "if4", None),
         ("cfg5", 16, 8192, "mxfp4", None)]


@pytest.mark.parametrize("cfg,rows,cols,fmt,obj", CASES)
def test_noalloc_matches_workspace_entry_point(cfg, rows, cols, fmt, obj):
    w = synth.make(cfg, rows=rows, cols=cols)
    x = _dev(w)
    imp = torch.from_numpy(w["importance"]).cuda() if obj == "sweep_wmse" else None
    ref = fq.quantize(x, fmt, obj or "absmax", importance=imp, workspace=fq.new_workspace())
    torch.cuda.synchronize()
    R, C = x.shape
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for call in range(2):   # two calls in a row share the built-in scratch
        out = fq.alloc_outputs(R, C, fmt)
        got = fq.quantize_noalloc(x, fmt, obj or "absmax", importance=imp, out=out, device_status=st)
        torch.cuda.synchronize()
        assert torch.equal(got[0], ref[0]), f"codes differ on call {call}"
        assert torch.equal(got[1], ref[1]), f"scales differ on call {call}"
        if fmt != "mxfp4":
            assert got[2].view(torch.int32).item() == ref[2].view(torch.int32).item()
        assert st.item() == fq.DEVSTAT_OK


def test_noalloc_status_is_per_call_and_memory_stays_put():
    bad = torch.randn(4, 64, device="cuda")
    bad[1, 3] = float("nan")
    good = torch.randn(4, 64, device="cuda")
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    out = fq.alloc_outputs(4, 64, "nvfp4")
    fq.quantize_noalloc(bad, "nvfp4", "sweep_mse", out=out, device_status=st)
    torch.cuda.synchronize()
    assert st.item() == fq.DEVSTAT_NONFINITE
    assert not out[0].any() and not out[1].any()
    free_before = torch.cuda.mem_get_info()[0]
    allocs_before = torch.cuda.memory_stats().get("allocation.all.allocated", 0)
    fq.quantize_noalloc(good, "nvfp4", "sweep_mse", out=out, device_status=st)
    torch.cuda.synchronize()
    assert st.item() == fq.DEVSTAT_OK
    ref = fq.quantize(good, "nvfp4", "sweep_mse", workspace=fq.new_workspace())
    torch.cuda.synchronize()
    assert torch.equal(out[0], ref[0]) and torch.equal(out[1], ref[1])
    allocs_ref = torch.cuda.memory_stats().get("allocation.all.allocated", 0)   # after quantize()'s workspace
    for _ in range(3):
        fq.quantize_noalloc(good, "nvfp4", "sweep_mse", out=out)
    torch.cuda.synchronize()
    # no allocation through torch's allocator, and the device's free memory did not drop by a
    # driver granule (2 MiB); other processes on the GPU may move it by less or upwards
    assert torch.cuda.memory_stats().get("allocation.all.allocated", 0) == allocs_ref
    assert torch.cuda.mem_get_info()[0] > free_before - (2 << 20)


def test_noalloc_empty_tensor_reports_ok():
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    x = torch.zeros(0, 64, device="cuda")
    out = fq.alloc_outputs(0, 64, "nvfp4")
    fq.quantize_noalloc(x, "nvfp4", "sweep_mse", out=out, device_status=st)
    torch.cuda.synchronize()
    assert st.item() == fq.DEVSTAT_OK


def test_noalloc_rejects_like_quantize():
    L = fq.lib()
    fake = 0x10000
    assert L.fp4q_quantize_noalloc(fake, 1, 4, 24, 24, 0, 2, None, fake, fake, fake, None, 0, None) == fq.ERR_SHAPE
    assert L.fp4q_quantize_noalloc(fake + 8, 1, 4, 32, 32, 0, 2, None, fake, fake, fake, None, 0, None) == fq.ERR_ALIGNMENT
    assert L.fp4q_quantize_noalloc(fake, 1, 1 << 30, 1 << 12, 1 << 12, 0, 2, None, fake, fake, fake, None, 0,
                                   None) == fq.ERR_SHAPE
    assert L.fp4q_quantize_noalloc(None, 1, 0, 32, 32, 0, 2, None, None, None, None, None, 0, None) == fq.OK
